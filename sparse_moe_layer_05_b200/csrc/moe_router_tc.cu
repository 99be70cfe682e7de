// moe_router_tc.cu -- the router on the tensor cores, with the top-k and the
// selected-set softmax in the same kernel, for every batch size.
//
//   s[t][e] = sum_i x[t][i] W_r[e][i] + b_r[e]
//   then top-k over e (lower index first on ties) and the softmax over the k
//   selected logits
// ("llm-surgery-dark-arts-gpt-oss-40b-64a8-init", section 2, "Proof": s_i =
// W_r[i].h + b_r[i], i in top-k(s), p_i = exp(s_i) / sum over the selected set.)
//
// Precision. x is bf16, so it enters a kind::f16 UMMA exactly. The fp32
// router weights are split once per call into three bf16 terms,
// hi = bf16(W), mid = bf16(W - hi), lo = W - hi - mid (each rounding to nearest
// even): an fp32 value has 24 significant bits and each term holds the next 8,
// so hi + mid + lo = W exactly (for |W| >= 2^-101, where no term is subnormal).
// Each product of x with a term is exact in fp32. The x.hi products go to one
// TMEM accumulator and the x.mid and x.lo products (2^-8 and 2^-16 of the
// logit's size) to a second, so the accumulator that carries the logit's
// magnitude sees d/16 accumulation steps, not 3d/16. The logit is
// hi_acc + lo_acc (+ the partial sums of the other CTAs of the cluster, in
// rank order) + b_r, in fp32. Every expert's column goes through the same
// operations, so identical router rows give identical logits.
//
// Near ties. The tensor core's fp32 accumulation differs from exact
// arithmetic by a small multiple of fp32 rounding of the running sums. For
// token t the kernel takes tau_t = 2^-17 ||x_t||_2 max_e ||W_r[e]||_2 (by
// Cauchy-Schwarz every partial sum of x_t . W_r[e] is at most
// ||x_t|| ||W_r[e]|| in size, and 2^-17 of it is far above the error of
// d/16 fp32 roundings of sums of that size for d <= 16384): where two
// neighbouring logits of the top-k list (or the k-th and a runner-up) lie
// within tau_t, their order is decided on fp64 dot products of the original
// bf16 x and fp32 W_r (moe_topk.cuh), which equal the exact values to about
// 1e-13 relative. Everywhere else the fp32 order is the exact order.
//
// Tiles. One cluster of C CTAs (C = 1, 2, 4 or 8) per 128 tokens (UMMA
// M = 128): CTA r of the cluster contracts k-blocks [r KB / C, (r+1) KB / C)
// of d (64 elements per block) for all experts at once (N = E rounded up to
// 16, at most 256), up to eight shared-memory stages: the x tile by one TMA
// box, the three weight terms by one 3-D box. Twelve UMMAs per stage (4 K
// steps x 3 terms). C grows while the grid stays within one wave of the SMs,
// so small batches (decode) spread d over eight SMs and large ones keep one
// CTA per token tile. While the UMMAs run, the epilogue warps add up
// ||x_t||^2 of their token rows from the same stages. At the end each CTA
// writes its partial logits to shared memory; after a cluster barrier CTA r
// finishes rows [r 128 / C, (r+1) 128 / C): it adds the C partials (through
// distributed shared memory, in rank order) and the bias, writes the logits,
// and one warp per token selects its k experts.
//
// Roles (256 threads): warp 0 TMA producer, warp 1 TMEM allocation and UMMA
// issue, warps 4-7 row norms, then TMEM -> shared memory; after the cluster
// barrier all threads sum the partials of this CTA's rows (in place) and all
// eight warps run the top-k. Every wait is bounded (moe_ptx.cuh); every CTA reaches both
// cluster barriers on every path.
#include <cuda_bf16.h>
#include <float.h>
#include <stdint.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"
#include "moe_perm_small.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int RT_M = 128;                 // tokens per cluster
constexpr int RT_BK = 64;                 // d elements per stage (128 bytes of bf16)
constexpr int RT_MAX_STAGES = 8;
constexpr int RT_MAX_CLUSTER = 8;
constexpr int RT_THREADS = 256;
constexpr int RT_SMEM_LIMIT = 232448 - 1024;
constexpr int RT_FIXED = 1024;            // barriers, TMEM address, flags
// the refinement margin tau_t relative to ||x_t|| max_e ||W_r[e]|| (2^-17)
constexpr float kRefineRel = 7.62939453125e-06f;

// The top-k kernel queues each token's refinements in shared memory and
// computes them with the whole block: each fp64 dot product is split over
// all 256 threads, so a refinement costs one pass of loads instead of a
// warp's chain of them. A token with more than RJ_PER_WARP of them refines
// alone.
constexpr int RJ_PER_WARP = 64;           // queued dot products per token
struct RefineReq {
  int row, m, pad0, pad1;
  unsigned long long refine_m, copy_m;
  double val[64];
  int cidx[64];
};
constexpr int TK_WARPS = 8;               // tokens per block of the top-k kernel

struct RouterTcShape {
  int npad;          // E rounded up to 16
  int nacc;          // TMEM accumulators: 3 (hi, mid, lo) or 2 (hi, mid + lo)
  int per;           // weight terms per UMMA (their B rows and accumulators are adjacent)
  int stage_bytes;   // x tile + three weight-term tiles
  int stages;
  int ld;            // floats per partial-logits row in shared memory
  int tmem_cols;
  int body;          // stages, or the partial logits and row norms after them
  int smem_alloc;
};

RouterTcShape router_tc_shape(int E) {
  RouterTcShape s;
  s.npad = (E + 15) / 16 * 16;
  s.stage_bytes = RT_M * 128 + 3 * s.npad * 128;
  s.ld = s.npad + 4;
  const int partial_bytes = RT_M * s.ld * 4 + RT_M * 4;
  int st = (RT_SMEM_LIMIT - RT_FIXED - 1024) / s.stage_bytes;
  if (st > RT_MAX_STAGES) st = RT_MAX_STAGES;
  s.stages = st;
  s.body = st * s.stage_bytes;
  if (s.body < partial_bytes) s.body = (partial_bytes + 1023) / 1024 * 1024;
  s.nacc = 3 * s.npad <= 512 ? 3 : 2;
  s.per = s.nacc == 3 ? (256 / s.npad < 3 ? 256 / s.npad : 3) : 1;
  int cols = 32;
  while (cols < s.nacc * s.npad) cols *= 2;
  s.tmem_cols = cols;
  s.smem_alloc = s.body + RT_FIXED + 1024;
  return s;
}

// W_r [E][d] fp32 -> terms [3][npad][d] bf16 (rows E..npad-1 zero),
// norms[npad] = ||W_r[e]||_2 (fp32, in one fixed order; 0 for the padding
// rows) and fps[npad], a 64-bit fingerprint of each row and its bias (sum of
// bits(w_i) (2i + 1) plus bits(b) times an odd constant, mod 2^64): rows with
// equal weights and bias (the copies of a silent-init layer) get equal
// fingerprints. One block per row.
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ W_r,
                                                           const float* __restrict__ b_r, int E,
                                                           int npad, int d,
                                                           uint16_t* __restrict__ terms,
                                                           float* __restrict__ norms,
                                                           unsigned long long* __restrict__ fps,
                                                           int* status, int* done_blocks) {
  pdl_wait_and_trigger();
  // the first kernel of the pass clears the status word and the top-k
  // kernel's count of finished blocks
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (status) *status = 0;
    *done_blocks = 0;
  }
  const int row = blockIdx.x;
  const size_t n = static_cast<size_t>(npad) * d;
  const size_t base = static_cast<size_t>(row) * d;
  float ss = 0.f;
  unsigned long long fp = 0ull;
  for (int i = threadIdx.x * 4; i < d; i += 256 * 4) {
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < E) w = __ldg(reinterpret_cast<const float4*>(W_r + base + i));
    const float wv[4] = {w.x, w.y, w.z, w.w};
    uint16_t h[4], m[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(wv[j]);
      const float r1 = wv[j] - __bfloat162float(hi);
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
      h[j] = __bfloat16_as_ushort(hi);
      m[j] = __bfloat16_as_ushort(mid);
      l[j] = __bfloat16_as_ushort(lo);
      ss = fmaf(wv[j], wv[j], ss);
      fp += static_cast<unsigned long long>(__float_as_uint(wv[j])) *
            static_cast<unsigned long long>(2 * (i + j) + 1);
    }
    *reinterpret_cast<uint2*>(terms + base + i) =
        make_uint2(h[0] | (uint32_t(h[1]) << 16), h[2] | (uint32_t(h[3]) << 16));
    *reinterpret_cast<uint2*>(terms + n + base + i) =
        make_uint2(m[0] | (uint32_t(m[1]) << 16), m[2] | (uint32_t(m[3]) << 16));
    *reinterpret_cast<uint2*>(terms + 2 * n + base + i) =
        make_uint2(l[0] | (uint32_t(l[1]) << 16), l[2] | (uint32_t(l[3]) << 16));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
    fp += __shfl_xor_sync(0xFFFFFFFFu, fp, off);
  }
  __shared__ float red[8];
  __shared__ unsigned long long redf[8];
  if ((threadIdx.x & 31) == 0) {
    red[threadIdx.x >> 5] = ss;
    redf[threadIdx.x >> 5] = fp;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    unsigned long long f = row < E ? static_cast<unsigned long long>(__float_as_uint(b_r[row])) *
                                         0x9E3779B97F4A7C15ull
                                   : 0ull;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      s += red[w];
      f += redf[w];
    }
    norms[row] = sqrtf(s);
    fps[row] = f;
  }
}

struct RouterTcArgs {
  const float* b_r;
  int T, E, d, npad, nacc, per, stages, ld, stage_bytes, body, tmem_cols, KB;
  float* logits;   // [T][E]
  float* xsq;      // [T]: ||x_t||^2
  int* status;
};

// Wait for an mbarrier phase regardless of the abort flag, at most
// kWaitLimitNs (used only on the way out after a wait gave up).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float4 ld_shared_cluster_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__global__ void __launch_bounds__(RT_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const RouterTcArgs args) {
  pdl_wait_and_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = args.stages;
  const uint32_t bar0 = sbase + args.body;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (RT_MAX_STAGES + s); };
  const uint32_t bar_acc = bar0 + 8u * (2 * RT_MAX_STAGES);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + args.body + 8 * (2 * RT_MAX_STAGES + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  // after the main loop: partial logits [128][ld] and ||x||^2 partials [128]
  float* partial = reinterpret_cast<float*>(smem);
  float* xsq_part = partial + RT_M * args.ld;

  const uint32_t rank = cluster_ctarank();
  uint32_t csize;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(csize));
  const int tile = static_cast<int>(blockIdx.x / csize);
  const int t0 = tile * RT_M;
  const int kb0 = static_cast<int>(rank) * args.KB / static_cast<int>(csize);
  const int kb1 = (static_cast<int>(rank) + 1) * args.KB / static_cast<int>(csize);
  const int nkb = kb1 - kb0;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    misc[2] = misc[3] = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1 + 4);   // the UMMA commit and the four norm warps
    }
    mbar_init(bar_acc, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), static_cast<uint32_t>(args.tmem_cols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  const uint32_t npad_u = static_cast<uint32_t>(args.npad);
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0, ph = 0, issued = 0;
      const uint32_t tx = static_cast<uint32_t>(args.stage_bytes);
      for (int i = 0; i < nkb; ++i) {
        if (!(ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, args.status))) break;
        const uint32_t st = sbase + s * args.stage_bytes;
        const int kx = (kb0 + i) * RT_BK;
        mbar_expect_tx(bar_full(s), tx);
        tma_load_2d(st, &tmX, kx, t0, bar_full(s));
        tma_load_3d(st + RT_M * 128, &tmW, kx, 0, 0, bar_full(s));
        issued = i + 1;
        if (++s == S) { s = 0; ph ^= 1; }
      }
      misc[2] = static_cast<uint32_t>(issued);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // three accumulators: terms t .. t + per - 1 in one UMMA (their B rows
      // and accumulator columns are adjacent); two: hi, then mid and lo into
      // the second
      const uint32_t idesc1 = idesc_bf16_f32(RT_M, args.npad);
      const uint32_t idescp = idesc_bf16_f32(RT_M, args.per * args.npad);
      const uint32_t term_bytes = npad_u * 128;
      int s = 0, ph = 0, consumed = 0;
      for (int i = 0; i < nkb; ++i) {
        if (!(ok = mbar_wait(bar_full(s), ph, abort_flag, args.status))) break;
        consumed = i + 1;
        tc_fence_after();
        const uint32_t st = sbase + s * args.stage_bytes;
        const uint32_t wb = st + RT_M * 128;
#pragma unroll
        for (int kk = 0; kk < RT_BK / 16; ++kk) {
          const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
          const uint64_t ad = sdesc_k_sw128(st + kk * 32);
          if (args.nacc == 3) {
            for (int t = 0; t < 3; t += args.per) {
              const bool whole = t + args.per <= 3;
              umma_bf16(tmem_base + static_cast<uint32_t>(t) * npad_u, ad,
                        sdesc_k_sw128(wb + t * term_bytes + kk * 32), whole ? idescp : idesc1, acc);
              if (!whole) break;
            }
          } else {
            umma_bf16(tmem_base, ad, sdesc_k_sw128(wb + kk * 32), idesc1, acc);
            umma_bf16(tmem_base + npad_u, ad, sdesc_k_sw128(wb + term_bytes + kk * 32), idesc1,
                      acc);
            umma_bf16(tmem_base + npad_u, ad, sdesc_k_sw128(wb + 2 * term_bytes + kk * 32),
                      idesc1, 1u);
          }
        }
        umma_commit(bar_empty(s));
        if (++s == S) { s = 0; ph ^= 1; }
      }
      misc[3] = static_cast<uint32_t>(consumed);
      // after the issued UMMAs (also when the loop gave up, so that the TMEM
      // is released only once they are done)
      umma_commit(bar_acc);
    }
  } else if (warp >= 4) {
    // ||x_t||^2 over this CTA's k-blocks from the staged x tiles (row r of a
    // tile is its 128 bytes at r * 128, chunks permuted by the swizzle), then
    // the partial logits TMEM -> shared memory once the last commit arrived
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    float xsq = 0.f;
    int s = 0, ph = 0;
    for (int i = 0; i < nkb; ++i) {
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar_full(s), ph, abort_flag, args.status));
      if (!ok) break;
      {
        const uint4* row = reinterpret_cast<const uint4*>(smem + s * args.stage_bytes + r * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 q = row[c];
          const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xFFFF0000u);
            xsq = fmaf(a, a, xsq);
            xsq = fmaf(b, b, xsq);
          }
        }
      }
      // these generic-proxy reads must be ordered before the next TMA write
      // into the stage (async proxy)
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(s));
      if (++s == S) { s = 0; ph ^= 1; }
    }
    if (ok && nkb > 0) ok = mbar_wait(bar_acc, 0, abort_flag, args.status);
    ok = __all_sync(0xFFFFFFFFu, ok);
    // the partial rows below overwrite the stages: no warp of the four may
    // still be reading the last x tile for its norms
    asm volatile("bar.sync 1, 128;" ::: "memory");
    tc_fence_after();
    float* prow = partial + static_cast<size_t>(r) * args.ld;
    if (ok && nkb > 0) {
      const uint32_t lanes = static_cast<uint32_t>(quad * 32) << 16;
      // partial logit = hi + (mid + lo), or hi + (mid and lo accumulated together)
      for (int c = 0; c < args.npad; c += 16) {
        uint32_t a[16], b[16], l[16];
        tmem_ld16_sync(tmem_base + lanes + c, a);
        tmem_ld16_sync(tmem_base + npad_u + lanes + c, b);
        if (args.nacc == 3) {
          tmem_ld16_sync(tmem_base + 2 * npad_u + lanes + c, l);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            b[i] = __float_as_uint(__uint_as_float(b[i]) + __uint_as_float(l[i]));
        }
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          float4 o;
          o.x = __uint_as_float(a[i]) + __uint_as_float(b[i]);
          o.y = __uint_as_float(a[i + 1]) + __uint_as_float(b[i + 1]);
          o.z = __uint_as_float(a[i + 2]) + __uint_as_float(b[i + 2]);
          o.w = __uint_as_float(a[i + 3]) + __uint_as_float(b[i + 3]);
          *reinterpret_cast<float4*>(prow + c + i) = o;
        }
      }
    } else {
      for (int c = 0; c < args.npad; c += 4)
        *reinterpret_cast<float4*>(prow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    xsq_part[r] = xsq;
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // a wait gave up: let the loads still in flight land and the issued UMMAs
    // finish before the shared and tensor memory are given back (bounded)
    for (uint32_t i = misc[3]; i < misc[2]; ++i)
      drain_wait(bar_full(static_cast<int>(i % S)), (i / S) & 1u);
    drain_wait(bar_acc, 0);
  }
  __syncthreads();
  // every CTA's partials are complete and visible to the cluster
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, static_cast<uint32_t>(args.tmem_cols));
  }

  // rows [rank 128 / C, (rank+1) 128 / C) are finished by this CTA: logits
  // and ||x_t||^2 to global memory for the top-k kernel
  if (!*abort_flag) {
    const int E = args.E;
    const int rpc = RT_M / static_cast<int>(csize);
    const int rbeg = static_cast<int>(rank) * rpc;
    const uint32_t pbase = smem_u32(partial);
    const uint32_t xbase = smem_u32(xsq_part);
    // 1. logits = the C partials in rank order + bias (four experts per item,
    //    every CTA's 16 bytes loaded before the adds), written out; ||x_t||^2
    const int nch = args.npad / 4;
    for (int it = threadIdx.x; it < rpc * nch; it += RT_THREADS) {
      const int rr = rbeg + it / nch;
      const int e0 = (it % nch) * 4;
      const uint32_t a = pbase + static_cast<uint32_t>((rr * args.ld + e0) * 4);
      float4 part[RT_MAX_CLUSTER];
#pragma unroll
      for (int q = 0; q < RT_MAX_CLUSTER; ++q)
        if (q < static_cast<int>(csize))
          part[q] = ld_shared_cluster_f32x4(mapa_shared(a, static_cast<uint32_t>(q)));
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < RT_MAX_CLUSTER; ++q) {
        if (q < static_cast<int>(csize)) {
          acc[0] += part[q].x;
          acc[1] += part[q].y;
          acc[2] += part[q].z;
          acc[3] += part[q].w;
        }
      }
      const int t = t0 + rr;
      if (t < args.T) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (e0 + i < E)
            args.logits[static_cast<size_t>(t) * E + e0 + i] = acc[i] + __ldg(args.b_r + e0 + i);
      }
    }
    for (int rr = rbeg + static_cast<int>(threadIdx.x); rr < rbeg + rpc; rr += RT_THREADS) {
      float xsq = 0.f;
      for (uint32_t q = 0; q < csize; ++q)
        xsq += ld_shared_cluster_f32(mapa_shared(xbase + static_cast<uint32_t>(rr * 4), q));
      if (t0 + rr < args.T) args.xsq[t0 + rr] = xsq;
    }
  }
  // no CTA leaves while another may still read its shared memory
  cluster_sync();
}

struct RouterTopkArgs {
  const float* logits;
  const float* xsq;
  const float* norms;
  const unsigned long long* fps;
  const uint16_t* x;
  const float* W_r;
  const float* b_r;
  int T, E, k, d;
  int32_t* topk_idx;
  float* topk_w;
  // T <= kPermChunk with the permutation requested: the last block to finish
  // builds it (counts may be null)
  int32_t *counts, *offsets, *mtile_prefix, *perm;
  int* done_blocks;
};

// One warp per token: top-k of its fp32 logits, near ties settled in fp64
// (the block's queued dot products computed by all its threads), softmax.
__global__ void __launch_bounds__(TK_WARPS * 32) router_topk_kernel(const RouterTopkArgs args) {
  pdl_wait_and_trigger();
  __shared__ RefineReq reqs[TK_WARPS];
  __shared__ PermSmallSmem perm_sm;
  __shared__ int last_block;
  __shared__ uint32_t jobs[TK_WARPS * RJ_PER_WARP];
  __shared__ int q_njob[TK_WARPS];
  __shared__ double red[4 * TK_WARPS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  const int t = static_cast<int>(blockIdx.x) * TK_WARPS + warp;
  float wmax = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    if (e < E) wmax = fmaxf(wmax, __ldg(args.norms + e));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wmax = fmaxf(wmax, __shfl_xor_sync(0xFFFFFFFFu, wmax, off));
  int njob = 0;
  if (t < args.T) {
    // lane l holds experts 128 h + 4 l + i (slot 4 h + i)
    const float* row = args.logits + static_cast<size_t>(t) * E;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = slot_expert(lane, j);
      v[j] = e < E ? __ldg(row + e) : -FLT_MAX;
    }
    float tau = kRefineRel * sqrtf(__ldg(args.xsq + t)) * wmax;
    if (!(tau <= FLT_MAX)) tau = 0.f;
    TopkList L;
    topk_list(v, E, args.k, tau, args.fps, lane, L);
    int32_t* idx_out = args.topk_idx + static_cast<size_t>(t) * args.k;
    float* w_out = args.topk_w + static_cast<size_t>(t) * args.k;
    double val[2] = {static_cast<double>(L.cval[0]), static_cast<double>(L.cval[1])};
    const uint64_t starts = topk_refine_starts(L);
    const int nj = __popcll(starts);
    if (L.refine_m == 0) {
      topk_emit(L, val, args.k, lane, idx_out, w_out);
    } else if (nj <= RJ_PER_WARP) {
      RefineReq& R = reqs[warp];
      if (lane == 0) {
        R.row = t;
        R.m = L.m;
        R.refine_m = L.refine_m;
        R.copy_m = L.copy_m;
      }
      R.cidx[lane] = L.cidx[0];
      R.cidx[32 + lane] = L.cidx[1];
      R.val[lane] = val[0];
      R.val[32 + lane] = val[1];
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        const int q = 32 * sl + lane;
        if ((starts >> q) & 1ull)
          jobs[warp * RJ_PER_WARP + __popcll(starts & ((1ull << q) - 1ull))] =
              static_cast<uint32_t>(q);
      }
      njob = nj;
    } else {
      topk_refine_warp(L, args.x + static_cast<size_t>(t) * args.d, args.W_r, args.b_r, args.d,
                       lane, val);
      topk_emit(L, val, args.k, lane, idx_out, w_out);
    }
  }
  if (lane == 0) q_njob[warp] = njob;
  __syncthreads();
  // the queued dot products, four at a time, each over all threads
  int jbase[TK_WARPS + 1];
  jbase[0] = 0;
#pragma unroll
  for (int w = 0; w < TK_WARPS; ++w) jbase[w + 1] = jbase[w] + q_njob[w];
  const int total = jbase[TK_WARPS];
  for (int base = 0; base < total; base += 4) {
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    int ex[4] = {0, 0, 0, 0}, rw[4] = {0, 0, 0, 0}, ps[4] = {0, 0, 0, 0};
    const uint16_t* xr[4] = {args.x, args.x, args.x, args.x};
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int J = base + g;
      if (J < total) {
        int w = 0;
        while (J >= jbase[w + 1]) ++w;
        rw[g] = w;
        ps[g] = static_cast<int>(jobs[w * RJ_PER_WARP + (J - jbase[w])]);
        ex[g] = reqs[w].cidx[ps[g]];
        xr[g] = args.x + static_cast<size_t>(reqs[w].row) * args.d;
      }
    }
    for (int i = 4 * static_cast<int>(threadIdx.x); i < args.d; i += 4 * TK_WARPS * 32) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (base + g < total) {
          const uint2 xb = __ldg(reinterpret_cast<const uint2*>(xr[g] + i));
          const float4 wv = __ldg(
              reinterpret_cast<const float4*>(args.W_r + static_cast<size_t>(ex[g]) * args.d + i));
          acc[g] = fma(static_cast<double>(__uint_as_float(xb.x << 16)), static_cast<double>(wv.x), acc[g]);
          acc[g] = fma(static_cast<double>(__uint_as_float(xb.x & 0xFFFF0000u)), static_cast<double>(wv.y), acc[g]);
          acc[g] = fma(static_cast<double>(__uint_as_float(xb.y << 16)), static_cast<double>(wv.z), acc[g]);
          acc[g] = fma(static_cast<double>(__uint_as_float(xb.y & 0xFFFF0000u)), static_cast<double>(wv.w), acc[g]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[g] += __shfl_xor_sync(0xFFFFFFFFu, acc[g], off);
      if (lane == 0) red[g * TK_WARPS + warp] = acc[g];
    }
    __syncthreads();
    if (static_cast<int>(threadIdx.x) < 4 && base + static_cast<int>(threadIdx.x) < total) {
      const int g = static_cast<int>(threadIdx.x);
      double sum = 0.0;
#pragma unroll
      for (int w = 0; w < TK_WARPS; ++w) sum += red[g * TK_WARPS + w];
      sum += static_cast<double>(__ldg(args.b_r + ex[g]));
      RefineReq& R = reqs[rw[g]];
      const int len = __ffsll(static_cast<long long>(~(R.copy_m >> ps[g])));
      for (int q = ps[g]; q < ps[g] + len; ++q) R.val[q] = sum;
    }
    __syncthreads();
  }
  if (njob > 0) {
    const RefineReq& R = reqs[warp];
    TopkList L;
    L.cidx[0] = R.cidx[lane];
    L.cidx[1] = R.cidx[32 + lane];
    L.cval[0] = 0.f;
    L.cval[1] = 0.f;
    L.m = R.m;
    L.refine_m = R.refine_m;
    L.copy_m = R.copy_m;
    const double val[2] = {R.val[lane], R.val[32 + lane]};
    topk_emit(L, val, args.k, lane, args.topk_idx + static_cast<size_t>(t) * args.k,
              args.topk_w + static_cast<size_t>(t) * args.k);
  }
  if (args.perm) {
    // the last block to finish sees every block's top-k (each block's stores,
    // then a device-scope fence, then its count) and builds the permutation
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
      last_block = atomicAdd(args.done_blocks, 1) == static_cast<int>(gridDim.x) - 1;
    __syncthreads();
    if (last_block) {
      __threadfence();
      perm_small_block(args.topk_idx, args.T, args.k, args.E, args.counts, args.offsets,
                       args.mtile_prefix, args.perm, perm_sm);
    }
  }
}

// Clusters of C CTAs of router_tc_kernel (the largest shared-memory shape)
// that can be resident at once on the current device, cached per device.
int max_active_clusters(int dev, int C, size_t smem) {
  static int cache[64][4] = {};
  int slot = C == 2 ? 1 : C == 4 ? 2 : C == 8 ? 3 : 0;
  if (dev < 0 || dev >= 64) return 0;
  if (!cache[dev][slot]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(C) * 16);
    cfg.blockDim = dim3(RT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(C);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, router_tc_kernel, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = -1;   // not available: this size is not used
    }
    cache[dev][slot] = n;
  }
  return cache[dev][slot];
}

int num_sms_of(int dev) {
  static int cache[64] = {};
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// CTAs per cluster: doubled (up to 8) while every CTA keeps at least one
// k-block and all clusters of the grid fit on the device at once.
int cluster_size(int T, int d, int dev, size_t smem) {
  const int tiles = (T + RT_M - 1) / RT_M;
  const int KB = (d + RT_BK - 1) / RT_BK;
  const int sms = num_sms_of(dev);
  int C = 1;
  while (C < RT_MAX_CLUSTER && 2 * C <= KB && tiles * 2 * C <= sms &&
         tiles <= max_active_clusters(dev, 2 * C, smem))
    C *= 2;
  return C;
}

}  // namespace

size_t router_tc_scratch_bytes(int E, int d, int T) {
  const size_t npad = static_cast<size_t>((E + 15) / 16 * 16);
  return 3 * npad * static_cast<size_t>(d) * 2 + npad * 4 + npad * 8 + static_cast<size_t>(T) * 4 +
         16;
}

cudaError_t launch_router_tc(const uint16_t* x, const float* W_r, const float* b_r, int T, int E,
                             int k, int d, void* scratch, float* logits, int32_t* topk_idx,
                             float* topk_w, int* status, cudaStream_t st, int32_t* counts,
                             int32_t* offsets, int32_t* mtile_prefix, int32_t* perm) {
  if (E < 1 || E > 256 || k < 1 || k > E || k > 32 || d % 32 != 0 || T < 1)
    return cudaErrorInvalidValue;
  const RouterTcShape sh = router_tc_shape(E);
  if (sh.stages < 2) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  static bool attr_set[64] = {false};
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    // the largest shape's requirement, set once per device
    const RouterTcShape big = router_tc_shape(256);
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         big.smem_alloc > sh.smem_alloc ? big.smem_alloc : sh.smem_alloc);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  uint16_t* terms = static_cast<uint16_t*>(scratch);
  float* norms = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) +
                                          3 * static_cast<size_t>(sh.npad) * d * 2);
  unsigned long long* fps = reinterpret_cast<unsigned long long*>(norms + sh.npad);
  float* xsq = reinterpret_cast<float*>(fps + sh.npad);
  int* done_blocks = reinterpret_cast<int*>(xsq + T);
  // the weight split: the first launch of the pass (it clears the status word)
  {
    cudaError_t e = launch_kernel(router_split_kernel, dim3(sh.npad), dim3(256), 0, st, W_r, b_r,
                                  E, sh.npad, d, terms, norms, fps, status, done_blocks);
    if (e != cudaSuccess) return e;
    pdl_launches() = true;   // the router kernel may overlap the split's tail
  }
  CUtensorMap tmX, tmW;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
    const cuuint32_t box[2] = {RT_BK, RT_M};
    if (!mx_encode_bf16_map(&tmX, x, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(sh.npad), 3};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                   static_cast<cuuint64_t>(d) * 2 * sh.npad};
    const cuuint32_t box[3] = {RT_BK, static_cast<cuuint32_t>(sh.npad), 3};
    if (!mx_encode_bf16_map(&tmW, terms, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const int C = cluster_size(T, d, dev, static_cast<size_t>(router_tc_shape(256).smem_alloc));
  RouterTcArgs a;
  a.b_r = b_r;
  a.T = T;
  a.E = E;
  a.d = d;
  a.npad = sh.npad;
  a.nacc = sh.nacc;
  a.per = sh.per;
  a.stages = sh.stages;
  a.ld = sh.ld;
  a.stage_bytes = sh.stage_bytes;
  a.body = sh.body;
  a.tmem_cols = sh.tmem_cols;
  a.KB = (d + RT_BK - 1) / RT_BK;
  a.logits = logits;
  a.xsq = xsq;
  a.status = status;
  const int tiles = (T + RT_M - 1) / RT_M;
  cudaError_t e = launch_kernel_cluster(router_tc_kernel, dim3(tiles * C), dim3(RT_THREADS),
                                        static_cast<size_t>(sh.smem_alloc), C, st, tmX, tmW, a);
  if (e != cudaSuccess) return e;
  RouterTopkArgs ta;
  ta.logits = logits;
  ta.xsq = xsq;
  ta.norms = norms;
  ta.fps = fps;
  ta.x = x;
  ta.W_r = W_r;
  ta.b_r = b_r;
  ta.T = T;
  ta.E = E;
  ta.k = k;
  ta.d = d;
  ta.topk_idx = topk_idx;
  ta.topk_w = topk_w;
  const bool fuse_perm = perm && T <= kPermChunk;
  ta.counts = fuse_perm ? counts : nullptr;
  ta.offsets = fuse_perm ? offsets : nullptr;
  ta.mtile_prefix = fuse_perm ? mtile_prefix : nullptr;
  ta.perm = fuse_perm ? perm : nullptr;
  ta.done_blocks = done_blocks;
  return launch_kernel(router_topk_kernel, dim3((T + TK_WARPS - 1) / TK_WARPS),
                       dim3(TK_WARPS * 32), 0, st, ta);
}

}  // namespace moe
