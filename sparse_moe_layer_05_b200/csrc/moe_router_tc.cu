// moe_router_tc.cu -- the router on the tensor cores, for batches of more than
// 256 tokens, with the top-k and the selected-set softmax in the same kernel.
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
// Each product of x with a term is exact in fp32 and the tensor core
// accumulates them in fp32: the logits are fp32 dot products as on the CUDA
// cores, in a different summation order. Every expert's column goes through
// the same operations, so identical router rows still give identical logits.
//
// Tiles. One CTA per 128 tokens (UMMA M = 128) and all experts at once (N = E
// rounded up to 16, at most 256, one TMEM accumulator), 64 elements of d per
// shared-memory stage: the x tile by one TMA box, the three weight terms by one
// 3-D box. Twelve UMMAs per stage (4 K steps x 3 terms). The epilogue adds the
// bias, stores the logits in shared memory (over the drained stages), and one
// warp per token selects its k experts there.
//
// Roles (256 threads): warp 0 TMA producer, warp 1 TMEM allocation and UMMA
// issue, warps 4-7 TMEM -> shared memory; then all eight warps run the top-k.
// Every wait is bounded (moe_ptx.cuh).
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"
#include "moe_topk.cuh"

namespace moe {
namespace {

constexpr int RT_M = 128;                 // tokens per CTA
constexpr int RT_BK = 64;                 // d elements per stage (128 bytes of bf16)
constexpr int RT_MAX_STAGES = 4;
constexpr int RT_THREADS = 256;
constexpr int RT_SMEM_LIMIT = 232448 - 1024;

struct RouterTcShape {
  int npad;          // E rounded up to 16
  int stage_bytes;   // x tile + three weight-term tiles
  int stages;
  int logits_ld;     // floats per logits row in shared memory
  int smem_alloc;
};

RouterTcShape router_tc_shape(int E) {
  RouterTcShape s;
  s.npad = (E + 15) / 16 * 16;
  s.stage_bytes = RT_M * 128 + 3 * s.npad * 128;
  s.logits_ld = s.npad + 4;
  const int logits_bytes = RT_M * s.logits_ld * 4;
  const int fixed = 1024;   // barriers and the TMEM address
  int st = (RT_SMEM_LIMIT - fixed) / s.stage_bytes;
  if (st > RT_MAX_STAGES) st = RT_MAX_STAGES;
  s.stages = st;
  int body = st * s.stage_bytes;
  if (body < logits_bytes) body = logits_bytes;
  s.smem_alloc = body + fixed + 1024;
  return s;
}

// W_r [E][d] fp32 -> terms [3][npad][d] bf16 (rows E..npad-1 zero).
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ W_r, int E,
                                                           int npad, int d,
                                                           uint16_t* __restrict__ terms,
                                                           int* status) {
  pdl_wait_and_trigger();
  // the first kernel of the pass clears the status word
  if (status && blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
  const int64_t n = static_cast<int64_t>(npad) * d;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / d;
    const float w = row < E ? W_r[i] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    terms[i] = __bfloat16_as_ushort(hi);
    terms[n + i] = __bfloat16_as_ushort(mid);
    terms[2 * n + i] = __bfloat16_as_ushort(lo);
  }
}

struct RouterTcArgs {
  const float* b_r;
  int T, E, k, d, npad, stages, logits_ld, stage_bytes;
  int32_t* topk_idx;
  float* topk_w;
  int* status;
};

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
  const int body = max(S * args.stage_bytes, RT_M * args.logits_ld * 4);
  const uint32_t bar0 = sbase + body;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (RT_MAX_STAGES + s); };
  const uint32_t bar_acc = bar0 + 8u * (2 * RT_MAX_STAGES);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + body + 8 * (2 * RT_MAX_STAGES + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_acc, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  const int t0 = blockIdx.x * RT_M;
  const int KB = (args.d + RT_BK - 1) / RT_BK;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0, ph = 0;
      const uint32_t tx = static_cast<uint32_t>(args.stage_bytes);
      for (int kb = 0; kb < KB; ++kb) {
        if (!(ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, args.status))) break;
        const uint32_t st = sbase + s * args.stage_bytes;
        mbar_expect_tx(bar_full(s), tx);
        tma_load_2d(st, &tmX, kb * RT_BK, t0, bar_full(s));
        tma_load_3d(st + RT_M * 128, &tmW, kb * RT_BK, 0, 0, bar_full(s));
        if (++s == S) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(RT_M, args.npad);
      const uint32_t term_bytes = static_cast<uint32_t>(args.npad) * 128;
      int s = 0, ph = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!(ok = mbar_wait(bar_full(s), ph, abort_flag, args.status))) break;
        tc_fence_after();
        const uint32_t st = sbase + s * args.stage_bytes;
        const uint32_t wb = st + RT_M * 128;
#pragma unroll
        for (int kk = 0; kk < RT_BK / 16; ++kk) {
#pragma unroll
          for (int h = 0; h < 3; ++h)
            umma_bf16(tmem_base, sdesc_k_sw128(st + kk * 32),
                      sdesc_k_sw128(wb + h * term_bytes + kk * 32), idesc,
                      (kb | kk | h) != 0 ? 1u : 0u);
        }
        umma_commit(bar_empty(s));
        if (++s == S) { s = 0; ph ^= 1; }
      }
      if (ok) umma_commit(bar_acc);
    }
  } else if (warp >= 4) {
    // TMEM -> shared memory logits (bias added); the stages are drained once
    // the last commit has arrived
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    ok = mbar_wait(bar_acc, 0, abort_flag, args.status);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (ok) {
      tc_fence_after();
      float* row = reinterpret_cast<float*>(smem) + static_cast<size_t>(r) * args.logits_ld;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      for (int c = 0; c < args.npad; c += 16) {
        uint32_t v[16];
        tmem_ld16_sync(taddr + c, v);
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          float4 o;
          o.x = __uint_as_float(v[i]) + (c + i < args.E ? __ldg(args.b_r + c + i) : 0.f);
          o.y = __uint_as_float(v[i + 1]) + (c + i + 1 < args.E ? __ldg(args.b_r + c + i + 1) : 0.f);
          o.z = __uint_as_float(v[i + 2]) + (c + i + 2 < args.E ? __ldg(args.b_r + c + i + 2) : 0.f);
          o.w = __uint_as_float(v[i + 3]) + (c + i + 3 < args.E ? __ldg(args.b_r + c + i + 3) : 0.f);
          *reinterpret_cast<float4*>(row + c + i) = o;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // top-k and softmax, one warp per token, over the logits in shared memory
  if (!*abort_flag) {
    for (int tt = warp; tt < RT_M; tt += RT_THREADS / 32) {
      const int t = t0 + tt;
      if (t >= args.T) break;
      topk_softmax_warp(reinterpret_cast<const float*>(smem) + static_cast<size_t>(tt) * args.logits_ld,
                        args.E, args.k, lane, args.topk_idx + static_cast<size_t>(t) * args.k,
                        args.topk_w + static_cast<size_t>(t) * args.k);
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace

size_t router_tc_terms_bytes(int E, int d) {
  return static_cast<size_t>(3) * ((E + 15) / 16 * 16) * d * 2;
}

cudaError_t launch_router_tc(const uint16_t* x, const float* W_r, const float* b_r, int T, int E,
                             int k, int d, uint16_t* terms, int32_t* topk_idx, float* topk_w,
                             int* status, cudaStream_t st) {
  if (E < 1 || E > 256 || d % 32 != 0 || T < 1) return cudaErrorInvalidValue;
  const RouterTcShape sh = router_tc_shape(E);
  if (sh.stages < 2) return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    // the largest shape's requirement, set once per device
    const RouterTcShape big = router_tc_shape(256);
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         big.smem_alloc > sh.smem_alloc ? big.smem_alloc : sh.smem_alloc);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // the weight split: the first launch of the pass (it clears the status word)
  {
    const int64_t n = static_cast<int64_t>(sh.npad) * d;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    cudaError_t e = launch_kernel(router_split_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0,
                                  st, W_r, E, sh.npad, d, terms, status);
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
  RouterTcArgs a;
  a.b_r = b_r;
  a.T = T;
  a.E = E;
  a.k = k;
  a.d = d;
  a.npad = sh.npad;
  a.stages = sh.stages;
  a.logits_ld = sh.logits_ld;
  a.stage_bytes = sh.stage_bytes;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.status = status;
  return launch_kernel(router_tc_kernel, dim3((T + RT_M - 1) / RT_M), dim3(RT_THREADS),
                       static_cast<size_t>(sh.smem_alloc), st, tmX, tmW, a);
}

}  // namespace moe
