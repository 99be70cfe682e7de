// moe_grouped_gemm.cu -- expert-grouped MXFP4 GEMMs on the sm_100a tensor
// cores (tcgen05, TMEM accumulators, TMA-fed shared memory).
//
//   gate/up:  for the rows r of expert e (permuted order),
//             H[r, n] = silu(x_r . Wgate[e][n] + bg[e][n]) * (x_r . Wup[e][n] + bu[e][n])
//   down:     Yw[pair(r), m] = p(pair(r)) * (H[r] . Wdown[e][m] + bd[e][m])
// (the biases are optional; without them those terms are zero).
//
// Field guide "gpt-oss 20B", "03 Sparse Mixture of Experts" (SwiGLU experts,
// weighted sum); "shrink/gpt_oss-mic", "Preserved properties" (silu);
// "gpt-oss-20b and gpt-oss-120b", "Four-bit expert weights" (MXFP4).
//
// One persistent CTA per SM walks the tiles (expert, n tile, m tile) that the
// device-side routing tables define; no host synchronisation is needed.
// A tile is 256 activation rows x 128 weight rows: the 128 x 64 decoded
// weight block of a k-block feeds two M = 128 UMMAs (rows 0-127 and 128-255),
// so each decoded weight serves 256 rows. When an expert's last tile has at
// most 128 rows the second UMMA (and its activation load) is skipped.
//
// Warp roles (512 threads):
//   warp 0      TMA producer of the activation tiles (bf16, 128B swizzle)
//   warp 2      TMA producer of the MXFP4 code boxes and the k-block's E8M0
//               scales (a ring of its own, so codes run ahead of activations)
//   warp 1      TMEM allocator and UMMA issuer (one thread)
//   warps 4-7   epilogue: TMEM -> registers -> SwiGLU / weighted store
//   warps 8-15  decoders: two threads per weight row, each turns 32 codes and
//               their scale into bf16 in the 128B-swizzled K-major layout
// Accumulators: per tile two 128 x 128 fp32 blocks (256 TMEM columns),
// double-buffered (512 columns) so the epilogue of one tile overlaps the main
// loop of the next.
//
// Both operands keep every 8-element chunk of a row in kPerm8 order (see
// moe_ptx.cuh); the H rows this kernel writes follow the same order.
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {
namespace {

constexpr int BM = kTileM;            // 256 rows per tile (two UMMA halves)
constexpr int BMH = 128;              // rows per UMMA
constexpr int BK = 64;                // contraction elements per k-block (128 B of bf16)
constexpr int NH = 64;                // weight rows per TMA box (half of the tile)
constexpr int BN = 2 * NH;            // 128 = UMMA N
constexpr int SA = 4;                 // activation stages
constexpr int SB = 4;                 // decoded weight stages
constexpr int SC = 6;                 // code stages
constexpr int A_HALF = BMH * BK * 2;  // 16384
constexpr int A_BYTES = 2 * A_HALF;   // 32768
constexpr int B_BYTES = BN * BK * 2;  // 16384
constexpr int C_CODES = BN * BK / 2;  // 4096 bytes of codes per stage
constexpr int S_BOX = NH * 2;         // scales of one box: 64 rows x 2 groups
constexpr int S_OFF0 = C_CODES;       // 4096
constexpr int S_OFF1 = C_CODES + 128; // 4224
constexpr int C_TX = C_CODES + 2 * S_BOX;
constexpr int C_BYTES = 4352;         // stage stride (128-byte aligned)
constexpr int NUM_THREADS = 512;
constexpr int EPI_WARP0 = 4;
constexpr int DEQ_WARP0 = 8;
constexpr int DEQ_THREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;         // column distance between the two tile buffers
constexpr int MAX_E = 256;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + SA * A_BYTES;
constexpr int OFF_C = OFF_B + SB * B_BYTES;
constexpr int OFF_BAR = OFF_C + SC * C_BYTES;
constexpr int NUM_BARS = 2 * SA + 2 * SB + 2 * SC + 4;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int OFF_TAB = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_TAB + 2 * (MAX_E + 1) * 4;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;   // slack for 1024-byte alignment
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(OFF_C % 1024 == 0 && C_BYTES % 128 == 0, "stage alignment");

enum Epi { EPI_SWIGLU = 0, EPI_DOWN = 1 };

struct Args {
  const int32_t* offsets;
  const int32_t* mprefix;
  int E, K, Nrows;
  int n_tiles;
  int row_step;     // weight rows advanced per n tile
  int half_off;     // row offset of the second box relative to the first
  int n_out;
  uint16_t* out;
  float* out_f32;
  const int32_t* perm;
  const float* topk_w;
  int* status;
  const float* bias;  // [E][2I] (SwiGLU) or [E][d] (down), or nullptr
};

struct TileInfo {
  int e, mt, nt, row0, rows;
};

__device__ __forceinline__ void decode_tile(int tile, int n_tiles, int E, const int* s_off,
                                            const int* s_mp, TileInfo& ti) {
  const int q = tile / n_tiles;
  int lo = 0, hi = E;  // largest e with s_mp[e] <= q
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mp[mid] <= q) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int mte = s_mp[e + 1] - s_mp[e];
  const int local = tile - s_mp[e] * n_tiles;
  ti.e = e;
  ti.nt = local / mte;
  ti.mt = local % mte;
  ti.row0 = s_off[e] + ti.mt * BM;
  const int cnt = s_off[e + 1] - s_off[e];
  ti.rows = min(BM, cnt - ti.mt * BM);
}

__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Bias of 8 gate columns col.. and the matching up columns (row layout
// [gate 0..n-1 | up 0..n-1]); zeros without a bias row. n is a multiple of 8
// and col < n, so both 32-byte reads stay inside the row.
__device__ __forceinline__ void load_bias8x2(const float* brow, int col, int n, float* bg,
                                             float* bu) {
  if (brow && col < n) {
    const float4* pg = reinterpret_cast<const float4*>(brow + col);
    const float4* pu = reinterpret_cast<const float4*>(brow + n + col);
    const float4 g0 = __ldg(pg), g1 = __ldg(pg + 1), u0 = __ldg(pu), u1 = __ldg(pu + 1);
    bg[0] = g0.x; bg[1] = g0.y; bg[2] = g0.z; bg[3] = g0.w;
    bg[4] = g1.x; bg[5] = g1.y; bg[6] = g1.z; bg[7] = g1.w;
    bu[0] = u0.x; bu[1] = u0.y; bu[2] = u0.z; bu[3] = u0.w;
    bu[4] = u1.x; bu[5] = u1.y; bu[6] = u1.z; bu[7] = u1.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) bg[i] = bu[i] = 0.f;
  }
}

// Bias of 16 output columns col.. (col + 16 <= the row length), or zeros.
__device__ __forceinline__ void load_bias16(const float* brow, int col, float* b) {
  if (brow) {
    const float4* p = reinterpret_cast<const float4*>(brow + col);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(p + i);
      b[4 * i] = v.x; b[4 * i + 1] = v.y; b[4 * i + 2] = v.z; b[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) b[i] = 0.f;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_mxfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmB,
                              const __grid_constant__ CUtensorMap tmS, const Args args) {
  pdl_wait_and_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar0 = sbase + OFF_BAR;
  auto bar_fullA = [&](int s) { return bar0 + 8u * s; };
  auto bar_emptyA = [&](int s) { return bar0 + 8u * (SA + s); };
  auto bar_fullB = [&](int s) { return bar0 + 8u * (2 * SA + s); };
  auto bar_emptyB = [&](int s) { return bar0 + 8u * (2 * SA + SB + s); };
  auto bar_fullC = [&](int s) { return bar0 + 8u * (2 * SA + 2 * SB + s); };
  auto bar_emptyC = [&](int s) { return bar0 + 8u * (2 * SA + 2 * SB + SC + s); };
  auto bar_accFull = [&](int s) { return bar0 + 8u * (2 * SA + 2 * SB + 2 * SC + s); };
  auto bar_accEmpty = [&](int s) { return bar0 + 8u * (2 * SA + 2 * SB + 2 * SC + 2 + s); };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* s_off = reinterpret_cast<int*>(smem + OFF_TAB);
  int* s_mp = s_off + (MAX_E + 1);

  const int E = args.E;
  for (int i = threadIdx.x; i <= E; i += NUM_THREADS) {
    s_off[i] = args.offsets[i];
    s_mp[i] = args.mprefix[i];
  }
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < SA; ++s) {
      mbar_init(bar_fullA(s), 1);
      mbar_init(bar_emptyA(s), 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(bar_fullB(s), DEQ_THREADS);
      mbar_init(bar_emptyB(s), 1);
    }
    for (int s = 0; s < SC; ++s) {
      mbar_init(bar_fullC(s), 1);
      mbar_init(bar_emptyC(s), DEQ_THREADS);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_accFull(s), 1);
      mbar_init(bar_accEmpty(s), 4 * 32);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmS);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];

  const int total = s_mp[E] * args.n_tiles;
  const int KB = (args.K + BK - 1) / BK;
  if (warp == 3) return;  // no role; the final barrier counts the others

  if (warp == 0) {
    // ------------------------------------------- producer: activations --
    if (lane == 0) {
      int sa = 0, pa = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        TileInfo ti;
        decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
        const bool two = ti.rows > BMH;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_emptyA(sa), pa ^ 1, abort_flag, args.status))) break;
          const uint32_t adst = sbase + OFF_A + sa * A_BYTES;
          mbar_expect_tx(bar_fullA(sa), two ? A_BYTES : A_HALF);
          tma_load_2d(adst, &tmA, kb * BK, ti.row0, bar_fullA(sa));
          if (two) tma_load_2d(adst + A_HALF, &tmA, kb * BK, ti.row0 + BMH, bar_fullA(sa));
          if (++sa == SA) { sa = 0; pa ^= 1; }
        }
      }
    }
  } else if (warp == 2) {
    // -------------------------------------- producer: codes and scales --
    // Runs ahead of the activation ring as far as the code ring allows.
    if (lane == 0) {
      int sc = 0, pc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        TileInfo ti;
        decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
        const int rA = ti.nt * args.row_step;
        const int rB = rA + args.half_off;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_emptyC(sc), pc ^ 1, abort_flag, args.status))) break;
          const uint32_t cdst = sbase + OFF_C + sc * C_BYTES;
          mbar_expect_tx(bar_fullC(sc), C_TX);
          tma_load_3d(cdst, &tmB, kb * (BK / 2), rA, ti.e, bar_fullC(sc));
          tma_load_3d(cdst + NH * (BK / 2), &tmB, kb * (BK / 2), rB, ti.e, bar_fullC(sc));
          // scales [E][K/32][Nrows]: groups 2kb, 2kb+1 of each box's 64 rows
          tma_load_3d(cdst + S_OFF0, &tmS, rA, 2 * kb, ti.e, bar_fullC(sc));
          tma_load_3d(cdst + S_OFF1, &tmS, rB, 2 * kb, ti.e, bar_fullC(sc));
          if (++sc == SC) { sc = 0; pc ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- UMMA issuer --
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BMH, BN);
      int sa = 0, pa = 0, sb = 0, pb = 0, it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        TileInfo ti;
        decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
        const bool two = ti.rows > BMH;
        const int ab = it & 1;
        const uint32_t ap = (it >> 1) & 1;
        if (!(ok = mbar_wait(bar_accEmpty(ab), ap ^ 1, abort_flag, args.status))) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + ab * ACC_COLS;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_fullA(sa), pa, abort_flag, args.status))) break;
          if (!(ok = mbar_wait(bar_fullB(sb), pb, abort_flag, args.status))) break;
          tc_fence_after();
          const uint32_t a_addr = sbase + OFF_A + sa * A_BYTES;
          const uint32_t b_addr = sbase + OFF_B + sb * B_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = sdesc_k_sw128(b_addr + kk * 32);
            const uint32_t acc = (kb | kk) != 0;
            umma_bf16(d0, sdesc_k_sw128(a_addr + kk * 32), bdesc, idesc, acc);
            if (two)
              umma_bf16(d0 + BN, sdesc_k_sw128(a_addr + A_HALF + kk * 32), bdesc, idesc, acc);
          }
          umma_commit(bar_emptyA(sa));
          umma_commit(bar_emptyB(sb));
          if (++sa == SA) { sa = 0; pa ^= 1; }
          if (++sb == SB) { sb = 0; pb ^= 1; }
        }
        if (ok) umma_commit(bar_accFull(ab));
      }
    }
  } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) {
    // ----------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      TileInfo ti;
      decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
      const int ab = it & 1;
      const uint32_t ap = (it >> 1) & 1;
      if (!mbar_wait(bar_accFull(ab), ap, abort_flag, args.status)) break;
      tc_fence_after();
      const int halves = ti.rows > BMH ? 2 : 1;
      for (int hh = 0; hh < halves; ++hh) {
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                               ab * ACC_COLS + hh * BN;
        const int r = hh * BMH + quad * 32 + lane;
        const bool valid = r < ti.rows;
        const int64_t grow = ti.row0 + r;
        if (EPI == EPI_SWIGLU) {
          // columns 0..63 gate, 64..127 up; H stored in kPerm8 chunk order
          const int col0 = ti.nt * NH;
          uint16_t* orow = args.out + grow * args.n_out;
          const float* brow = args.bias ? args.bias + static_cast<int64_t>(ti.e) * 2 * args.n_out
                                        : nullptr;
#pragma unroll 1
          for (int c = 0; c < NH; c += 8) {
            uint32_t g[8], u[8];
            tmem_ld8x2_sync(taddr + c, taddr + NH + c, g, u);
            const int col = col0 + c;
            float bg[8], bu[8];
            load_bias8x2(brow, col, args.n_out, bg, bu);
            float h[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              h[i] = silu_f(__uint_as_float(g[i]) + bg[i]) * (__uint_as_float(u[i]) + bu[i]);
            if (valid && col < args.n_out) {
              *reinterpret_cast<uint4*>(orow + col) =
                  make_uint4(pack_bf16x2(h[0], h[4]), pack_bf16x2(h[1], h[5]),
                             pack_bf16x2(h[2], h[6]), pack_bf16x2(h[3], h[7]));
            }
          }
        } else {
          // weighted un-permute: fp32 row p * y of pair perm[row] at yw[pair]
          const int col0 = ti.nt * BN;
          int pair = 0;
          float w = 0.f;
          if (valid) {
            pair = args.perm[grow];
            w = args.topk_w[pair];
          }
          float* orow = args.out_f32 + static_cast<int64_t>(pair) * args.n_out;
          const float* brow = args.bias ? args.bias + static_cast<int64_t>(ti.e) * args.n_out
                                        : nullptr;
#pragma unroll 1
          for (int c = 0; c < BN; c += 16) {
            uint32_t y[16];
            tmem_ld16_sync(taddr + c, y);
            const int col = col0 + c;
            if (valid && col < args.n_out) {
              float b[16];
              load_bias16(brow, col, b);
              float4* dst = reinterpret_cast<float4*>(orow + col);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(w * (__uint_as_float(y[4 * i]) + b[4 * i]),
                                     w * (__uint_as_float(y[4 * i + 1]) + b[4 * i + 1]),
                                     w * (__uint_as_float(y[4 * i + 2]) + b[4 * i + 2]),
                                     w * (__uint_as_float(y[4 * i + 3]) + b[4 * i + 3]));
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_accEmpty(ab));
    }
  } else if (warp >= DEQ_WARP0) {
    // ----------------------------------------------------------- decoders --
    const int t = threadIdx.x - DEQ_WARP0 * 32;
    const int n = t >> 1;             // weight row inside the tile (0..127)
    const int g = t & 1;              // scale group inside the k-block
    const int soff = (n < NH ? S_OFF0 : S_OFF1) + g * NH + (n & (NH - 1));
    const int sw = n & 7;
    int sc = 0, pc = 0, sb = 0, pb = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        if (!(ok = mbar_wait(bar_fullC(sc), pc, abort_flag, args.status))) break;
        const uint8_t* stage = smem + OFF_C + sc * C_BYTES;
        const uint4 q = *reinterpret_cast<const uint4*>(stage + n * 32 + g * 16);
        const uint32_t s = stage[soff];
        uint4 o[4];
        mxfp4x32_to_bf16(q, s, o);
        if (!(ok = mbar_wait(bar_emptyB(sb), pb ^ 1, abort_flag, args.status))) break;
        uint8_t* brow = smem + OFF_B + sb * B_BYTES + n * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(brow + (((4 * g + c) ^ sw) << 4)) = o[c];
        // One proxy fence orders this thread's generic-proxy accesses before
        // the async proxy's next ones: the code-stage reads above (the next
        // TMA write into that stage must not overtake them) and the
        // decoded-weight writes (the UMMA must see them).
        fence_proxy_async_smem();
        mbar_arrive(bar_emptyC(sc));
        if (++sc == SC) { sc = 0; pc ^= 1; }
        mbar_arrive(bar_fullB(sb));
        if (++sb == SB) { sb = 0; pb ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ================================================================= pair ====
// CTA-pair variant for experts with many rows: a cluster of 2 CTAs (one per
// SM) computes a 256 x 240 tile with tcgen05 cta_group::2 UMMAs (M = 256,
// N = 240). CTA r holds activation rows r*128..r*128+127 and decodes weight
// rows r*120..r*120+119 of the tile (the gate rows on CTA 0 and the matching
// up rows on CTA 1 for the gate/up GEMM), so each SM decodes 120 rows per
// k-block for 128 x 240 MACs and reads half as much B per MAC as a 1-SM tile.
// All loads and decodes stay local to each CTA (warp 0 loads activations,
// warp 2 codes and scales, warps 8-15 decode). The even CTA issues the UMMAs;
// in the odd CTA warp 3 forwards "stage ready" per k-block and the first
// epilogue thread forwards "accumulator released" per tile to the even CTA,
// each with one remote mbarrier arrive.
namespace pair {

constexpr int BMH = 128;              // activation rows per CTA
constexpr int BK = 64;
constexpr int NH = 120;               // weight rows per CTA
constexpr int BN = 2 * NH;            // 240 = UMMA N
constexpr int SA = 5, SB = 5, SC = 8;
constexpr int A_BYTES = BMH * BK * 2;       // 16384
constexpr int B_BYTES = NH * BK * 2;        // 15360
constexpr int C_CODES = NH * BK / 2;        // 3840
constexpr int S_ROWS = 144;                 // 16-aligned window holding 120 rows
constexpr int S_OFF = 3840;                 // scale box offset in a code stage
constexpr int C_TX = C_CODES + 2 * S_ROWS;  // 4128
constexpr int C_BYTES = 4224;
constexpr int NUM_THREADS = 512;
constexpr int DEQ_THREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + SA * A_BYTES;
constexpr int OFF_C = OFF_B + SB * B_BYTES;
constexpr int OFF_BAR = OFF_C + SC * C_BYTES;
// fullA, emptyA, fullB, emptyB, peerFull (SB), fullC, emptyC, accFull,
// accEmpty, peerAccEmpty
constexpr int NUM_BARS = 2 * SA + 3 * SB + 2 * SC + 6;
constexpr int OFF_MISC = (OFF_BAR + NUM_BARS * 8 + 15) & ~15;
constexpr int OFF_TAB = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_TAB + 2 * (MAX_E + 1) * 4;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(OFF_B % 1024 == 0 && OFF_C % 1024 == 0 && B_BYTES % 1024 == 0, "alignment");

}  // namespace pair

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::NUM_THREADS, 1)
    grouped_mxfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                                   const __grid_constant__ CUtensorMap tmB,
                                   const __grid_constant__ CUtensorMap tmS, const Args args) {
  pdl_wait_and_trigger();
  // local copies shadow the single-CTA kernel's constants of the same names
  constexpr int BMH = pair::BMH;
  constexpr int BK = pair::BK;
  constexpr int NH = pair::NH;
  constexpr int BN = pair::BN;
  constexpr int SA = pair::SA;
  constexpr int SB = pair::SB;
  constexpr int SC = pair::SC;
  constexpr int A_BYTES = pair::A_BYTES;
  constexpr int B_BYTES = pair::B_BYTES;
  constexpr int S_ROWS = pair::S_ROWS;
  constexpr int S_OFF = pair::S_OFF;
  constexpr int C_TX = pair::C_TX;
  constexpr int C_BYTES = pair::C_BYTES;
  constexpr int NUM_THREADS = pair::NUM_THREADS;
  constexpr int DEQ_THREADS = pair::DEQ_THREADS;
  constexpr int TMEM_COLS = pair::TMEM_COLS;
  constexpr int ACC_COLS = pair::ACC_COLS;
  constexpr int OFF_A = pair::OFF_A;
  constexpr int OFF_B = pair::OFF_B;
  constexpr int OFF_C = pair::OFF_C;
  constexpr int OFF_BAR = pair::OFF_BAR;
  constexpr int OFF_MISC = pair::OFF_MISC;
  constexpr int OFF_TAB = pair::OFF_TAB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  const uint32_t bar0 = sbase + OFF_BAR;
  auto bar_fullA = [&](int s) { return bar0 + 8u * s; };
  auto bar_emptyA = [&](int s) { return bar0 + 8u * (SA + s); };
  auto bar_fullB = [&](int s) { return bar0 + 8u * (2 * SA + s); };
  auto bar_emptyB = [&](int s) { return bar0 + 8u * (2 * SA + SB + s); };
  auto bar_peerFull = [&](int s) { return bar0 + 8u * (2 * SA + 2 * SB + s); };
  auto bar_fullC = [&](int s) { return bar0 + 8u * (2 * SA + 3 * SB + s); };
  auto bar_emptyC = [&](int s) { return bar0 + 8u * (2 * SA + 3 * SB + SC + s); };
  auto bar_accFull = [&](int s) { return bar0 + 8u * (2 * SA + 3 * SB + 2 * SC + s); };
  auto bar_accEmpty = [&](int s) { return bar0 + 8u * (2 * SA + 3 * SB + 2 * SC + 2 + s); };
  auto bar_peerAcc = [&](int s) { return bar0 + 8u * (2 * SA + 3 * SB + 2 * SC + 4 + s); };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* s_off = reinterpret_cast<int*>(smem + OFF_TAB);
  int* s_mp = s_off + (MAX_E + 1);

  const int E = args.E;
  for (int i = threadIdx.x; i <= E; i += NUM_THREADS) {
    s_off[i] = args.offsets[i];
    s_mp[i] = args.mprefix[i];
  }
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < SA; ++s) {
      mbar_init(bar_fullA(s), 1);
      mbar_init(bar_emptyA(s), 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(bar_fullB(s), DEQ_THREADS);
      mbar_init(bar_emptyB(s), 1);
      mbar_init(bar_peerFull(s), 1);
    }
    for (int s = 0; s < SC; ++s) {
      mbar_init(bar_fullC(s), 1);
      mbar_init(bar_emptyC(s), DEQ_THREADS);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_accFull(s), 1);
      mbar_init(bar_accEmpty(s), 4 * 32);
      mbar_init(bar_peerAcc(s), 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmS);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(misc), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];

  const int total = s_mp[E] * args.n_tiles;
  const int KB = (args.K + BK - 1) / BK;

  if (warp == 0) {
    // ------------------------------------------- producer: activations --
    if (lane == 0) {
      int sa = 0, pa = 0;
      bool ok = true;
      for (int tile = pair_id; tile < total && ok; tile += npairs) {
        TileInfo ti;
        decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
        const int rAct = ti.row0 + static_cast<int>(rank) * BMH;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait_cluster(bar_emptyA(sa), pa ^ 1, abort_flag, args.status))) break;
          mbar_expect_tx(bar_fullA(sa), A_BYTES);
          tma_load_2d(sbase + OFF_A + sa * A_BYTES, &tmA, kb * BK, rAct, bar_fullA(sa));
          if (++sa == SA) { sa = 0; pa ^= 1; }
        }
      }
    }
  } else if (warp == 2) {
    // -------------------------------------- producer: codes and scales --
    if (lane == 0) {
      int sc = 0, pc = 0;
      bool ok = true;
      for (int tile = pair_id; tile < total && ok; tile += npairs) {
        TileInfo ti;
        decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
        const int rW = ti.nt * args.row_step + static_cast<int>(rank) * args.half_off;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_emptyC(sc), pc ^ 1, abort_flag, args.status))) break;
          const uint32_t cdst = sbase + OFF_C + sc * C_BYTES;
          mbar_expect_tx(bar_fullC(sc), C_TX);
          tma_load_3d(cdst, &tmB, kb * (BK / 2), rW, ti.e, bar_fullC(sc));
          tma_load_3d(cdst + S_OFF, &tmS, rW & ~15, 2 * kb, ti.e, bar_fullC(sc));
          if (++sc == SC) { sc = 0; pc ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------- UMMA issuer (even CTA) --
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * BMH, BN);
      int sa = 0, pa = 0, sb = 0, pb = 0, it = 0;
      bool ok = true;
      for (int tile = pair_id; tile < total && ok; tile += npairs, ++it) {
        const int ab = it & 1;
        const uint32_t ap = (it >> 1) & 1;
        if (!(ok = mbar_wait(bar_accEmpty(ab), ap ^ 1, abort_flag, args.status))) break;
        if (!(ok = mbar_wait_cluster(bar_peerAcc(ab), ap ^ 1, abort_flag, args.status))) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * ACC_COLS;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_fullA(sa), pa, abort_flag, args.status))) break;
          if (!(ok = mbar_wait(bar_fullB(sb), pb, abort_flag, args.status))) break;
          if (!(ok = mbar_wait_cluster(bar_peerFull(sb), pb, abort_flag, args.status))) break;
          tc_fence_after();
          const uint32_t a_addr = sbase + OFF_A + sa * A_BYTES;
          const uint32_t b_addr = sbase + OFF_B + sb * B_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_pair(d, sdesc_k_sw128(a_addr + kk * 32), sdesc_k_sw128(b_addr + kk * 32),
                           idesc, (kb | kk) != 0);
          umma_commit_pair(bar_emptyA(sa));
          umma_commit_pair(bar_emptyB(sb));
          if (++sa == SA) { sa = 0; pa ^= 1; }
          if (++sb == SB) { sb = 0; pb ^= 1; }
        }
        if (ok) umma_commit_pair(bar_accFull(ab));
      }
    }
  } else if (warp == 3) {
    // ------------------------------------ stage relay (odd CTA) --
    if (rank == 1 && lane == 0) {
      int sa = 0, pa = 0, sb = 0, pb = 0;
      bool ok = true;
      for (int tile = pair_id; tile < total && ok; tile += npairs) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_fullA(sa), pa, abort_flag, args.status))) break;
          if (!(ok = mbar_wait(bar_fullB(sb), pb, abort_flag, args.status))) break;
          // relaxed: a release at cluster scope per k-block cost about as much
          // as the k-block itself; the stage was already observed complete
          mbar_arrive_remote_relaxed(mapa_shared(bar_peerFull(sb), 0));
          if (++sa == SA) { sa = 0; pa ^= 1; }
          if (++sb == SB) { sb = 0; pb ^= 1; }
        }
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ----------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    int it = 0;
    for (int tile = pair_id; tile < total; tile += npairs, ++it) {
      TileInfo ti;
      decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
      const int ab = it & 1;
      const uint32_t ap = (it >> 1) & 1;
      if (!mbar_wait_cluster(bar_accFull(ab), ap, abort_flag, args.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + ab * ACC_COLS;
      const int r = static_cast<int>(rank) * BMH + quad * 32 + lane;
      const bool valid = r < ti.rows;
      const int64_t grow = ti.row0 + r;
      if (EPI == EPI_SWIGLU) {
        // columns 0..119 gate (even CTA's rows), 120..239 up (odd CTA's rows)
        const int col0 = ti.nt * NH;
        uint16_t* orow = args.out + grow * args.n_out;
        const float* brow = args.bias ? args.bias + static_cast<int64_t>(ti.e) * 2 * args.n_out
                                      : nullptr;
#pragma unroll 1
        for (int c = 0; c < NH; c += 8) {
          uint32_t g[8], u[8];
          tmem_ld8x2_sync(taddr + c, taddr + NH + c, g, u);
          const int col = col0 + c;
          float bg[8], bu[8];
          load_bias8x2(brow, col, args.n_out, bg, bu);
          float h[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            h[i] = silu_f(__uint_as_float(g[i]) + bg[i]) * (__uint_as_float(u[i]) + bu[i]);
          if (valid && col < args.n_out) {
            *reinterpret_cast<uint4*>(orow + col) =
                make_uint4(pack_bf16x2(h[0], h[4]), pack_bf16x2(h[1], h[5]),
                           pack_bf16x2(h[2], h[6]), pack_bf16x2(h[3], h[7]));
          }
        }
      } else {
        const int col0 = ti.nt * BN;
        int pr = 0;
        float w = 0.f;
        if (valid) {
          pr = args.perm[grow];
          w = args.topk_w[pr];
        }
        float* orow = args.out_f32 + static_cast<int64_t>(pr) * args.n_out;
        const float* brow = args.bias ? args.bias + static_cast<int64_t>(ti.e) * args.n_out
                                      : nullptr;
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          uint32_t y[16];
          tmem_ld16_sync(taddr + c, y);
          const int col = col0 + c;
          if (valid && col < args.n_out) {
            float b[16];
            load_bias16(brow, col, b);
            float4* dst = reinterpret_cast<float4*>(orow + col);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(w * (__uint_as_float(y[4 * i]) + b[4 * i]),
                                   w * (__uint_as_float(y[4 * i + 1]) + b[4 * i + 1]),
                                   w * (__uint_as_float(y[4 * i + 2]) + b[4 * i + 2]),
                                   w * (__uint_as_float(y[4 * i + 3]) + b[4 * i + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_accEmpty(ab));
      if (rank == 1 && threadIdx.x == 4 * 32) {
        // accumulator relay: once all 128 epilogue threads of this CTA have
        // released the buffer, tell the even CTA's UMMA issuer
        if (!mbar_wait(bar_accEmpty(ab), ap, abort_flag, args.status)) break;
        mbar_arrive_remote(mapa_shared(bar_peerAcc(ab), 0));
      }
    }
  } else {
    // ----------------------------------------------------------- decoders --
    const int t = threadIdx.x - 8 * 32;
    const int n = t >> 1;             // weight row of this CTA (0..119 active)
    const int g = t & 1;
    const bool active = n < NH;
    const int sw = n & 7;
    int sc = 0, pc = 0, sb = 0, pb = 0;
    bool ok = true;
    for (int tile = pair_id; tile < total && ok; tile += npairs) {
      TileInfo ti;
      decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
      const int rW = ti.nt * args.row_step + static_cast<int>(rank) * args.half_off;
      const int soff = S_OFF + g * S_ROWS + (rW & 15) + (active ? n : 0);
      for (int kb = 0; kb < KB; ++kb) {
        if (!(ok = mbar_wait(bar_fullC(sc), pc, abort_flag, args.status))) break;
        const uint8_t* stage = smem + OFF_C + sc * C_BYTES;
        uint4 q = make_uint4(0, 0, 0, 0);
        uint32_t sv = 0;
        if (active) {
          q = *reinterpret_cast<const uint4*>(stage + n * 32 + g * 16);
          sv = stage[soff];
        }
        uint4 o[4];
        mxfp4x32_to_bf16(q, sv, o);
        if (!(ok = mbar_wait_cluster(bar_emptyB(sb), pb ^ 1, abort_flag, args.status))) break;
        if (active) {
          uint8_t* brow = smem + OFF_B + sb * B_BYTES + n * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(brow + (((4 * g + c) ^ sw) << 4)) = o[c];
        }
        // one proxy fence for the code-stage reads and the decoded-weight
        // writes (see the single-CTA kernel)
        fence_proxy_async_smem();
        mbar_arrive(bar_emptyC(sc));
        if (++sc == SC) { sc = 0; pc ^= 1; }
        mbar_arrive(bar_fullB(sb));
        if (++sb == SB) { sb = 0; pb ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ================================================================= swap ====
// Decode-sized variant (few routed rows per expert): the operands swap roles.
// The decoded weight tile is the UMMA A operand (M = 128 weight rows) and the
// expert's routed rows are B (N = 64 tokens), so the tensor work follows the
// actual token count instead of a 128/256-row tile, and the kernel streams
// weights. The decoders store the decoded rows straight into tensor memory
// (tcgen05.st, one TMEM lane per weight row) and the UMMA reads A from there:
// decoded weights never pass through shared memory, whose bandwidth would
// otherwise bound the weight stream. For gate/up a tile holds 64 gate rows
// and the matching 64 up rows interleaved (gate j in lane 2j, up j in lane
// 2j+1), so the SwiGLU epilogue pairs adjacent lanes with one shuffle. Each
// CTA builds its tile table (expert, weight block, token block) from the
// device offsets; experts with no tokens cost nothing.
namespace swp {

constexpr int MW = 128;               // weight rows per tile (UMMA M = TMEM lanes)
constexpr int NT = 64;                // tokens per tile (UMMA N)
constexpr int BK = 64;
constexpr int NH = 64;                // weight rows per TMA box
constexpr int ST = 6, SW = 8, SC = 12;
constexpr int T_BYTES = NT * BK * 2;        // 8192
constexpr int C_CODES = MW * BK / 2;        // 4096
constexpr int S_OFF0 = C_CODES, S_OFF1 = C_CODES + 128;
constexpr int C_TX = C_CODES + 2 * NH * 2;
constexpr int C_BYTES = 4352;
constexpr int NUM_THREADS = 512;
constexpr int DEQ_THREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int A_COL0 = 2 * NT;              // decoded weight stages after the accumulators
constexpr int A_COLS = BK / 2;              // 32 columns (64 bf16 of K) per stage
static_assert(A_COL0 + SW * A_COLS <= TMEM_COLS, "TMEM budget");

constexpr int OFF_T = 0;
constexpr int OFF_C = OFF_T + ST * T_BYTES;
constexpr int OFF_BAR = OFF_C + SC * C_BYTES;
constexpr int NUM_BARS = 2 * ST + 2 * SW + 2 * SC + 4;
constexpr int OFF_MISC = (OFF_BAR + NUM_BARS * 8 + 15) & ~15;
constexpr int OFF_TAB = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_TAB + 2 * (MAX_E + 1) * 4;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(OFF_C % 1024 == 0, "alignment");

}  // namespace swp

// position of element e (0..7) inside a chunk stored in kPerm8 order
__device__ __forceinline__ int perm8_pos(int e) { return e < 4 ? 2 * e : 2 * (e - 4) + 1; }

template <int EPI>
__global__ void __launch_bounds__(swp::NUM_THREADS, 1)
    grouped_mxfp4_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmA,
                                   const __grid_constant__ CUtensorMap tmB,
                                   const __grid_constant__ CUtensorMap tmS, const Args args) {
  pdl_wait_and_trigger();
  // local copies shadow the single-CTA kernel's constants of the same names
  constexpr int MW = swp::MW, NT = swp::NT, BK = swp::BK, NH = swp::NH;
  constexpr int ST = swp::ST, SW = swp::SW, SC = swp::SC;
  constexpr int T_BYTES = swp::T_BYTES, C_BYTES = swp::C_BYTES;
  constexpr int C_TX = swp::C_TX, S_OFF0 = swp::S_OFF0, S_OFF1 = swp::S_OFF1;
  constexpr int A_COL0 = swp::A_COL0, A_COLS = swp::A_COLS;
  constexpr int OFF_T = swp::OFF_T, OFF_C = swp::OFF_C;
  constexpr int OFF_BAR = swp::OFF_BAR, OFF_MISC = swp::OFF_MISC, OFF_TAB = swp::OFF_TAB;
  constexpr int NUM_THREADS = swp::NUM_THREADS, DEQ_THREADS = swp::DEQ_THREADS;
  constexpr int TMEM_COLS = swp::TMEM_COLS;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar0 = sbase + OFF_BAR;
  auto bar_fullT = [&](int s) { return bar0 + 8u * s; };
  auto bar_emptyT = [&](int s) { return bar0 + 8u * (ST + s); };
  auto bar_fullW = [&](int s) { return bar0 + 8u * (2 * ST + s); };
  auto bar_emptyW = [&](int s) { return bar0 + 8u * (2 * ST + SW + s); };
  auto bar_fullC = [&](int s) { return bar0 + 8u * (2 * ST + 2 * SW + s); };
  auto bar_emptyC = [&](int s) { return bar0 + 8u * (2 * ST + 2 * SW + SC + s); };
  auto bar_accFull = [&](int s) { return bar0 + 8u * (2 * ST + 2 * SW + 2 * SC + s); };
  auto bar_accEmpty = [&](int s) { return bar0 + 8u * (2 * ST + 2 * SW + 2 * SC + 2 + s); };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* s_off = reinterpret_cast<int*>(smem + OFF_TAB);
  int* s_tp = s_off + (MAX_E + 1);   // prefix of tiles per expert

  const int E = args.E;
  for (int i = threadIdx.x; i <= E; i += NUM_THREADS) s_off[i] = args.offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      s_tp[e] = acc;
      const int cnt = s_off[e + 1] - s_off[e];
      acc += ((cnt + NT - 1) / NT) * args.n_tiles;
    }
    s_tp[E] = acc;
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar_fullT(s), 1);
      mbar_init(bar_emptyT(s), 1);
    }
    for (int s = 0; s < SW; ++s) {
      mbar_init(bar_fullW(s), DEQ_THREADS);
      mbar_init(bar_emptyW(s), 1);
    }
    for (int s = 0; s < SC; ++s) {
      mbar_init(bar_fullC(s), 1);
      mbar_init(bar_emptyC(s), DEQ_THREADS);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_accFull(s), 1);
      mbar_init(bar_accEmpty(s), 4 * 32);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmS);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];

  const int total = s_tp[E];
  const int KB = (args.K + BK - 1) / BK;
  // tile -> (expert, weight block, token block); tiles of an expert are
  // weight-block major so that consecutive CTAs stream consecutive weights
  auto decode = [&](int tile, int& e, int& wb, int& row0, int& rows) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_tp[mid] <= tile) lo = mid; else hi = mid;
    }
    e = lo;
    const int cnt = s_off[e + 1] - s_off[e];
    const int ntb = (cnt + NT - 1) / NT;
    const int local = tile - s_tp[e];
    wb = local / ntb;
    const int tb = local % ntb;
    row0 = s_off[e] + tb * NT;
    rows = min(NT, cnt - tb * NT);
  };
  if (warp == 3) return;  // no role

  if (warp == 0) {
    // ------------------------------------------------ producer: tokens --
    if (lane == 0) {
      int st = 0, pt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, wb, row0, rows;
        decode(tile, e, wb, row0, rows);
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_emptyT(st), pt ^ 1, abort_flag, args.status))) break;
          mbar_expect_tx(bar_fullT(st), T_BYTES);
          tma_load_2d(sbase + OFF_T + st * T_BYTES, &tmA, kb * BK, row0, bar_fullT(st));
          if (++st == ST) { st = 0; pt ^= 1; }
        }
      }
    }
  } else if (warp == 2) {
    // --------------------------------------- producer: codes and scales --
    if (lane == 0) {
      int sc = 0, pc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, wb, row0, rows;
        decode(tile, e, wb, row0, rows);
        const int rA = wb * args.row_step;
        const int rB = rA + args.half_off;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_emptyC(sc), pc ^ 1, abort_flag, args.status))) break;
          const uint32_t cdst = sbase + OFF_C + sc * C_BYTES;
          mbar_expect_tx(bar_fullC(sc), C_TX);
          tma_load_3d(cdst, &tmB, kb * (BK / 2), rA, e, bar_fullC(sc));
          tma_load_3d(cdst + NH * (BK / 2), &tmB, kb * (BK / 2), rB, e, bar_fullC(sc));
          tma_load_3d(cdst + S_OFF0, &tmS, rA, 2 * kb, e, bar_fullC(sc));
          tma_load_3d(cdst + S_OFF1, &tmS, rB, 2 * kb, e, bar_fullC(sc));
          if (++sc == SC) { sc = 0; pc ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- UMMA issuer --
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(MW, NT);
      int st = 0, pt = 0, sw = 0, pw = 0, it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t ap = (it >> 1) & 1;
        if (!(ok = mbar_wait(bar_accEmpty(ab), ap ^ 1, abort_flag, args.status))) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * NT;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_fullT(st), pt, abort_flag, args.status))) break;
          if (!(ok = mbar_wait(bar_fullW(sw), pw, abort_flag, args.status))) break;
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + A_COL0 + sw * A_COLS;
          const uint32_t t_addr = sbase + OFF_T + st * T_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_tmem_a(d, a_tmem + kk * 8, sdesc_k_sw128(t_addr + kk * 32), idesc,
                             (kb | kk) != 0);
          umma_commit(bar_emptyT(st));
          umma_commit(bar_emptyW(sw));
          if (++st == ST) { st = 0; pt ^= 1; }
          if (++sw == SW) { sw = 0; pw ^= 1; }
        }
        if (ok) umma_commit(bar_accFull(ab));
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ----------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    const int r = quad * 32 + lane;          // weight row of the tile = TMEM lane
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      int e, wb, row0, rows;
      decode(tile, e, wb, row0, rows);
      const int ab = it & 1;
      const uint32_t ap = (it >> 1) & 1;
      if (!mbar_wait(bar_accFull(ab), ap, abort_flag, args.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + ab * NT;
      // this lane's weight row carries one bias value for the whole tile
      float bl = 0.f;
      if (args.bias) {
        if (EPI == EPI_SWIGLU) {
          const int jb = wb * NH + (r >> 1);
          if (jb < args.n_out)
            bl = args.bias[static_cast<int64_t>(e) * 2 * args.n_out + (r & 1) * args.n_out + jb];
        } else if (wb * MW + r < args.n_out) {
          bl = args.bias[static_cast<int64_t>(e) * args.n_out + wb * MW + r];
        }
      }
#pragma unroll 1
      for (int c = 0; c < NT && c < rows; c += 16) {
        uint32_t y[16];
        tmem_ld16_sync(taddr + c, y);
        if (EPI == EPI_SWIGLU) {
          // even lanes hold gate row j = r/2, odd lanes the up row j
          const int j = wb * NH + (r >> 1);
          const int col = (j & ~7) + perm8_pos(j & 7);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float v = __uint_as_float(y[i]) + bl;
            const float u = __shfl_xor_sync(0xFFFFFFFFu, v, 1);
            if (!(lane & 1) && c + i < rows && j < args.n_out) {
              const float h = silu_f(v) * u;
              const __nv_bfloat16 hb = __float2bfloat16_rn(h);
              args.out[static_cast<int64_t>(row0 + c + i) * args.n_out + col] =
                  *reinterpret_cast<const uint16_t*>(&hb);
            }
          }
        } else {
          const int col = wb * MW + r;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (c + i < rows) {
              const int pr = args.perm[row0 + c + i];
              const float w = args.topk_w[pr];
              if (col < args.n_out)
                args.out_f32[static_cast<int64_t>(pr) * args.n_out + col] =
                    w * (__uint_as_float(y[i]) + bl);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_accEmpty(ab));
    }
  } else if (warp >= 8) {
    // ----------------------------------------------------------- decoders --
    // Warp 8+q and warp 12+q both serve TMEM lanes 32q..32q+31 (one weight
    // row per lane); the first decodes scale group 0 of the k-block (columns
    // 0..15 of the stage), the second group 1 (columns 16..31).
    const int wl = warp - 8;
    const int quad = wl & 3, g = wl >> 2;
    const int r = quad * 32 + lane;  // TMEM lane = weight row of the tile
    // source row in the code stage: SwiGLU lanes interleave gate row r/2
    // (first box) and up row r/2 (second box)
    const int n = (EPI == EPI_SWIGLU) ? ((r & 1) ? NH + (r >> 1) : (r >> 1)) : r;
    const int soff = (n < NH ? S_OFF0 : S_OFF1) + g * NH + (n & (NH - 1));
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + A_COL0 +
                               g * (A_COLS / 2);
    int sc = 0, pc = 0, sw = 0, pw = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        if (!(ok = mbar_wait(bar_fullC(sc), pc, abort_flag, args.status))) break;
        const uint8_t* stage = smem + OFF_C + sc * C_BYTES;
        const uint4 q = *reinterpret_cast<const uint4*>(stage + n * 32 + g * 16);
        const uint32_t sv = stage[soff];
        // the next TMA write into this code stage must not overtake these reads
        fence_proxy_async_smem();
        mbar_arrive(bar_emptyC(sc));
        if (++sc == SC) { sc = 0; pc ^= 1; }
        uint4 o[4];
        mxfp4x32_to_bf16(q, sv, o);
        if (!(ok = mbar_wait(bar_emptyW(sw), pw ^ 1, abort_flag, args.status))) break;
        tc_fence_after();
        tmem_st16_sync(lane_addr + sw * A_COLS, o);
        tc_fence_before();
        mbar_arrive(bar_fullW(sw));
        if (++sw == SW) { sw = 0; pw ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ----------------------------------------------------------- host side ----

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
            const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
            CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, dt, rank, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Activations [rows][K] bf16, box 64 x 128, 128-byte swizzle.
bool make_act_map(CUtensorMap* m, const void* base, int rows, int K) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {BK, BMH};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                CU_TENSOR_MAP_SWIZZLE_128B);
}

// Codes [E][Nrows][K/2] uint8, box 32 bytes x 64 rows x 1 expert.
bool make_code_map(CUtensorMap* m, const void* base, int E, int Nrows, int K) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(Nrows),
                              static_cast<cuuint64_t>(E)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K / 2),
                                 static_cast<cuuint64_t>(K / 2) * static_cast<cuuint64_t>(Nrows)};
  const cuuint32_t box[3] = {BK / 2, NH, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Transposed scales [E][K/32][Nrows] uint8, box `rows` x 2 groups x 1 expert.
bool make_scale_map(CUtensorMap* m, const void* base, int E, int Nrows, int K, int rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(Nrows), static_cast<cuuint64_t>(K / 32),
                              static_cast<cuuint64_t>(E)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(Nrows),
                                 static_cast<cuuint64_t>(Nrows) * static_cast<cuuint64_t>(K / 32)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(rows), 2, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Codes [E][Nrows][K/2] uint8, box 32 bytes x `rows` rows x 1 expert.
bool make_code_map_rows(CUtensorMap* m, const void* base, int E, int Nrows, int K, int rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(Nrows),
                              static_cast<cuuint64_t>(E)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K / 2),
                                 static_cast<cuuint64_t>(K / 2) * static_cast<cuuint64_t>(Nrows)};
  const cuuint32_t box[3] = {BK / 2, static_cast<cuuint32_t>(rows), 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Activation rows [rows][K] bf16 as the swap kernel's B operand: box 64 x 64.
bool make_tok_map(CUtensorMap* m, const void* base, int rows, int K) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {swp::BK, swp::NT};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int EPI>
cudaError_t launch_swap_impl(const GroupedGemmProblem& p, int num_sms, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_mxfp4_gemm_swap_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         swp::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tmA, tmB, tmS;
  if (!make_tok_map(&tmA, p.A, p.P, p.K)) return cudaErrorInvalidValue;
  if (!make_code_map_rows(&tmB, p.codes, p.E, p.Nrows, p.K, swp::NH)) return cudaErrorInvalidValue;
  if (!make_scale_map(&tmS, p.scales_t, p.E, p.Nrows, p.K, swp::NH)) return cudaErrorInvalidValue;
  Args a;
  a.offsets = p.offsets;
  a.mprefix = p.mprefix;
  a.E = p.E;
  a.K = p.K;
  a.Nrows = p.Nrows;
  a.n_out = p.n_out;
  a.out = p.out;
  a.out_f32 = p.out_f32;
  a.perm = p.perm;
  a.topk_w = p.topk_w;
  a.bias = p.bias;
  a.status = p.status;
  if (EPI == EPI_SWIGLU) {
    a.n_tiles = (p.n_out + swp::NH - 1) / swp::NH;   // weight blocks of 64 gate + 64 up rows
    a.row_step = swp::NH;
    a.half_off = p.n_out;
  } else {
    a.n_tiles = (p.n_out + swp::MW - 1) / swp::MW;   // weight blocks of 128 output rows
    a.row_step = swp::MW;
    a.half_off = swp::NH;
  }
  const int64_t tiles_bound =
      ((static_cast<int64_t>(p.P) + swp::NT - 1) / swp::NT + p.E) * a.n_tiles;
  const int grid = static_cast<int>(tiles_bound < num_sms ? tiles_bound : num_sms);
  launch_kernel(grouped_mxfp4_gemm_swap_kernel<EPI>, dim3(grid), dim3(swp::NUM_THREADS), swp::SMEM_ALLOC, st, tmA, tmB,
                                                                                      tmS, a);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_pair_impl(const GroupedGemmProblem& p, int num_sms, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_mxfp4_gemm_pair_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         pair::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tmA, tmB, tmS;
  if (!make_act_map(&tmA, p.A, p.P, p.K)) return cudaErrorInvalidValue;
  if (!make_code_map_rows(&tmB, p.codes, p.E, p.Nrows, p.K, pair::NH)) return cudaErrorInvalidValue;
  if (!make_scale_map(&tmS, p.scales_t, p.E, p.Nrows, p.K, pair::S_ROWS))
    return cudaErrorInvalidValue;
  Args a;
  a.offsets = p.offsets;
  a.mprefix = p.mprefix;
  a.E = p.E;
  a.K = p.K;
  a.Nrows = p.Nrows;
  a.n_out = p.n_out;
  a.out = p.out;
  a.out_f32 = p.out_f32;
  a.perm = p.perm;
  a.topk_w = p.topk_w;
  a.bias = p.bias;
  a.status = p.status;
  if (EPI == EPI_SWIGLU) {
    a.n_tiles = (p.n_out + pair::NH - 1) / pair::NH;
    a.row_step = pair::NH;
    a.half_off = p.n_out;   // the odd CTA decodes the up rows
  } else {
    a.n_tiles = (p.n_out + pair::BN - 1) / pair::BN;
    a.row_step = pair::BN;
    a.half_off = pair::NH;
  }
  const int64_t mt_bound = (static_cast<int64_t>(p.P) + BM - 1) / BM + p.E;
  const int64_t tiles_bound = mt_bound * a.n_tiles;
  int64_t pairs = num_sms / 2;
  if (tiles_bound < pairs) pairs = tiles_bound;
  const int grid = static_cast<int>(2 * pairs);
  launch_kernel(grouped_mxfp4_gemm_pair_kernel<EPI>, dim3(grid), dim3(pair::NUM_THREADS), pair::SMEM_ALLOC, st, tmA, tmB,
                                                                                      tmS, a);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_impl(const GroupedGemmProblem& p, int num_sms, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_mxfp4_gemm_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tmA, tmB, tmS;
  if (!make_act_map(&tmA, p.A, p.P, p.K)) return cudaErrorInvalidValue;
  if (!make_code_map(&tmB, p.codes, p.E, p.Nrows, p.K)) return cudaErrorInvalidValue;
  if (!make_scale_map(&tmS, p.scales_t, p.E, p.Nrows, p.K, NH)) return cudaErrorInvalidValue;
  Args a;
  a.offsets = p.offsets;
  a.mprefix = p.mprefix;
  a.E = p.E;
  a.K = p.K;
  a.Nrows = p.Nrows;
  a.n_out = p.n_out;
  a.out = p.out;
  a.out_f32 = p.out_f32;
  a.perm = p.perm;
  a.topk_w = p.topk_w;
  a.bias = p.bias;
  a.status = p.status;
  if (EPI == EPI_SWIGLU) {
    a.n_tiles = (p.n_out + NH - 1) / NH;
    a.row_step = NH;
    a.half_off = p.n_out;   // up rows start at I
  } else {
    a.n_tiles = (p.n_out + BN - 1) / BN;
    a.row_step = BN;
    a.half_off = NH;
  }
  // upper bound of the tile count: every expert may add one partial M tile
  const int64_t mt_bound = (static_cast<int64_t>(p.P) + BM - 1) / BM + p.E;
  const int64_t tiles_bound = mt_bound * a.n_tiles;
  const int grid = static_cast<int>(tiles_bound < num_sms ? tiles_bound : num_sms);
  launch_kernel(grouped_mxfp4_gemm_kernel<EPI>, dim3(grid), dim3(NUM_THREADS), SMEM_ALLOC, st, tmA, tmB, tmS, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_gateup_swiglu(const GroupedGemmProblem& p, int num_sms, cudaStream_t st) {
  if (p.tiles == TILES_SWAP) return launch_swap_impl<EPI_SWIGLU>(p, num_sms, st);
  if (p.tiles == TILES_PAIR) return launch_pair_impl<EPI_SWIGLU>(p, num_sms, st);
  return launch_impl<EPI_SWIGLU>(p, num_sms, st);
}

cudaError_t launch_gemm_down_combine(const GroupedGemmProblem& p, int num_sms, cudaStream_t st) {
  if (p.tiles == TILES_SWAP) return launch_swap_impl<EPI_DOWN>(p, num_sms, st);
  if (p.tiles == TILES_PAIR) return launch_pair_impl<EPI_DOWN>(p, num_sms, st);
  return launch_impl<EPI_DOWN>(p, num_sms, st);
}

}  // namespace moe
