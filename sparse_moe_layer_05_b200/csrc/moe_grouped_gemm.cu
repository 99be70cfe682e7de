// moe_grouped_gemm.cu -- expert-grouped MXFP4 GEMMs on the sm_100a tensor
// cores (tcgen05, TMEM accumulators, TMA-fed shared memory).
//
//   gate/up:  for the rows r of expert e (permuted order),
//             H[r, n] = silu(x_r . Wgate[e][n]) * (x_r . Wup[e][n])
//   down:     Yw[pair(r), m] = p(pair(r)) * (H[r] . Wdown[e][m])
//
// Field guide "gpt-oss 20B", "03 Sparse Mixture of Experts" (SwiGLU experts,
// weighted sum); "shrink/gpt_oss-mic", "Preserved properties" (silu);
// "gpt-oss-20b and gpt-oss-120b", "Four-bit expert weights" (MXFP4).
//
// One persistent CTA per SM walks the tiles (expert, n tile, m tile) that the
// device-side routing tables define; no host synchronisation is needed.
// Warp roles inside a CTA (512 threads):
//   warp 0      TMA producer: activation tile (bf16, 128B swizzle) and the two
//               MXFP4 code boxes of the weight tile
//   warp 1      TMEM allocator and UMMA issuer (one elected thread)
//   warps 4-7   epilogue: TMEM -> registers -> SwiGLU / weighted store
//   warps 8-15  decoders: MXFP4 codes -> bf16 weight tile in the 128B
//               swizzled K-major layout the UMMA descriptor expects
// Accumulators: two 128 x 240 fp32 buffers in TMEM (512 columns allocated),
// so the epilogue of one tile overlaps the main loop of the next.
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {
namespace {

constexpr int BM = kTileM;        // rows per tile
constexpr int BK = 64;            // contraction elements per k-block (128 B of bf16)
constexpr int NH = 120;           // weight rows per TMA box (one half of the tile)
constexpr int BN = 2 * NH;        // UMMA N
constexpr int SA = 4;             // activation stages
constexpr int SB = 3;             // decoded weight stages
constexpr int SC = 4;             // code stages
constexpr int A_BYTES = BM * BK * 2;   // 16384
constexpr int B_BYTES = BN * BK * 2;   // 30720
constexpr int C_BYTES = BN * BK / 2;   // 7680
constexpr int NUM_THREADS = 512;
constexpr int EPI_WARP0 = 4;
constexpr int DEQ_WARP0 = 8;
constexpr int DEQ_THREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;     // column distance between the two accumulators
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

enum Epi { EPI_SWIGLU = 0, EPI_DOWN = 1 };

struct Args {
  const uint8_t* scales;
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

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_mxfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmB, const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  const uint32_t bar0 = smem_u32(bars);
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
  const int KG = args.K / 32;  // scale groups per row

  if (warp == 0) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      int sa = 0, pa = 0, sc = 0, pc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        TileInfo ti;
        decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
        const int rA = ti.nt * args.row_step;
        const int rB = rA + args.half_off;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_emptyA(sa), pa ^ 1, abort_flag, args.status))) break;
          mbar_expect_tx(bar_fullA(sa), A_BYTES);
          tma_load_2d(sbase + OFF_A + sa * A_BYTES, &tmA, kb * BK, ti.row0, bar_fullA(sa));
          if (++sa == SA) { sa = 0; pa ^= 1; }
          if (!(ok = mbar_wait(bar_emptyC(sc), pc ^ 1, abort_flag, args.status))) break;
          mbar_expect_tx(bar_fullC(sc), C_BYTES);
          const uint32_t cdst = sbase + OFF_C + sc * C_BYTES;
          tma_load_3d(cdst, &tmB, kb * (BK / 2), rA, ti.e, bar_fullC(sc));
          tma_load_3d(cdst + NH * (BK / 2), &tmB, kb * (BK / 2), rB, ti.e, bar_fullC(sc));
          if (++sc == SC) { sc = 0; pc ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- UMMA issuer --
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN);
      int sa = 0, pa = 0, sb = 0, pb = 0, it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t ap = (it >> 1) & 1;
        if (!(ok = mbar_wait(bar_accEmpty(ab), ap ^ 1, abort_flag, args.status))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * ACC_COLS;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_fullA(sa), pa, abort_flag, args.status))) break;
          if (!(ok = mbar_wait(bar_fullB(sb), pb, abort_flag, args.status))) break;
          tc_fence_after();
          const uint32_t a_addr = sbase + OFF_A + sa * A_BYTES;
          const uint32_t b_addr = sbase + OFF_B + sb * B_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            umma_bf16(d_tmem, sdesc_k_sw128(a_addr + kk * 32), sdesc_k_sw128(b_addr + kk * 32),
                      idesc, (kb | kk) != 0);
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
    const int r = quad * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      TileInfo ti;
      decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
      const int ab = it & 1;
      const uint32_t ap = (it >> 1) & 1;
      if (!mbar_wait(bar_accFull(ab), ap, abort_flag, args.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + ab * ACC_COLS;
      const bool valid = r < ti.rows;
      const int64_t grow = ti.row0 + r;
      if (EPI == EPI_SWIGLU) {
        const int col0 = ti.nt * NH;
        uint16_t* orow = args.out + grow * args.n_out;
#pragma unroll 1
        for (int c = 0; c < NH; c += 8) {
          uint32_t g[8], u[8];
          tmem_ld8(taddr + c, g);
          tmem_ld8(taddr + NH + c, u);
          tmem_ld_wait();
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
            o[i] = pack_bf16x2(silu_f(g0) * u0, silu_f(g1) * u1);
          }
          const int col = col0 + c;
          if (valid) {
            if (col + 8 <= args.n_out) {
              *reinterpret_cast<uint4*>(orow + col) = make_uint4(o[0], o[1], o[2], o[3]);
            } else {
              for (int i = 0; i < 8 && col + i < args.n_out; ++i)
                orow[col + i] = static_cast<uint16_t>(o[i >> 1] >> (16 * (i & 1)));
            }
          }
        }
      } else {
        // weighted un-permute: fp32 row p * y of pair perm[row], stored at
        // yw[pair] so that the per-token sum reads k contiguous rows
        const int col0 = ti.nt * BN;
        int pair = 0;
        float w = 0.f;
        if (valid) {
          pair = args.perm[grow];
          w = args.topk_w[pair];
        }
        float* orow = args.out_f32 + static_cast<int64_t>(pair) * args.n_out;
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          uint32_t y[16];
          tmem_ld16(taddr + c, y);
          tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = w * __uint_as_float(y[i]);
          const int col = col0 + c;
          if (valid) {
            if (col + 16 <= args.n_out) {
              float4* dst = reinterpret_cast<float4*>(orow + col);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (col + i < args.n_out) orow[col + i] = v[i];
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_accEmpty(ab));
    }
  } else if (warp >= DEQ_WARP0) {
    // ----------------------------------------------------------- decoders --
    const int n = threadIdx.x - DEQ_WARP0 * 32;   // weight row inside the tile
    const bool active = n < BN;
    int sc = 0, pc = 0, sb = 0, pb = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      TileInfo ti;
      decode_tile(tile, args.n_tiles, E, s_off, s_mp, ti);
      const int rA = ti.nt * args.row_step;
      const int wrow = (n < NH) ? rA + n : rA + args.half_off + (n - NH);
      const bool row_ok = active && wrow < args.Nrows;
      const uint8_t* srow =
          args.scales + (static_cast<int64_t>(ti.e) * args.Nrows + (row_ok ? wrow : 0)) * KG;
      const int sw = n & 7;
      for (int kb = 0; kb < KB; ++kb) {
        uint32_t s0 = 0, s1 = 0;
        if (row_ok) {
          const int g0 = 2 * kb;
          s0 = srow[g0];
          if (g0 + 1 < KG) s1 = srow[g0 + 1];
        }
        if (!(ok = mbar_wait(bar_fullC(sc), pc, abort_flag, args.status))) break;
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;
        if (active) {
          const uint4* src = reinterpret_cast<const uint4*>(smem + OFF_C + sc * C_BYTES + n * 32);
          q0 = src[0];
          q1 = src[1];
        }
        mbar_arrive(bar_emptyC(sc));
        if (++sc == SC) { sc = 0; pc ^= 1; }
        if (!(ok = mbar_wait(bar_emptyB(sb), pb ^ 1, abort_flag, args.status))) break;
        if (active) {
          uint8_t* brow = smem + OFF_B + sb * B_BYTES + n * 128;
          uint4 o[4];
          mxfp4x32_to_bf16(q0, s0, o);
#pragma unroll
          for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(brow + ((c ^ sw) << 4)) = o[c];
          mxfp4x32_to_bf16(q1, s1, o);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(brow + (((c + 4) ^ sw) << 4)) = o[c];
        }
        fence_proxy_async_smem();
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

// [rows][K] bf16, box 64 x 128, 128-byte swizzle.
bool make_act_map(CUtensorMap* m, const void* base, int rows, int K) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t box[2] = {BK, BM};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [E][Nrows][K/2] uint8 codes, box 32 bytes x NH rows x 1 expert.
bool make_code_map(CUtensorMap* m, const void* base, int E, int Nrows, int K) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(Nrows),
                        static_cast<cuuint64_t>(E)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(K / 2),
                           static_cast<cuuint64_t>(K / 2) * static_cast<cuuint64_t>(Nrows)};
  cuuint32_t box[3] = {BK / 2, NH, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
  CUtensorMap tmA, tmB;
  if (!make_act_map(&tmA, p.A, p.P, p.K)) return cudaErrorInvalidValue;
  if (!make_code_map(&tmB, p.codes, p.E, p.Nrows, p.K)) return cudaErrorInvalidValue;
  Args a;
  a.scales = p.scales;
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
  grouped_mxfp4_gemm_kernel<EPI><<<grid, NUM_THREADS, SMEM_ALLOC, st>>>(tmA, tmB, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_gateup_swiglu(const GroupedGemmProblem& p, int num_sms, cudaStream_t st) {
  return launch_impl<EPI_SWIGLU>(p, num_sms, st);
}

cudaError_t launch_gemm_down_combine(const GroupedGemmProblem& p, int num_sms, cudaStream_t st) {
  return launch_impl<EPI_DOWN>(p, num_sms, st);
}

}  // namespace moe
