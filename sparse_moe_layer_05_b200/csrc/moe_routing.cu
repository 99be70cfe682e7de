// moe_routing.cu -- the stable expert permutation, the activation gather and
// the per-token combine (the router itself is moe_router_tc.cu).
//
// Field guide "gpt-oss 20B", "03 Sparse Mixture of Experts": score all
// experts, keep the top k, normalise only those, and sum the weighted expert
// outputs of each token.
#include <cuda_bf16.h>
#include <float.h>
#include <stdint.h>

#include "moe_internal.h"
#include "moe_perm_small.cuh"
#include "moe_ptx.cuh"

namespace moe {
namespace {

// --------------------------------------------------------- K2 histogram ----
__global__ void __launch_bounds__(256) perm_hist_kernel(const int32_t* __restrict__ topk_idx,
                                                        int T, int k, int E,
                                                        int32_t* __restrict__ chunk_hist) {
  pdl_wait_and_trigger();
  __shared__ int h[256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int64_t q0 = (int64_t)blockIdx.x * kPermChunk * k;
  const int64_t q1 = (int64_t)min(T, (blockIdx.x + 1) * kPermChunk) * k;
  for (int64_t q = q0 + threadIdx.x; q < q1; q += blockDim.x) atomicAdd(&h[topk_idx[q]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(size_t)blockIdx.x * E + e] = h[e];
}

// ------------------------------------------------------------- K2 scan ----
// One block. Thread e walks the chunks of expert e; then a block-wide scan of
// the expert counts gives the offsets and the M-tile prefix.
__global__ void __launch_bounds__(256) perm_scan_kernel(const int32_t* __restrict__ chunk_hist,
                                                        int nchunks, int E,
                                                        int32_t* __restrict__ counts,
                                                        int32_t* __restrict__ offsets,
                                                        int32_t* __restrict__ chunk_base,
                                                        int32_t* __restrict__ mtile_prefix) {
  pdl_wait_and_trigger();
  __shared__ int s_cnt[256], s_mt[256];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    for (int b = 0; b < nchunks; ++b) {
      const int c = chunk_hist[(size_t)b * E + e];
      chunk_base[(size_t)b * E + e] = run;
      run += c;
    }
  }
  s_cnt[e] = (e < E) ? run : 0;
  s_mt[e] = (e < E) ? (run + kTileM - 1) / kTileM : 0;
  __syncthreads();
  if (e == 0) {  // E <= 256: a serial scan is cheap and plainly ordered
    int a = 0, m = 0;
    for (int i = 0; i < E; ++i) {
      const int c = s_cnt[i], mt = s_mt[i];
      s_cnt[i] = a;
      s_mt[i] = m;
      a += c;
      m += mt;
    }
    offsets[E] = a;
    mtile_prefix[E] = m;
  }
  __syncthreads();
  if (e < E) {
    offsets[e] = s_cnt[e];
    mtile_prefix[e] = s_mt[e];
    if (counts) counts[e] = run;
    for (int b = 0; b < nchunks; ++b) chunk_base[(size_t)b * E + e] += s_cnt[e];
  }
}

// ---------------------------------------------------------- K2 scatter ----
// Block b owns the pairs of token chunk b; warp w the w-th eighth of them, in
// pair order. Pass 1 counts per (warp, expert); the per-warp bases follow
// from the chunk base; pass 2 ranks pairs inside each 32-pair round with
// match_any, so that the order inside an expert is ascending pair id.
__global__ void __launch_bounds__(256) perm_scatter_kernel(const int32_t* __restrict__ topk_idx,
                                                           int T, int k, int E,
                                                           const int32_t* __restrict__ chunk_base,
                                                           int32_t* __restrict__ perm,
                                                           int32_t* __restrict__ inv) {
  pdl_wait_and_trigger();
  __shared__ int wbase[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 8 * 256; i += blockDim.x) (&wbase[0][0])[i] = 0;
  __syncthreads();
  const int64_t qc0 = (int64_t)blockIdx.x * kPermChunk * k;
  const int64_t qc1 = (int64_t)min(T, (blockIdx.x + 1) * kPermChunk) * k;
  const int64_t seg = (int64_t)(kPermChunk / 8) * k;
  const int64_t q0 = qc0 + warp * seg;
  const int64_t q1 = min(qc1, q0 + seg);
  for (int64_t q = q0 + lane; q < q1; q += 32) atomicAdd(&wbase[warp][topk_idx[q]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = chunk_base[(size_t)blockIdx.x * E + e];
    for (int w = 0; w < 8; ++w) {
      const int c = wbase[w][e];
      wbase[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  for (int64_t qb = q0; qb < q1; qb += 32) {
    const int64_t q = qb + lane;
    const bool valid = q < q1;
    const int e = valid ? topk_idx[q] : -1 - lane;
    const uint32_t m = __match_any_sync(0xFFFFFFFFu, e);
    const int rank = __popc(m & lt);
    int pos = 0;
    if (valid) pos = wbase[warp][e] + rank;
    __syncwarp();
    if (valid && lane == __ffs(m) - 1) wbase[warp][e] += __popc(m);
    __syncwarp();
    if (valid) {
      perm[pos] = (int32_t)q;
      if (inv) inv[q] = pos;
    }
  }
}

// ------------------------------------------------------ K2, small batches ----
// For T <= kPermChunk (one chunk): histogram, scan and stable scatter in one
// block (moe_perm_small.cuh).
__global__ void __launch_bounds__(256) perm_small_kernel(const int32_t* __restrict__ topk_idx,
                                                         int T, int k, int E,
                                                         int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ mtile_prefix,
                                                         int32_t* __restrict__ perm) {
  pdl_wait_and_trigger();
  __shared__ PermSmallSmem sm;
  perm_small_block(topk_idx, T, k, E, counts, offsets, mtile_prefix, perm, sm);
}

// ----------------------------------------------------------- K2 gather ----
// xp[r] = x[perm[r] / k], each 8-element chunk stored in kPerm8 order (the
// operand order of the grouped GEMMs).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ perm, int P,
                                                          int k, int d,
                                                          uint16_t* __restrict__ xp) {
  pdl_wait_and_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int vec = d / 8;  // 16-byte vectors per row
  for (int r = warp; r < P; r += nwarps) {
    const int t = perm[r] / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)r * d);
    for (int c = lane; c < vec; c += 32) dst[c] = chunk8_to_perm(__ldg(src + c));
  }
}

// ------------------------------------------------------------- combine ----
// out[t] = sum_j yw[t*k + j], j ascending, fp32, rounded once to bf16.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ yw, int T, int k,
                                                      int d, const uint16_t* __restrict__ resid,
                                                      uint16_t* __restrict__ out) {
  pdl_wait_and_trigger();
  const int vec = d / 8;
  const int64_t n = (int64_t)T * vec;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / vec;
    const int c = (int)(i % vec);
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.f;
    for (int j = 0; j < k; ++j) {
      const float4* src = reinterpret_cast<const float4*>(yw + ((size_t)t * k + j) * d) + 2 * c;
      const float4 a = __ldg(src), b = __ldg(src + 1);
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    if (resid) {  // residual add (fp32), before the single rounding to bf16
      const uint4 r = __ldg(reinterpret_cast<const uint4*>(resid + (size_t)t * d) + c);
      const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[2 * u] += __uint_as_float(rw[u] << 16);
        acc[2 * u + 1] += __uint_as_float(rw[u] & 0xFFFF0000u);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * u], acc[2 * u + 1]);
      o[u] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(out + (size_t)t * d)[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ----------------------------------------------------- pre-MoE RMSNorm ----
// x = bf16((h / sqrt(mean(h^2) + eps)) * g), one warp per row: lane l sums the
// squares of elements 4l + 128i .. +3 in increasing i (fp32 fma), a butterfly
// adds the 32 partial sums, then every element is divided by the root and
// multiplied by its gain, rounded once.
// Field guide "gpt-oss 20B", "04 One decoder block" (RMSNorm before the MoE).
__global__ void __launch_bounds__(256) rms_norm_kernel(const uint16_t* __restrict__ h,
                                                       const float* __restrict__ g, float eps,
                                                       int T, int d, uint16_t* __restrict__ x) {
  pdl_wait_and_trigger();
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
    const uint16_t* hr = h + (size_t)t * d;
    float ss = 0.f;
    for (int k = lane * 4; k < d; k += 128) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(hr + k));
      const float a = __uint_as_float(v.x << 16), b = __uint_as_float(v.x & 0xFFFF0000u);
      const float c = __uint_as_float(v.y << 16), e = __uint_as_float(v.y & 0xFFFF0000u);
      ss = fmaf(a, a, ss);
      ss = fmaf(b, b, ss);
      ss = fmaf(c, c, ss);
      ss = fmaf(e, e, ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
    const float root = sqrtf(ss / (float)d + eps);
    uint16_t* xr = x + (size_t)t * d;
    for (int k = lane * 4; k < d; k += 128) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(hr + k));
      const float4 gv = __ldg(reinterpret_cast<const float4*>(g + k));
      const __nv_bfloat162 lo = __floats2bfloat162_rn((__uint_as_float(v.x << 16) / root) * gv.x,
                                                      (__uint_as_float(v.x & 0xFFFF0000u) / root) * gv.y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn((__uint_as_float(v.y << 16) / root) * gv.z,
                                                      (__uint_as_float(v.y & 0xFFFF0000u) / root) * gv.w);
      reinterpret_cast<uint2*>(xr + k)[0] =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
  }
}

// ------------------------------------------------------- MXFP4 decode ----
__global__ void __launch_bounds__(256) mxfp4_to_bf16_kernel(const uint8_t* __restrict__ codes,
                                                            const uint8_t* __restrict__ scales,
                                                            int rows, int K,
                                                            uint16_t* __restrict__ out) {
  pdl_wait_and_trigger();
  const int groups = K / 32;
  const int64_t n = (int64_t)rows * groups;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n;
       g += (int64_t)gridDim.x * blockDim.x) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(codes) + g);
    uint4 o[4];
    mxfp4x32_to_bf16(q, scales[g], o);
    uint4* dst = reinterpret_cast<uint4*>(out) + g * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = chunk8_from_perm(o[i]);
  }
}

// -------------------------------------------------- scale transpose ----
// [E][N][G] -> [E][G][N]. A block takes 64 consecutive rows n (64*G
// contiguous bytes), stages them in shared memory and writes, for every group
// g, the 64 bytes out[g][n0 .. n0+63] as four 16-byte stores. N is a multiple
// of 32, so full 64-row blocks store whole vectors; the last block of an
// expert may hold 32 rows.
constexpr int TR_ROWS = 64;

__global__ void __launch_bounds__(256) transpose_scales_kernel(const uint8_t* __restrict__ in,
                                                               int N, int G,
                                                               const int32_t* __restrict__ counts,
                                                               uint8_t* __restrict__ out) {
  pdl_wait_and_trigger();
  extern __shared__ __align__(16) uint8_t tsm[];  // [TR_ROWS][G]
  const int e = blockIdx.y;
  if (counts && counts[e] == 0) return;  // no GEMM tile reads this expert's scales
  const int n0 = blockIdx.x * TR_ROWS;
  const int rows = min(TR_ROWS, N - n0);
  const uint8_t* src = in + ((size_t)e * N + n0) * G;
  const int bytes = rows * G;
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (bytes & 15) == 0) {
    for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(tsm)[i] = __ldg(reinterpret_cast<const uint4*>(src) + i);
  } else {
    for (int i = threadIdx.x; i < bytes; i += blockDim.x) tsm[i] = src[i];
  }
  __syncthreads();
  uint8_t* dst = out + (size_t)e * N * G + n0;
  const int vecs = rows / 16;
  for (int i = threadIdx.x; i < G * vecs; i += blockDim.x) {
    const int g = i / vecs, v = i % vecs;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = v * 16 + q * 4;
      w[q] = (uint32_t)tsm[(r + 0) * G + g] | ((uint32_t)tsm[(r + 1) * G + g] << 8) |
             ((uint32_t)tsm[(r + 2) * G + g] << 16) | ((uint32_t)tsm[(r + 3) * G + g] << 24);
    }
    *reinterpret_cast<uint4*>(dst + (size_t)g * N + v * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// --------------------------------------------------- timeout self-test ----
// A bounded wait on a barrier whose phase never completes; the wait gives up
// after kWaitLimitNs and records MOE_ERR_TIMEOUT in *status.
__global__ void wait_timeout_selftest_kernel(int* status) {
  pdl_wait_and_trigger();
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, status);
}

int grid_for(int64_t n, int per_block, int cap) {
  int64_t b = (n + per_block - 1) / per_block;
  if (b < 1) b = 1;
  if (b > cap) b = cap;
  return (int)b;
}

}  // namespace

bool& pdl_launches() {
  static thread_local bool on = false;
  return on;
}

cudaError_t launch_perm_small(const int32_t* topk_idx, int T, int k, int E, int32_t* counts,
                              int32_t* offsets, int32_t* mtile_prefix, int32_t* perm,
                              cudaStream_t st) {
  if (T < 1 || T > kPermChunk) return cudaErrorInvalidValue;
  launch_kernel(perm_small_kernel, dim3(1), dim3(256), 0, st, topk_idx, T, k, E, counts, offsets, mtile_prefix, perm);
  return cudaGetLastError();
}

cudaError_t launch_perm_hist(const int32_t* topk_idx, int T, int k, int E, int32_t* chunk_hist,
                             cudaStream_t st) {
  launch_kernel(perm_hist_kernel, dim3(perm_chunks(T)), dim3(256), 0, st, topk_idx, T, k, E, chunk_hist);
  return cudaGetLastError();
}

cudaError_t launch_perm_scan(const int32_t* chunk_hist, int nchunks, int E, int32_t* counts,
                             int32_t* offsets, int32_t* chunk_base, int32_t* mtile_prefix,
                             cudaStream_t st) {
  launch_kernel(perm_scan_kernel, dim3(1), dim3(256), 0, st, chunk_hist, nchunks, E, counts, offsets, chunk_base,
                                      mtile_prefix);
  return cudaGetLastError();
}

cudaError_t launch_perm_scatter(const int32_t* topk_idx, int T, int k, int E,
                                const int32_t* chunk_base, int32_t* perm, int32_t* inv,
                                cudaStream_t st) {
  launch_kernel(perm_scatter_kernel, dim3(perm_chunks(T)), dim3(256), 0, st, topk_idx, T, k, E, chunk_base, perm, inv);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* perm, int P, int k, int d,
                               uint16_t* xp, cudaStream_t st) {
  launch_kernel(gather_rows_kernel, dim3(grid_for(P, 8, 148 * 16)), dim3(256), 0, st, x, perm, P, k, d,
                xp);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* yw, int T, int k, int d, const uint16_t* resid,
                           uint16_t* out, cudaStream_t st) {
  const int64_t n = (int64_t)T * (d / 8);
  launch_kernel(combine_kernel, dim3(grid_for(n, 256, 148 * 16)), dim3(256), 0, st, yw, T, k, d, resid,
                out);
  return cudaGetLastError();
}

cudaError_t launch_rms_norm(const uint16_t* h, const float* g, float eps, int T, int d,
                            uint16_t* x, cudaStream_t st) {
  launch_kernel(rms_norm_kernel, dim3(grid_for(T, 8, 148 * 8)), dim3(256), 0, st, h, g, eps, T, d, x);
  return cudaGetLastError();
}

cudaError_t launch_transpose_scales(const uint8_t* in, int E, int N, int G, const int32_t* counts,
                                    uint8_t* out, cudaStream_t st) {
  const int smem = TR_ROWS * G;  // G <= 512 (K <= 16384): at most 32 KB
  dim3 grid((N + TR_ROWS - 1) / TR_ROWS, E);
  launch_kernel(transpose_scales_kernel, dim3(grid), dim3(256), smem, st, in, N, G, counts, out);
  return cudaGetLastError();
}

cudaError_t launch_mxfp4_to_bf16(const uint8_t* codes, const uint8_t* scales, int rows, int K,
                                 uint16_t* out, cudaStream_t st) {
  const int64_t n = (int64_t)rows * (K / 32);
  launch_kernel(mxfp4_to_bf16_kernel, dim3(grid_for(n, 256, 148 * 16)), dim3(256), 0, st, codes, scales,
                rows, K, out);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(int* status, cudaStream_t st) {
  launch_kernel(wait_timeout_selftest_kernel, dim3(1), dim3(32), 0, st, status);
  return cudaGetLastError();
}

}  // namespace moe
