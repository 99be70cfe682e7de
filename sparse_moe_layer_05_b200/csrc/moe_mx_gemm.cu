// moe_mx_gemm.cu -- expert-grouped MXFP4 GEMMs on the block-scaled tensor-core
// path (tcgen05.mma .kind::mxf8f6f4): the E2M1 weight codes go from HBM to
// shared memory by TMA (which widens them to 8-bit containers) and the E8M0
// weight scales are applied by the tensor core, so no CUDA core decodes a
// weight.
//
//   gate/up:  H[r, j] = silu(x_r . Wgate[e][j] + bg[e][j]) * (x_r . Wup[e][j] + bu[e][j])
//   down:     Yw[pair(r), m] = p(pair(r)) * (H[r] . Wdown[e][m] + bd[e][m])
// (the biases are optional; without them those terms are zero).
//
// Field guide "gpt-oss 20B", "03 Sparse Mixture of Experts" (SwiGLU experts,
// weighted sum); "gpt-oss-20b and gpt-oss-120b", "Four-bit expert weights"
// (E2M1 codes, one power-of-two scale per 32 weights).
//
// Activations. The tensor core's block-scaled kinds take no bf16 operand, so
// each bf16 activation row is split, per group of 32 along K, into two E4M3
// terms with E8M0 scales: hi = e4m3(x / 2^Eh) and lo = e4m3((x / 2^Eh - hi) *
// 2^4), Eh = floor(log2 max|x|) - 7, scale bytes Eh + 127 and Eh + 123. For
// every element with |x| >= 2^-13 max|x| of its group the split is exact
// (x = 2^Eh hi + 2^(Eh-4) lo: x has 8 significant bits, hi keeps 4, the
// remainder fits lo's 4 bits, |x/2^Eh - hi| <= 8); smaller elements keep an
// error below 2^-21 max|x|. (Both hold for groups with max|x| >= 2^-116,
// where Eh needs no clamping.) hi and lo enter one UMMA as separate columns of B
// (tokens 0..NT-1 hi, NT..2NT-1 lo) and the epilogue adds the two results.
//
// Tiles. 128 weight rows (UMMA M) x NT tokens (UMMA N = 2 NT), 128 K per
// shared-memory stage. Token rows live in a per-expert padded layout (each
// expert's segment rounded up to a multiple of NT rows), so a token tile is
// NT consecutive rows and its B scales one contiguous block.
//
// Issue rate. With few tokens per expert each UMMA is short, and one thread
// issuing the UMMAs, scale copies and commits of a k-block bounds the rate
// (the issue latency of these tcgen05 operations, not the tensor pipe, is the
// limit; it scales with the number of issuing threads per SM). So two CTAs
// share an SM and each has two issuing threads: the CTA's k-blocks, numbered
// q = 0, 1, 2, ... across its tiles, go to issuer q % 2, each accumulating
// into its own TMEM buffer; the epilogue adds the two in a fixed order. With
// an even number of stages, stage q % STAGES is always served by the same
// issuer, so every waiter of a stage's barrier waits for its phases in
// order (a parity wait cannot tell phase k done from phase k-1 pending).
//
// Warp roles (256 threads per CTA):
//   warp 0      TMA producer, three copies per k-block: the weight codes
//               (E2M1 -> 8-bit containers, one box), the hi and lo token rows
//               (one box over both), the B scale block
//   warp 1      TMEM allocator and UMMA issuer 0 (even q)
//   warp 3      UMMA issuer 1 (odd q)
//   warp 2      A-scale builder: turns the tile's E8M0 weight scales (one
//               bulk copy per tile into shared memory, double-buffered) into
//               the per-k-block layout tcgen05.cp reads
//   warps 4..    epilogue, in groups of four (TMEM lane quarters 0..3)
//
// K tail. The 4-bit tensor maps need row lengths in multiples of 128, so a K
// that is 64 mod 128 is covered by the (K/128) full k-blocks of a main map and
// one last k-block [K-128, K) from a second map based (K-128)/2 bytes into each
// row; of that block only the K steps past the last full k-block are issued.
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {
namespace {

constexpr int kMaxE = 256;

// --------------------------------------------------- hi/lo E4M3 split ----

// Groups of 32 along K: G = K/32 groups, KB = ceil(K/128) k-blocks; the last
// k-block of a K that is not a multiple of 128 covers [K-128, K).
__host__ __device__ __forceinline__ void group_to_kblock(int g, int G, int KB, int& kb, int& kk) {
  const bool tail = (G % 4) != 0;
  if (!tail || g < 4 * (KB - 1)) {
    kb = g >> 2;
    kk = g & 3;
  } else {
    kb = KB - 1;
    kk = g - (G - 4);
  }
}

// Byte offset of the B scale of token n (0..NT-1), term h (0 hi, 1 lo), K
// step kk inside the block of one (token tile, k-block). B column c = h*NT + n
// of the UMMA takes its scale from TMEM lane c%32 of column c/32: word w =
// c/32 of lane c%32, four words (16 bytes) per lane in a 512-byte tcgen05.cp
// atom.
__device__ __forceinline__ int sfb_offset(int NT, int n, int h, int kk) {
  const int c = h * NT + n;
  const int w = c >> 5;
  return (w >> 2) * 512 + (c & 31) * 16 + (w & 3) * 4 + kk;
}

// Bytes of one B-scale block: one 512-byte tcgen05.cp atom per 128 UMMA B
// columns (terms x NT: hi and lo columns of the bf16 split, one set otherwise).
__host__ __device__ constexpr int sfb_block_bytes(int NT, int terms = 2) {
  return 512 * ((terms * NT + 127) / 128);
}

// Splits 32 fp32 values (already bf16-exact) into hi / lo E4M3 bytes given the
// group's max |v|; returns the hi scale byte (lo's is 4 less).
__device__ __forceinline__ uint32_t split_group32(const float (&v)[32], float amax,
                                                  uint32_t (&hi)[8], uint32_t (&lo)[8]) {
  int eh;
  if (amax == 0.f) {
    eh = 0;
  } else {
    // floor(log2 amax) from the exponent field, minus 7 so that max|v|/2^eh
    // lies in [128, 256); eh >= -123 keeps the lo scale byte (eh + 123) >= 0
    // (groups with max|v| below 2^-116 lose the exactness bound below).
    const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127;
    eh = max(e - 7, -123);
  }
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - eh) << 23);   // 2^-eh
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t hw = 0, lw = 0;
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float a = v[4 * q + u] * inv, b = v[4 * q + u + 1] * inv;
      const uint32_t h2 = f32x2_to_e4m3x2(a, b);
      const float2 hb = e4m3x2_to_f32x2(h2);
      const uint32_t l2 = f32x2_to_e4m3x2((a - hb.x) * 16.f, (b - hb.y) * 16.f);
      hw |= h2 << (8 * u);
      lw |= l2 << (8 * u);
    }
    hi[q] = hw;
    lo[q] = lw;
  }
  return static_cast<uint32_t>(eh + 127);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// ------------------------------------------- MX conversion (w4a8, w4a4) ----
// The OCP Microscaling conversion of one group of 32 values: shared scale
// X = 2^(floor(log2 max|v|) - emax), emax 8 for E4M3 and 2 for E2M1;
// elements v / X rounded to the nearest element value (ties to even),
// magnitudes above the largest normal (448, 6) clamped to it. X's exponent is
// kept in the E8M0 range (at least -127: groups whose max|v| is below
// 2^(emax - 127) keep that smallest scale); an all-zero group takes X = 1.
template <int ACT>
__device__ __forceinline__ int mx_scale_exp(float amax) {
  constexpr int emax = ACT == ACT_E2M1 ? 2 : 8;
  if (!(amax > 0.f)) return 0;
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127;  // floor(log2)
  return max(e - emax, -127);
}

// 32 values -> element codes: E4M3 bytes in w[0..7] (element i in byte i),
// or E2M1 codes packed two per byte in w[0..3] (element 2i in the low nibble
// of byte i). Returns the E8M0 scale byte.
template <int ACT>
__device__ __forceinline__ uint32_t mx_quant_group32(const float (&v)[32], float amax,
                                                     uint32_t (&w)[8]) {
  const int x = mx_scale_exp<ACT>(amax);
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - x) << 23);   // 2^-x
  if (ACT == ACT_E4M3) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      w[q] = f32x2_to_e4m3x2(v[4 * q] * inv, v[4 * q + 1] * inv) |
             (f32x2_to_e4m3x2(v[4 * q + 2] * inv, v[4 * q + 3] * inv) << 16);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t a = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        a |= f32x2_to_e2m1x2(v[8 * q + 2 * b] * inv, v[8 * q + 2 * b + 1] * inv) << (8 * b);
      w[q] = a;
    }
#pragma unroll
    for (int q = 4; q < 8; ++q) w[q] = 0;
  }
  return static_cast<uint32_t>(x + 127);
}

// 32 bf16 values at src (16-byte aligned) -> fp32 and their max |v|.
__device__ __forceinline__ float load_group32(const uint16_t* src16, float (&v)[32]) {
  const uint4* src = reinterpret_cast<const uint4*>(src16);
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 w = __ldg(src + c);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      v[8 * c + 2 * u] = bf16_bits_to_f32(ww[u] & 0xFFFFu);
      v[8 * c + 2 * u + 1] = bf16_bits_to_f32(ww[u] >> 16);
      amax = fmaxf(amax, fmaxf(fabsf(v[8 * c + 2 * u]), fabsf(v[8 * c + 2 * u + 1])));
    }
  }
  return amax;
}

// Stores one converted group: 32 bytes (E4M3) or 16 bytes (E2M1) at dst.
template <int ACT>
__device__ __forceinline__ void store_group32(uint8_t* dst, const uint32_t (&w)[8]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(w[0], w[1], w[2], w[3]);
  if (ACT == ACT_E4M3) d[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// One thread per (permuted row, group of 32): gathers x[token] into the padded
// token layout as hi / lo E4M3 rows and writes the B scale blocks.
template <int NT>
__global__ void __launch_bounds__(256) mx_quant_gather_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
    const int32_t* __restrict__ offsets, int E, int P, int k, int K, uint8_t* __restrict__ qhi,
    uint8_t* __restrict__ qlo, uint8_t* __restrict__ sfb) {
  pdl_wait_and_trigger();
  __shared__ int s_off[kMaxE + 1], s_tb[kMaxE + 1];
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0;
    for (int e = 0; e < E; ++e) {
      s_tb[e] = a;
      a += (s_off[e + 1] - s_off[e] + NT - 1) / NT;
    }
    s_tb[E] = a;
  }
  __syncthreads();
  const int G = K / 32, KB = (K + 127) / 128;
  constexpr int SFB = sfb_block_bytes(NT);
  const int64_t n = static_cast<int64_t>(P) * G;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / G), g = static_cast<int>(i % G);
    int lo_e = 0, hi_e = E;   // largest e with s_off[e] <= p
    while (hi_e - lo_e > 1) {
      const int mid = (lo_e + hi_e) >> 1;
      if (s_off[mid] <= p) lo_e = mid; else hi_e = mid;
    }
    const int e = lo_e;
    const int pr = s_tb[e] * NT + (p - s_off[e]);
    const int t = perm[p] / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * K + 32 * g);
    float v[32];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 w = __ldg(src + c);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[8 * c + 2 * u] = bf16_bits_to_f32(ww[u] & 0xFFFFu);
        v[8 * c + 2 * u + 1] = bf16_bits_to_f32(ww[u] >> 16);
        amax = fmaxf(amax, fmaxf(fabsf(v[8 * c + 2 * u]), fabsf(v[8 * c + 2 * u + 1])));
      }
    }
    uint32_t hw[8], lw[8];
    const uint32_t sh = split_group32(v, amax, hw, lw);
    uint4* dh = reinterpret_cast<uint4*>(qhi + static_cast<size_t>(pr) * K + 32 * g);
    uint4* dl = reinterpret_cast<uint4*>(qlo + static_cast<size_t>(pr) * K + 32 * g);
    dh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    dh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    dl[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    dl[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    int kb, kk;
    group_to_kblock(g, G, KB, kb, kk);
    uint8_t* blk = sfb + (static_cast<size_t>(pr / NT) * KB + kb) * SFB;
    blk[sfb_offset(NT, pr % NT, 0, kk)] = static_cast<uint8_t>(sh);
    blk[sfb_offset(NT, pr % NT, 1, kk)] = static_cast<uint8_t>(sh - 4);
  }
}

// The same rows, token-major: one thread per (token, group of 32) converts
// the group once and writes it to each of the token's k permuted rows (inv:
// pair id t*k + j -> permuted row), so the conversion work does not grow
// with k. Results identical to mx_quant_gather_kernel.
template <int NT>
__global__ void __launch_bounds__(256) mx_quant_gather_tok_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ inv, const int32_t* __restrict__ offsets, int E, int T, int k,
    int K, uint8_t* __restrict__ qhi, uint8_t* __restrict__ qlo, uint8_t* __restrict__ sfb) {
  pdl_wait_and_trigger();
  __shared__ int s_off[kMaxE + 1], s_tb[kMaxE + 1];
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0;
    for (int e = 0; e < E; ++e) {
      s_tb[e] = a;
      a += (s_off[e + 1] - s_off[e] + NT - 1) / NT;
    }
    s_tb[E] = a;
  }
  __syncthreads();
  const int G = K / 32, KB = (K + 127) / 128;
  constexpr int SFB = sfb_block_bytes(NT);
  const int64_t n = static_cast<int64_t>(T) * G;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / G), g = static_cast<int>(i % G);
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * K + 32 * g);
    float v[32];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 w = __ldg(src + c);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[8 * c + 2 * u] = bf16_bits_to_f32(ww[u] & 0xFFFFu);
        v[8 * c + 2 * u + 1] = bf16_bits_to_f32(ww[u] >> 16);
        amax = fmaxf(amax, fmaxf(fabsf(v[8 * c + 2 * u]), fabsf(v[8 * c + 2 * u + 1])));
      }
    }
    uint32_t hw[8], lw[8];
    const uint32_t sh = split_group32(v, amax, hw, lw);
    const uint4 h0 = make_uint4(hw[0], hw[1], hw[2], hw[3]), h1 = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    const uint4 l0 = make_uint4(lw[0], lw[1], lw[2], lw[3]), l1 = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    int kb, kk;
    group_to_kblock(g, G, KB, kb, kk);
    for (int j = 0; j < k; ++j) {
      const int q = t * k + j;
      const int e = __ldg(topk_idx + q);
      const int pr = s_tb[e] * NT + (__ldg(inv + q) - s_off[e]);
      uint4* dh = reinterpret_cast<uint4*>(qhi + static_cast<size_t>(pr) * K + 32 * g);
      uint4* dl = reinterpret_cast<uint4*>(qlo + static_cast<size_t>(pr) * K + 32 * g);
      dh[0] = h0;
      dh[1] = h1;
      dl[0] = l0;
      dl[1] = l1;
      uint8_t* blk = sfb + (static_cast<size_t>(pr / NT) * KB + kb) * SFB;
      blk[sfb_offset(NT, pr % NT, 0, kk)] = static_cast<uint8_t>(sh);
      blk[sfb_offset(NT, pr % NT, 1, kk)] = static_cast<uint8_t>(sh - 4);
    }
  }
}

// Plain row split (no gather): rows [R][K] bf16 -> hi, lo [R][K] E4M3 and
// scales [R][K/32][2] (hi byte, lo byte).
__global__ void __launch_bounds__(256) mx_split_rows_kernel(const uint16_t* __restrict__ x, int R,
                                                            int K, uint8_t* __restrict__ qhi,
                                                            uint8_t* __restrict__ qlo,
                                                            uint8_t* __restrict__ scales) {
  pdl_wait_and_trigger();
  const int G = K / 32;
  const int64_t n = static_cast<int64_t>(R) * G;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / G;
    const int g = static_cast<int>(i % G);
    const uint4* src = reinterpret_cast<const uint4*>(x + r * K + 32 * g);
    float v[32];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 w = __ldg(src + c);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[8 * c + 2 * u] = bf16_bits_to_f32(ww[u] & 0xFFFFu);
        v[8 * c + 2 * u + 1] = bf16_bits_to_f32(ww[u] >> 16);
        amax = fmaxf(amax, fmaxf(fabsf(v[8 * c + 2 * u]), fabsf(v[8 * c + 2 * u + 1])));
      }
    }
    uint32_t hw[8], lw[8];
    const uint32_t sh = split_group32(v, amax, hw, lw);
    uint4* dh = reinterpret_cast<uint4*>(qhi + r * K + 32 * g);
    uint4* dl = reinterpret_cast<uint4*>(qlo + r * K + 32 * g);
    dh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    dh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    dl[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    dl[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    scales[(r * G + g) * 2] = static_cast<uint8_t>(sh);
    scales[(r * G + g) * 2 + 1] = static_cast<uint8_t>(sh - 4);
  }
}

// One thread per (permuted row, group of 32) for the quantised activation
// modes: x[token] -> one MX-converted row in the padded token layout (K bytes,
// or K/2 for E2M1) and its scale byte in the B-scale blocks.
// KB256: the scale blocks of the kind::mxf4 kernel, per 256-wide k-block:
// 1024 bytes per (token tile, k-block), group byte b (0..7) of token n at
// (b / 4) * 512 + the 32x128b atom byte of (n, b % 4).
template <int NT, int ACT, bool KB256 = false>
__global__ void __launch_bounds__(256) mx_act_quant_gather_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
    const int32_t* __restrict__ offsets, int E, int P, int k, int K, uint8_t* __restrict__ q,
    uint8_t* __restrict__ sfb) {
  pdl_wait_and_trigger();
  __shared__ int s_off[kMaxE + 1], s_tb[kMaxE + 1];
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0;
    for (int e = 0; e < E; ++e) {
      s_tb[e] = a;
      a += (s_off[e + 1] - s_off[e] + NT - 1) / NT;
    }
    s_tb[E] = a;
  }
  __syncthreads();
  const int G = K / 32, KB = KB256 ? (K + 255) / 256 : (K + 127) / 128;
  constexpr int SFB = KB256 ? 1024 : sfb_block_bytes(NT, 1);
  constexpr int GB = ACT == ACT_E2M1 ? 16 : 32;     // bytes of one converted group
  const size_t row_bytes = static_cast<size_t>(G) * GB;
  const int64_t n = static_cast<int64_t>(P) * G;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / G), g = static_cast<int>(i % G);
    int lo_e = 0, hi_e = E;   // largest e with s_off[e] <= p
    while (hi_e - lo_e > 1) {
      const int mid = (lo_e + hi_e) >> 1;
      if (s_off[mid] <= p) lo_e = mid; else hi_e = mid;
    }
    const int e = lo_e;
    const int pr = s_tb[e] * NT + (p - s_off[e]);
    const int t = perm[p] / k;
    float v[32];
    const float amax = load_group32(x + static_cast<size_t>(t) * K + 32 * g, v);
    uint32_t w[8];
    const uint32_t sx = mx_quant_group32<ACT>(v, amax, w);
    store_group32<ACT>(q + static_cast<size_t>(pr) * row_bytes + static_cast<size_t>(g) * GB, w);
    if (KB256) {
      // 8 groups per k-block; the last k-block of a K that is not a multiple
      // of 256 covers [K-256, K)
      int kb, b;
      if ((G % 8) == 0 || g < 8 * (KB - 1)) {
        kb = g >> 3;
        b = g & 7;
      } else {
        kb = KB - 1;
        b = g - (G - 8);
      }
      uint8_t* blk = sfb + (static_cast<size_t>(pr / NT) * KB + kb) * SFB;
      blk[(b >> 2) * 512 + sfb_offset(NT, pr % NT, 0, b & 3)] = static_cast<uint8_t>(sx);
    } else {
      int kb, kk;
      group_to_kblock(g, G, KB, kb, kk);
      uint8_t* blk = sfb + (static_cast<size_t>(pr / NT) * KB + kb) * SFB;
      blk[sfb_offset(NT, pr % NT, 0, kk)] = static_cast<uint8_t>(sx);
    }
  }
}

// The MX conversion on plain rows: [R][K] bf16 -> q rows and scales [R][K/32].
template <int ACT>
__global__ void __launch_bounds__(256) mx_act_quant_rows_kernel(const uint16_t* __restrict__ x,
                                                                int R, int K,
                                                                uint8_t* __restrict__ q,
                                                                uint8_t* __restrict__ scales) {
  pdl_wait_and_trigger();
  const int G = K / 32;
  constexpr int GB = ACT == ACT_E2M1 ? 16 : 32;
  const int64_t n = static_cast<int64_t>(R) * G;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v[32];
    const float amax = load_group32(x + i * 32, v);
    uint32_t w[8];
    scales[i] = static_cast<uint8_t>(mx_quant_group32<ACT>(v, amax, w));
    store_group32<ACT>(q + i * GB, w);
  }
}

// ------------------------------------------------------------ the GEMM ----

enum Epi { EPI_SWIGLU = 0, EPI_DOWN = 1 };

// NT tokens per tile, ISSUERS UMMA-issuing threads per CTA, CTAS CTAs per SM,
// EPI_WARPS epilogue warps (groups of four, one per TMEM lane quarter; group
// g takes every (EPI_WARPS/4)-th chunk of token columns).
template <int NT_, int ISSUERS_, int CTAS_, int EPI_WARPS_, int ACT_ = ACT_HILO>
struct MxCfg {
  static constexpr int NT = NT_;
  static constexpr int ISSUERS = ISSUERS_;
  static constexpr int CTAS = CTAS_;
  static constexpr int EPI_WARPS = EPI_WARPS_;
  static constexpr int EPI_GROUPS = EPI_WARPS / 4;
  static constexpr int ACT = ACT_;                  // activation operand (ACT_*)
  static constexpr int TERMS = ACT == ACT_HILO ? 2 : 1;
  static constexpr int MW = 128;                    // weight rows per tile
  static constexpr int N = TERMS * NT;              // UMMA N: (hi and lo) token columns
  static constexpr int A_BYTES = 128 * 128;         // E2M1 in 8-bit containers
  static constexpr int A_TX = 128 * 64;             // packed bytes the TMA counts
  static constexpr int B_BYTES = N * 128;           // 8-bit elements (E2M1 widened by TMA)
  static constexpr int B_TX = ACT == ACT_E2M1 ? N * 64 : B_BYTES;
  static constexpr uint32_t BTYPE = ACT == ACT_E2M1 ? 5u : 0u;   // instruction B type
  static constexpr int SFB_BYTES = sfb_block_bytes(NT, TERMS);
  static constexpr int OFF_B = A_BYTES;
  static constexpr int OFF_SFA = OFF_B + B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + 512;
  static constexpr int STAGE_BYTES = ((OFF_SFB + SFB_BYTES) + 1023) / 1024 * 1024;
  // even, so that with two issuers stage s is always consumed by issuer s % 2
  static constexpr int STAGES = 4;
  static constexpr int OFF_TS = STAGES * STAGE_BYTES;   // two tile-scale buffers
  static constexpr int TS_BYTES = 128 * (kMxMaxK / 32);
  static constexpr int OFF_BAR = OFF_TS + 2 * TS_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 8;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TAB = OFF_MISC + 16;
  static constexpr int OFF_XCH = OFF_TAB + 3 * (kMaxE + 1) * 4;
  static constexpr int CH = 8;                      // epilogue token chunk (TMEM columns)
  static constexpr int SMEM_BYTES = OFF_XCH + EPI_GROUPS * 2 * 4 * CH * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr int NUM_THREADS = 128 + 32 * EPI_WARPS;
  static constexpr int TMEM_COLS = CTAS == 2 ? 256 : 512;
  // accumulators: issuer u, tile buffer b at column (2u + b) N; then each
  // issuer's scale columns (A: 4, B: 4 per 512-byte atom)
  static constexpr int SF_COL0 = 2 * ISSUERS * N;
  static constexpr int SF_COLS = 4 + 4 * (SFB_BYTES / 512);
  static constexpr int TX_BYTES = A_TX + B_TX + SFB_BYTES;
  static_assert(NT % CH == 0 && N <= 256 && N % 16 == 0, "tile width");
  static_assert(EPI_WARPS % 4 == 0 && EPI_GROUPS <= 4, "epilogue warps");
  static_assert(SF_COL0 + ISSUERS * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(CTAS * (SMEM_ALLOC + 1024) <= 233472 && SMEM_ALLOC <= 232448, "shared memory");
  static_assert(OFF_B % 1024 == 0 && (NT * 128) % 1024 == 0, "swizzle atom alignment");
};

// Decode: 16-token tiles, two issuers, two CTAs per SM. Prefill: 120-token
// tiles (UMMA N = 240, long enough per instruction for one issuer to keep the
// tensor pipe busy), one CTA per SM, and 12 epilogue warps so that draining a
// tile's 15 column chunks keeps pace with its UMMAs.
using MxSmall = MxCfg<16, 2, 2, 4>;
using MxLarge = MxCfg<120, 1, 1, 12>;
// The quantised activation modes: one term, so 128-token tiles fill UMMA N =
// 128 in the large variant (N must be a multiple of 16: 120 is not).
template <int ACT> using MxSmallQ = MxCfg<16, 2, 2, 4, ACT>;
template <int ACT> using MxLargeQ = MxCfg<128, 1, 1, 12, ACT>;
// the largest token tile of any variant (the padded token layout's granule)
constexpr int kMxMaxNT = 128;

struct MxArgs {
  const int32_t* offsets;
  int E, K, I;              // K: contraction length; I: intermediate size (SwiGLU tiles)
  int n_wb;                 // weight blocks per expert
  int rows_per_expert;      // weight rows of one expert in the scale array
  const uint8_t* scales;    // [E][rows_per_expert][K/32] E8M0
  const uint8_t* sfb;       // B scale blocks [token tile][KB][SFB_BYTES]
  // SwiGLU: quantized H for the down GEMM
  uint8_t* h_hi;
  uint8_t* h_lo;
  uint8_t* h_sfb;
  int h_kb;                 // k-blocks of the down GEMM (ceil(I/128))
  // down: weighted rows
  float* out_f32;
  int n_out;
  const int32_t* perm;
  const float* topk_w;
  int* status;
  const float* bias;        // [E][2I] (SwiGLU) or [E][d] (down), or nullptr
};

__device__ __forceinline__ float silu_mx(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int EPI, class C>
__global__ void __launch_bounds__(C::NUM_THREADS, C::CTAS)
    grouped_mx_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmAt,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmBt, const MxArgs args) {
  pdl_wait_and_trigger();
  constexpr int NT = C::NT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto bar_accFull = [&](int b) { return bar0 + 8u * (2 * C::STAGES + b); };
  auto bar_accEmpty = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 2 + b); };
  auto bar_tsFull = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 4 + b); };
  auto bar_tsEmpty = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 6 + b); };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* s_off = reinterpret_cast<int*>(smem + C::OFF_TAB);
  int* s_tp = s_off + (kMaxE + 1);   // prefix of tiles per expert
  int* s_tb = s_tp + (kMaxE + 1);    // prefix of token tiles per expert
  float* s_xch = reinterpret_cast<float*>(smem + C::OFF_XCH);

  const int E = args.E;
  for (int i = threadIdx.x; i <= E; i += C::NUM_THREADS) s_off[i] = args.offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    int acc = 0, tb = 0;
    for (int e = 0; e < E; ++e) {
      s_tp[e] = acc;
      s_tb[e] = tb;
      const int ntb = (s_off[e + 1] - s_off[e] + NT - 1) / NT;
      acc += ntb * args.n_wb;
      tb += ntb;
    }
    s_tp[E] = acc;
    s_tb[E] = tb;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_full(s), 2);    // producer (with the TMA bytes) + A-scale builder
      mbar_init(bar_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accFull(b), C::ISSUERS);     // one commit per issuer
      mbar_init(bar_accEmpty(b), C::EPI_WARPS * 32);
      mbar_init(bar_tsFull(b), 1);
      mbar_init(bar_tsEmpty(b), 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmAt);
    tma_prefetch_desc(&tmB);
    if (C::ACT == ACT_E2M1) tma_prefetch_desc(&tmBt);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];

  const int total = s_tp[E];
  const int K = args.K;
  const int G = K / 32;
  const int KB = (K + 127) / 128;
  const bool tail = (K % 128) != 0;         // K % 64 == 0: the tail k-block has 2 K steps
  // tile -> (expert, weight block, token block), weight-block major inside an
  // expert so that neighbouring CTAs stream neighbouring weights
  auto decode = [&](int tile, int& e, int& wb, int& tb, int& rows) {
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
    tb = local % ntb;
    rows = min(NT, cnt - tb * NT);
  };

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0) {
      // The tile's weight scales (rows of G bytes, contiguous per block) go to
      // tile-scale buffer it&1; the next tile's are requested a few k-blocks
      // into the current tile, once the builder has released that buffer.
      auto load_tile_scales = [&](int tile, int itx) -> bool {
        int e, wb, tb, rows;
        decode(tile, e, wb, tb, rows);
        const int b = itx & 1;
        if (!mbar_wait(bar_tsEmpty(b), ((itx >> 1) & 1) ^ 1, abort_flag, args.status)) return false;
        const uint32_t ts = sbase + C::OFF_TS + b * C::TS_BYTES;
        if (EPI == EPI_SWIGLU) {
          const uint32_t half = 64u * G;
          mbar_expect_tx(bar_tsFull(b), 2 * half);
          bulk_load(ts, args.scales + (static_cast<size_t>(e) * 2 * args.I + wb * 64) * G, half,
                    bar_tsFull(b));
          bulk_load(ts + half,
                    args.scales + (static_cast<size_t>(e) * 2 * args.I + args.I + wb * 64) * G,
                    half, bar_tsFull(b));
        } else {
          const uint32_t bytes =
              static_cast<uint32_t>(min(128, args.rows_per_expert - wb * 128)) * G;
          mbar_expect_tx(bar_tsFull(b), bytes);
          bulk_load(ts, args.scales + (static_cast<size_t>(e) * args.rows_per_expert + wb * 128) * G,
                    bytes, bar_tsFull(b));
        }
        return true;
      };
      int s = 0, ph = 0, it = 0;
      bool ok = blockIdx.x >= total || load_tile_scales(blockIdx.x, 0);
      const int kb_next = min(3, KB - 1);
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        int e, wb, tb, rows;
        decode(tile, e, wb, tb, rows);
        const int tok_tile = s_tb[e] + tb;
        const int row_b = tok_tile * NT;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, args.status))) break;
          const uint32_t st = sbase + s * C::STAGE_BYTES;
          const uint32_t fb = bar_full(s);
          mbar_expect_tx(fb, C::TX_BYTES);
          const bool last_tail = tail && kb == KB - 1;
          const CUtensorMap* am = last_tail ? &tmAt : &tmA;
          const int ax = last_tail ? 0 : kb * 128;
          if (EPI == EPI_SWIGLU) {
            // row blocks q = 0..3 of 16 gate rows then the same 16 up rows
            // (TMEM lanes 32q..32q+15 gate, 32q+16..32q+31 up)
            tma_load_4d(st, am, ax, 0, 2 * e, 4 * wb, fb);
          } else {
            tma_load_3d(st, am, ax, wb * 128, e, fb);
          }
          const int bx = last_tail ? K - 128 : kb * 128;
          if (C::ACT == ACT_HILO)
            tma_load_3d(st + C::OFF_B, &tmB, bx, row_b, 0, fb);   // hi rows, then lo rows
          else if (C::ACT == ACT_E4M3)
            tma_load_2d(st + C::OFF_B, &tmB, bx, row_b, fb);
          else   // packed E2M1 rows, widened like the weight codes (tail map for [K-128, K))
            tma_load_2d(st + C::OFF_B, last_tail ? &tmBt : &tmB, last_tail ? 0 : kb * 128, row_b, fb);
          bulk_load(st + C::OFF_SFB,
                    args.sfb + (static_cast<size_t>(tok_tile) * KB + kb) * C::SFB_BYTES,
                    C::SFB_BYTES, fb);
          if (++s == C::STAGES) { s = 0; ph ^= 1; }
          if (kb == kb_next && tile + static_cast<int>(gridDim.x) < total &&
              !(ok = load_tile_scales(tile + gridDim.x, it + 1)))
            break;
        }
      }
    }
  } else if (warp == 2) {
    // -------------------------------------------------- A-scale builder --
    // Lane l fills bytes 16l..16l+15 of the k-block's 512-byte atom: the 4
    // scale bytes of A-tile rows l, l+32, l+64, l+96, read from the tile's
    // scale block (2-byte aligned rows of G bytes).
    int srow[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (EPI == EPI_SWIGLU)   // gate rows first, then up rows, 64 each
        srow[j] = (lane < 16) ? 16 * j + lane : 64 + 16 * j + (lane - 16);
      else
        srow[j] = 32 * j + lane;
    }
    int s = 0, ph = 0, it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
      const int b = it & 1;
      if (!(ok = mbar_wait(bar_tsFull(b), (it >> 1) & 1, abort_flag, args.status))) break;
      const uint8_t* ts = smem + C::OFF_TS + b * C::TS_BYTES;
      for (int kb = 0; kb < KB; ++kb) {
        const int gs = (tail && kb == KB - 1) ? G - 4 : 4 * kb;
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint16_t* p = reinterpret_cast<const uint16_t*>(ts + srow[j] * G + gs);
          w[j] = static_cast<uint32_t>(p[0]) | (static_cast<uint32_t>(p[1]) << 16);
        }
        if (!(ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, args.status))) break;
        *reinterpret_cast<uint4*>(smem + s * C::STAGE_BYTES + C::OFF_SFA + lane * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
        // orders this k-block's shared-memory reads and writes before the
        // async-proxy accesses that follow (tcgen05.cp of the atom; the next
        // bulk copy into the tile-scale buffer)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_full(s));
        if (++s == C::STAGES) { s = 0; ph ^= 1; }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_tsEmpty(b));
    }
  } else if (warp == 1 || (C::ISSUERS == 2 && warp == 3)) {
    // ------------------------------------------------------- UMMA issuers --
    // Issuer u takes the k-blocks with q % 2 == u (q counts this CTA's
    // k-blocks across tiles), i.e. the stages s with s % 2 == u; the other
    // issuer's k-blocks are stepped over without touching their barriers.
    const int u = warp == 1 ? 0 : 1;
    if (lane == 0) {
      const uint32_t idesc0 = idesc_mx_e2m1(C::MW, C::N, 0, 0, C::BTYPE);
      const uint32_t sfa_t = tmem_base + C::SF_COL0 + u * C::SF_COLS, sfb_t = sfa_t + 4;
      int s = 0, ph = 0, it = 0, q = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t ap = (it >> 1) & 1;
        if (!(ok = mbar_wait(bar_accEmpty(ab), ap ^ 1, abort_flag, args.status))) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (2 * u + ab) * C::N;
        uint32_t accum = 0;   // the issuer's first k-block of the tile overwrites its buffer
        for (int kb = 0; kb < KB; ++kb, ++q) {
          if ((q % C::ISSUERS) == u) {
            if (!(ok = mbar_wait(bar_full(s), ph, abort_flag, args.status))) break;
            tc_fence_after();
            const uint32_t st = sbase + s * C::STAGE_BYTES;
            tmem_cp_32x128b_x4(sfa_t, sdesc_k_noswizzle(st + C::OFF_SFA, 128));
#pragma unroll
            for (int a = 0; a < C::SFB_BYTES / 512; ++a)
              tmem_cp_32x128b_x4(sfb_t + 4 * a, sdesc_k_noswizzle(st + C::OFF_SFB + 512 * a, 128));
            // K steps with compile-time indices (a data-dependent trip count
            // here measurably slows the issue of each UMMA); the tail k-block
            // of a K that is 64 mod 128 issues its last two steps only
            auto step = [&](const int kk, const uint32_t acc) {
              umma_mxf8f6f4(d, sdesc_k_sw128(st + kk * 32), sdesc_k_sw128(st + C::OFF_B + kk * 32),
                            idesc0 | (static_cast<uint32_t>(kk) << 4) |
                                (static_cast<uint32_t>(kk) << 29),
                            sfa_t | (static_cast<uint32_t>(kk) << 30),
                            sfb_t | (static_cast<uint32_t>(kk) << 30), acc);
            };
            if (!(tail && kb == KB - 1)) {
              step(0, accum);
              step(1, 1u);
              step(2, 1u);
              step(3, 1u);
            } else {
              step(2, accum);
              step(3, 1u);
            }
            accum = 1;
            umma_commit(bar_empty(s));
          }
          if (++s == C::STAGES) { s = 0; ph ^= 1; }
        }
        if (ok) umma_commit(bar_accFull(ab));
      }
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- epilogue --
    // Chunks of CH token columns: hi and lo of every issuer's buffer are
    // loaded and added, then SwiGLU + the hi/lo split of H (gate/up) or the
    // weighted store (down). Every epilogue warp passes the SwiGLU exchange
    // barrier once per chunk, also after a failed wait, so that no warp is
    // left at it alone.
    constexpr int CH = C::CH;
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. +31
    const int grp = (warp - 4) >> 2;           // epilogue group: chunks grp, grp + G, ...
    const int m = quad * 32 + lane;            // weight row of the tile
    const uint32_t lanes = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    int it = 0, xc = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      int e, wb, tb, rows;
      decode(tile, e, wb, tb, rows);
      const int ab = it & 1;
      const uint32_t ap = (it >> 1) & 1;
      if (ok) ok = mbar_wait(bar_accFull(ab), ap, abort_flag, args.status);
      ok = __all_sync(0xFFFFFFFFu, ok);        // the TMEM loads below are warp-collective
      if (!ok && EPI != EPI_SWIGLU) break;
      if (ok) tc_fence_after();
      // with two issuers and a single k-block per tile only issuer
      // (it*KB) % 2 wrote its buffer
      const bool use0 = C::ISSUERS == 1 || KB > 1 || ((it * KB) & 1) == 0;
      const bool use1 = C::ISSUERS == 2 && (KB > 1 || ((it * KB) & 1) == 1);
      const uint32_t t0 = tmem_base + lanes + ab * C::N;
      const uint32_t t1 = tmem_base + lanes + (2 + ab) * C::N;
      const int tok_tile = s_tb[e] + tb;
      const int j = wb * 64 + 16 * quad + (lane & 15);      // SwiGLU: H column of this lane
      const bool jv = j < args.I && lane < 16;
      const int col = wb * 128 + m;                          // down: output column
      // the bias of this lane's weight row (gate or up row j, or output column)
      float bl = 0.f;
      if (args.bias) {
        if (EPI == EPI_SWIGLU) {
          if (j < args.I)
            bl = args.bias[static_cast<int64_t>(e) * 2 * args.I + (lane >> 4) * args.I + j];
        } else if (col < args.n_out) {
          bl = args.bias[static_cast<int64_t>(e) * args.n_out + col];
        }
      }
#pragma unroll 1
      for (int c = grp * CH; c < NT; c += C::EPI_GROUPS * CH, ++xc) {
        float y[CH];
#pragma unroll
        for (int i = 0; i < CH; ++i) y[i] = 0.f;
        if (ok && c < rows) {
          uint32_t a[8], b[8];
          if (C::TERMS == 2) {   // hi and lo products of the bf16 split
            if (use0) {
              tmem_ld8x2_sync(t0 + c, t0 + NT + c, a, b);
#pragma unroll
              for (int i = 0; i < CH; ++i) y[i] = __uint_as_float(a[i]) + __uint_as_float(b[i]);
            }
            if (use1) {
              tmem_ld8x2_sync(t1 + c, t1 + NT + c, a, b);
#pragma unroll
              for (int i = 0; i < CH; ++i) y[i] += __uint_as_float(a[i]) + __uint_as_float(b[i]);
            }
          } else {
            if (use0) {
              tmem_ld8_sync(t0 + c, a);
#pragma unroll
              for (int i = 0; i < CH; ++i) y[i] = __uint_as_float(a[i]);
            }
            if (use1) {
              tmem_ld8_sync(t1 + c, a);
#pragma unroll
              for (int i = 0; i < CH; ++i) y[i] += __uint_as_float(a[i]);
            }
          }
        }
        if (EPI == EPI_SWIGLU) {
          // lanes 0-15: gate row j, lanes 16-31: up row j; y becomes h for the
          // gate lanes and 0 elsewhere
          float* xch = s_xch + (grp * 2 + (xc & 1)) * 4 * CH;
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            y[i] += bl;
            const float u = __shfl_xor_sync(0xFFFFFFFFu, y[i], 16);
            float hv = 0.f;
            if (ok && jv && c + i < rows) {
              hv = silu_mx(y[i]) * u;
              // bf16 precision: H is a bf16 row (split exactly below); the
              // quantised modes convert the fp32 value itself
              if (C::ACT == ACT_HILO) hv = __bfloat162float(__float2bfloat16_rn(hv));
            }
            y[i] = hv;
            float pm = fabsf(hv);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xFFFFFFFFu, pm, o));
            if (lane == 0) xch[quad * CH + i] = pm;
          }
          // max |h| over the 32 j of a group: quarters 0+1 and 2+3 (named
          // barrier 1 + grp over the group's four warps)
          asm volatile("bar.sync %0, 128;" ::"r"(1 + grp) : "memory");
          if (ok && C::ACT != ACT_HILO) {
            // one MX-converted element per H value: E4M3 bytes, or E2M1 codes
            // packed in pairs (the even H column in the low nibble: lanes j
            // and j + 1 are neighbours, the even one stores the byte)
            const int gj = 2 * wb + (quad >> 1);
            int kb4, kk4;
            group_to_kblock(gj, args.I / 32, args.h_kb, kb4, kk4);
            uint8_t* hsfb = args.h_sfb + (static_cast<size_t>(tok_tile) * args.h_kb + kb4) *
                                             sfb_block_bytes(NT, 1);
#pragma unroll
            for (int i = 0; i < CH; ++i) {
              const int t = c + i;
              const float amax = fmaxf(xch[quad * CH + i], xch[(quad ^ 1) * CH + i]);
              const int ex = mx_scale_exp<C::ACT>(amax);
              const float a = y[i] * __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
              const size_t row = static_cast<size_t>(tok_tile * NT + t);
              if (C::ACT == ACT_E4M3) {
                if (jv && t < rows)
                  args.h_hi[row * args.I + j] = static_cast<uint8_t>(f32x2_to_e4m3x2(a, 0.f) & 0xFF);
              } else {
                const uint32_t code = f32_to_e2m1(a);
                const uint32_t odd = __shfl_xor_sync(0xFFFFFFFFu, code, 1);
                if (jv && t < rows && !(j & 1))
                  args.h_hi[row * (args.I / 2) + j / 2] = static_cast<uint8_t>(code | (odd << 4));
              }
              if (t < rows && lane == 0 && !(quad & 1))
                hsfb[sfb_offset(NT, t, 0, kk4)] = static_cast<uint8_t>(ex + 127);
            }
          } else if (ok) {
            const int gj = 2 * wb + (quad >> 1);
            int kb4, kk4;
            group_to_kblock(gj, args.I / 32, args.h_kb, kb4, kk4);
            uint8_t* hsfb = args.h_sfb + (static_cast<size_t>(tok_tile) * args.h_kb + kb4) *
                                             sfb_block_bytes(NT);
#pragma unroll
            for (int i = 0; i < CH; ++i) {
              const int t = c + i;
              if (t < rows) {
                const float amax = fmaxf(xch[quad * CH + i], xch[(quad ^ 1) * CH + i]);
                int eh = 0;
                if (amax != 0.f) {
                  const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127;
                  eh = max(ex - 7, -123);
                }
                const float inv = __uint_as_float(static_cast<uint32_t>(127 - eh) << 23);
                const float a = y[i] * inv;
                const uint32_t h2 = f32x2_to_e4m3x2(a, 0.f);
                const float2 hb = e4m3x2_to_f32x2(h2);
                const uint32_t l2 = f32x2_to_e4m3x2((a - hb.x) * 16.f, 0.f);
                if (jv) {
                  const size_t o = static_cast<size_t>(tok_tile * NT + t) * args.I + j;
                  args.h_hi[o] = static_cast<uint8_t>(h2 & 0xFF);
                  args.h_lo[o] = static_cast<uint8_t>(l2 & 0xFF);
                }
                if (lane == 0 && !(quad & 1)) {
                  hsfb[sfb_offset(NT, t, 0, kk4)] = static_cast<uint8_t>(eh + 127);
                  hsfb[sfb_offset(NT, t, 1, kk4)] = static_cast<uint8_t>(eh + 123);
                }
              }
            }
          }
        } else if (ok && col < args.n_out) {
          const int p0 = s_off[e] + tb * NT;
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            if (c + i < rows) {
              const int pr = args.perm[p0 + c + i];
              args.out_f32[static_cast<int64_t>(pr) * args.n_out + col] =
                  args.topk_w[pr] * (y[i] + bl);
            }
          }
        }
      }
      if (ok) {
        tc_fence_before();
        mbar_arrive(bar_accEmpty(ab));     // this tile's accumulators are read
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ----------------------------------------------------------- host side ----

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

bool encode_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};   // element strides, one per dimension (rank <= 5)
  if (rank < 1 || rank > 5) return false;
  return enc(m, dt, rank, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E2M1 code maps (K elements first, then `rank`-1 row dimensions given by
// dims_rest / strides / box_rest): the main map covers the first
// 128*floor(K/128) elements of each row, the tail map the last 128 (based
// (K-128)/2 bytes into the row); both widen to 8-bit containers.
bool make_code_maps(CUtensorMap* main_map, CUtensorMap* tail_map, const uint8_t* codes, int K,
                    int rank, const cuuint64_t* dims_rest, const cuuint64_t* strides,
                    const cuuint32_t* box_rest) {
  cuuint64_t dims[5];
  cuuint32_t box[5];
  for (int i = 1; i < rank; ++i) {
    dims[i] = dims_rest[i - 1];
    box[i] = box_rest[i - 1];
  }
  box[0] = 128;
  const int kmain = (K / 128) * 128;
  bool ok = true;
  if (kmain > 0) {
    dims[0] = static_cast<cuuint64_t>(kmain);
    ok = encode_map(main_map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, rank, codes, dims, strides,
                    box);
  }
  if (ok && (K % 128) != 0) {
    dims[0] = 128;
    ok = encode_map(tail_map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, rank, codes + (K - 128) / 2,
                    dims, strides, box);
  } else if (ok) {
    *tail_map = *main_map;
  }
  if (ok && kmain == 0) *main_map = *tail_map;
  return ok;
}

// E4M3 token rows: hi rows [rows][K] followed by lo rows [rows][K], as one
// (K, rows, 2) tensor; box 128 x NT x 2 (hi tile, then lo tile).
bool make_tok8_map(CUtensorMap* m, const uint8_t* hi, int rows, int K, int nt) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows), 2};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K),
                                 static_cast<cuuint64_t>(K) * static_cast<cuuint64_t>(rows)};
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(nt), 2};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, hi, dims, strides, box);
}

// One plane of E4M3 token rows [rows][K]; box 128 x NT.
bool make_tok8_map1(CUtensorMap* m, const uint8_t* q, int rows, int K, int nt) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(nt)};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box);
}

template <int EPI, class C>
cudaError_t launch_mx_impl(const MxGemmProblem& p, int num_sms, cudaStream_t st) {
  constexpr int NT = C::NT;
  // the kernel assumes K % 64 == 0 (tail k-blocks of 2 steps) and K <= kMxMaxK
  if (p.K % 64 != 0 || p.K < 128 || p.K > kMxMaxK) return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_mx_gemm_kernel<EPI, C>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // the hi and lo token rows are read as the two planes of one tensor
  if (C::ACT == ACT_HILO && p.b_lo != p.b_hi + static_cast<size_t>(p.tok_rows) * p.K)
    return cudaErrorInvalidValue;
  if (p.act != C::ACT) return cudaErrorInvalidValue;
  CUtensorMap tmA, tmAt, tmB, tmBt;
  const cuuint64_t rb = static_cast<cuuint64_t>(p.K / 2);
  bool ok;
  if (EPI == EPI_SWIGLU) {
    // codes [E][2][I][K/2] as (K, 16 rows, 2E planes, I/16 row blocks): one
    // box = 4 row blocks x (16 gate rows, 16 up rows)
    const cuuint64_t dims[3] = {16, static_cast<cuuint64_t>(2 * p.E),
                                static_cast<cuuint64_t>(p.I / 16)};
    const cuuint64_t strides[3] = {rb, rb * static_cast<cuuint64_t>(p.I), rb * 16};
    const cuuint32_t box[3] = {16, 2, 4};
    ok = make_code_maps(&tmA, &tmAt, p.codes, p.K, 4, dims, strides, box);
  } else {
    // codes [E][d][K/2] as (K, d rows, E): one box = 128 rows
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.n_out), static_cast<cuuint64_t>(p.E)};
    const cuuint64_t strides[2] = {rb, rb * static_cast<cuuint64_t>(p.n_out)};
    const cuuint32_t box[2] = {128, 1};
    ok = make_code_maps(&tmA, &tmAt, p.codes, p.K, 3, dims, strides, box);
  }
  if (C::ACT == ACT_HILO) {
    ok = ok && make_tok8_map(&tmB, p.b_hi, p.tok_rows, p.K, NT);
    tmBt = tmB;
  } else if (C::ACT == ACT_E4M3) {
    ok = ok && make_tok8_map1(&tmB, p.b_hi, p.tok_rows, p.K, NT);
    tmBt = tmB;
  } else {
    // packed E2M1 token rows [tok_rows][K/2], widened to 8-bit containers
    const cuuint64_t dims[1] = {static_cast<cuuint64_t>(p.tok_rows)};
    const cuuint64_t strides[1] = {rb};
    const cuuint32_t box[1] = {static_cast<cuuint32_t>(NT)};
    ok = ok && make_code_maps(&tmB, &tmBt, p.b_hi, p.K, 2, dims, strides, box);
  }
  if (!ok) return cudaErrorInvalidValue;
  MxArgs a;
  a.offsets = p.offsets;
  a.E = p.E;
  a.K = p.K;
  a.I = p.I;
  a.scales = p.scales;
  a.sfb = p.b_sfb;
  a.h_hi = p.h_hi;
  a.h_lo = p.h_lo;
  a.h_sfb = p.h_sfb;
  a.h_kb = (p.I + 127) / 128;
  a.out_f32 = p.out_f32;
  a.n_out = p.n_out;
  a.perm = p.perm;
  a.topk_w = p.topk_w;
  a.bias = p.bias;
  a.status = p.status;
  if (EPI == EPI_SWIGLU) {
    a.n_wb = (p.I + 63) / 64;
    a.rows_per_expert = 2 * p.I;
  } else {
    a.n_wb = (p.n_out + 127) / 128;
    a.rows_per_expert = p.n_out;
  }
  const int64_t tiles_bound = (static_cast<int64_t>(p.P) / NT + p.E) * a.n_wb;
  int64_t grid = C::CTAS * static_cast<int64_t>(num_sms);
  if (tiles_bound < grid) grid = tiles_bound;
  if (grid < 1) grid = 1;
  launch_kernel(grouped_mx_gemm_kernel<EPI, C>, dim3(static_cast<int>(grid)), dim3(C::NUM_THREADS), C::SMEM_ALLOC, st, 
      tmA, tmAt, tmB, tmBt, a);
  return cudaGetLastError();
}


int grid_for_n(int64_t n, int per_thread_block, int cap) {
  int64_t b = (n + per_thread_block - 1) / per_thread_block;
  if (b < 1) b = 1;
  if (b > cap) b = cap;
  return static_cast<int>(b);
}

}  // namespace

bool mx_make_code_maps(CUtensorMap* main_map, CUtensorMap* tail_map, const uint8_t* codes, int K,
                       int rank, const cuuint64_t* dims_rest, const cuuint64_t* strides,
                       const cuuint32_t* box_rest) {
  return make_code_maps(main_map, tail_map, codes, K, rank, dims_rest, strides, box_rest);
}
bool mx_make_tok8_map(CUtensorMap* m, const uint8_t* hi, int rows, int K, int nt) {
  return make_tok8_map(m, hi, rows, K, nt);
}
bool mx_make_tok8_map1(CUtensorMap* m, const uint8_t* q, int rows, int K, int nt) {
  return make_tok8_map1(m, q, rows, K, nt);
}
bool mx_make_bytes_map(CUtensorMap* m, const uint8_t* base, int rank, const cuuint64_t* dims,
                       const cuuint64_t* strides, const cuuint32_t* box) {
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, base, dims, strides, box);
}
bool mx_encode_bf16_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                        const cuuint64_t* strides, const cuuint32_t* box) {
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides, box);
}

int mx_tile_tokens(int variant, int act) {
  if (variant == kMxPair) return kMxMaxNT;
  if (act == ACT_HILO) return variant == kMxLarge ? MxLarge::NT : MxSmall::NT;
  return variant == kMxLarge ? MxLargeQ<ACT_E4M3>::NT : MxSmallQ<ACT_E4M3>::NT;
}

size_t mx_tok_rows(int P, int E) {
  static_assert(MxLarge::NT <= kMxMaxNT && MxLargeQ<ACT_E4M3>::NT <= kMxMaxNT, "granule");
  return static_cast<size_t>(P) + static_cast<size_t>(E) * (kMxMaxNT - 1);
}

size_t mx_sfb_bytes(int P, int E, int K) {
  size_t best = 0;
  const int variants[5][2] = {{MxSmall::NT, 2}, {MxLarge::NT, 2}, {MxSmallQ<ACT_E4M3>::NT, 1},
                              {MxLargeQ<ACT_E4M3>::NT, 1}, {kMxMaxNT, 2}};
  for (const auto& v : variants) {
    const size_t tiles = (static_cast<size_t>(P) + v[0] - 1) / v[0] + E;
    const size_t b = tiles * ((K + 127) / 128) * sfb_block_bytes(v[0], v[1]);
    if (b > best) best = b;
  }
  // the kind::mxf4 pair kernel's blocks: 1024 bytes per 256-wide k-block
  const size_t f4 = ((static_cast<size_t>(P) + kMxMaxNT - 1) / kMxMaxNT + E) * ((K + 255) / 256) * 1024;
  return f4 > best ? f4 : best;
}

cudaError_t launch_mx_quant_gather(int variant, const uint16_t* x, const int32_t* perm,
                                   const int32_t* offsets, int E, int P, int k, int K, uint8_t* qhi,
                                   uint8_t* qlo, uint8_t* sfb, const int32_t* topk_idx,
                                   const int32_t* inv, int T, cudaStream_t st) {
  if (inv && topk_idx) {
    const int grid = grid_for_n(static_cast<int64_t>(T) * (K / 32), 256, 148 * 8);
    if (variant == kMxPair)
      launch_kernel(mx_quant_gather_tok_kernel<kMxMaxNT>, dim3(grid), dim3(256), 0, st, x,
                    topk_idx, inv, offsets, E, T, k, K, qhi, qlo, sfb);
    else if (variant == kMxLarge)
      launch_kernel(mx_quant_gather_tok_kernel<MxLarge::NT>, dim3(grid), dim3(256), 0, st, x,
                    topk_idx, inv, offsets, E, T, k, K, qhi, qlo, sfb);
    else
      launch_kernel(mx_quant_gather_tok_kernel<MxSmall::NT>, dim3(grid), dim3(256), 0, st, x,
                    topk_idx, inv, offsets, E, T, k, K, qhi, qlo, sfb);
    return cudaGetLastError();
  }
  const int64_t n = static_cast<int64_t>(P) * (K / 32);
  const int grid = grid_for_n(n, 256, 148 * 8);
  if (variant == kMxPair)
    launch_kernel(mx_quant_gather_kernel<kMxMaxNT>, dim3(grid), dim3(256), 0, st, x, perm, offsets, E, P, k, K, qhi, qlo,
                                                            sfb);
  else if (variant == kMxLarge)
    launch_kernel(mx_quant_gather_kernel<MxLarge::NT>, dim3(grid), dim3(256), 0, st, x, perm, offsets, E, P, k, K, qhi,
                                                               qlo, sfb);
  else
    launch_kernel(mx_quant_gather_kernel<MxSmall::NT>, dim3(grid), dim3(256), 0, st, x, perm, offsets, E, P, k, K, qhi,
                                                               qlo, sfb);
  return cudaGetLastError();
}

cudaError_t launch_mx_act_quant_gather(int variant, int act, const uint16_t* x,
                                       const int32_t* perm, const int32_t* offsets, int E, int P,
                                       int k, int K, uint8_t* q, uint8_t* sfb, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(P) * (K / 32);
  const int grid = grid_for_n(n, 256, 148 * 8);
  constexpr int NS = MxSmallQ<ACT_E4M3>::NT, NL = MxLargeQ<ACT_E4M3>::NT;
  static_assert(NL == kMxMaxNT, "the large and pair variants share the 128-row layout");
  if (act == ACT_E4M3) {
    if (variant != kMxSmall)
      launch_kernel(mx_act_quant_gather_kernel<NL, ACT_E4M3>, dim3(grid), dim3(256), 0, st, x, perm, offsets, E, P, k, K, q, sfb);
    else
      launch_kernel(mx_act_quant_gather_kernel<NS, ACT_E4M3>, dim3(grid), dim3(256), 0, st, x, perm, offsets, E, P, k, K, q, sfb);
  } else if (act == ACT_F4) {
    if (variant != kMxPair) return cudaErrorInvalidValue;
    launch_kernel(mx_act_quant_gather_kernel<NL, ACT_E2M1, true>, dim3(grid), dim3(256), 0, st, x, perm, offsets, E, P, k,
                                                                        K, q, sfb);
  } else if (act == ACT_E2M1) {
    if (variant != kMxSmall)
      launch_kernel(mx_act_quant_gather_kernel<NL, ACT_E2M1>, dim3(grid), dim3(256), 0, st, x, perm, offsets, E, P, k, K, q, sfb);
    else
      launch_kernel(mx_act_quant_gather_kernel<NS, ACT_E2M1>, dim3(grid), dim3(256), 0, st, x, perm, offsets, E, P, k, K, q, sfb);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_mx_act_quant_rows(int act, const uint16_t* x, int R, int K, uint8_t* q,
                                     uint8_t* scales, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(R) * (K / 32);
  const int grid = grid_for_n(n, 256, 148 * 8);
  if (act == ACT_E4M3)
    launch_kernel(mx_act_quant_rows_kernel<ACT_E4M3>, dim3(grid), dim3(256), 0, st, x, R, K, q, scales);
  else if (act == ACT_E2M1)
    launch_kernel(mx_act_quant_rows_kernel<ACT_E2M1>, dim3(grid), dim3(256), 0, st, x, R, K, q, scales);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_mx_split_rows(const uint16_t* x, int R, int K, uint8_t* qhi, uint8_t* qlo,
                                 uint8_t* scales, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(R) * (K / 32);
  launch_kernel(mx_split_rows_kernel, dim3(grid_for_n(n, 256, 148 * 8)), dim3(256), 0, st, x, R, K, qhi, qlo,
                scales);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_mx_dispatch(int variant, const MxGemmProblem& p, int num_sms, cudaStream_t st) {
  const bool large = variant == kMxLarge;
  switch (p.act) {
    case ACT_HILO:
      return large ? launch_mx_impl<EPI, MxLarge>(p, num_sms, st)
                   : launch_mx_impl<EPI, MxSmall>(p, num_sms, st);
    case ACT_E4M3:
      return large ? launch_mx_impl<EPI, MxLargeQ<ACT_E4M3>>(p, num_sms, st)
                   : launch_mx_impl<EPI, MxSmallQ<ACT_E4M3>>(p, num_sms, st);
    case ACT_E2M1:
      return large ? launch_mx_impl<EPI, MxLargeQ<ACT_E2M1>>(p, num_sms, st)
                   : launch_mx_impl<EPI, MxSmallQ<ACT_E2M1>>(p, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_mx_gemm_gateup_swiglu(int variant, const MxGemmProblem& p, int num_sms,
                                         cudaStream_t st) {
  return launch_mx_dispatch<EPI_SWIGLU>(variant, p, num_sms, st);
}

cudaError_t launch_mx_gemm_down(int variant, const MxGemmProblem& p, int num_sms,
                                cudaStream_t st) {
  return launch_mx_dispatch<EPI_DOWN>(variant, p, num_sms, st);
}

}  // namespace moe
