// moe_topk.cuh -- top-k over one token's expert logits and the softmax over
// the selected set, one warp per token ("llm-surgery-dark-arts-gpt-oss-40b-
// 64a8-init", section 2, "Proof": i in top-k(s), p_i = exp(s_i) / sum over
// the selected set). Used by the router kernel of moe_router_tc.cu.
#pragma once

#include <float.h>
#include <stdint.h>

namespace moe {

// The arg-max of the top-k compares 32-bit keys that order the logits totally: a float's
// bits mapped to an unsigned integer that increases with the value, -0 taken
// as +0 (equal logits tie, the lower index wins), and every NaN mapped below
// -inf (key 0). A NaN logit therefore loses to every number, NaNs tie among
// themselves, and every lane of the warp agrees on each round's winner.
__device__ __forceinline__ uint32_t logit_order_key(float f) {
  if (f != f) return 0u;                          // NaN: below everything
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                   // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The logit a key stands for (-0 comes back as +0, any NaN as a NaN).
__device__ __forceinline__ float logit_of_key(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Same 64-bit order for fp64 values (a float widened to double keeps its
// place among the floats).
__device__ __forceinline__ uint64_t value_order_key(double f) {
  if (f != f) return 0ull;
  uint64_t u = static_cast<uint64_t>(__double_as_longlong(f));
  if (u == 0x8000000000000000ull) u = 0ull;
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

// Expert held in slot j of lane l: four consecutive experts per lane in each
// half of 128 (so that a lane reads its logits with 16-byte loads).
__device__ __forceinline__ int slot_expert(int lane, int j) {
  return 128 * (j >> 2) + 4 * lane + (j & 3);
}

// One warp per token: the top-k of the token's logits v (slot j of lane l
// holds expert slot_expert(l, j), -FLT_MAX past E), the order of near ties
// settled in fp64, and the softmax over the k selected. Three steps, which a
// kernel may run apart (all refinements of a block together, for instance):
//
// 1. topk_list: rounds of a warp arg-max on (logit descending, index
//    ascending; two redux instructions per round) list the k largest logits,
//    then go on while the next one lies within tau of the k-th (the
//    candidates that might belong in the top k), at most 64 entries. Position
//    p of the list sits in lane p % 32, slot p / 32. An entry is to be
//    refined when its gap to the entry before or after it is at most tau.
//    Rows with equal fingerprints (fps: equal router rows and biases, e.g.
//    copied experts) and equal fp32 logits are copies: a gap of zero between
//    copies needs no refinement (their logits are equal on every evaluation
//    and already in index order); where one copy is refined, all copies of
//    its group are, with one value. Entries whose gaps are all above tau keep
//    their fp32 value, which lies within tau/2 of the exact one on either
//    side, so no refined entry can pass them. tau = 0 turns refinement off.
// 2. The refined entries' logits become fp64 dot products of the bf16 x row
//    with the fp32 router row (every product exact in fp64), plus the bias:
//    topk_refine_warp does it with the warp alone.
// 3. topk_emit: with any entry refined, k rounds of the arg-max over the list
//    (fp64 values) give the final order, else the list's first k entries are
//    the result; then the softmax over the k and the stores.
struct TopkList {
  int cidx[2];       // expert at positions lane and 32 + lane
  float cval[2];     // its fp32 logit
  int m;             // entries in the list
  uint64_t refine_m; // positions to refine (bit p)
  uint64_t copy_m;   // bit p: the entry at p + 1 is a copy of the one at p
};

__device__ __forceinline__ void topk_list(const float (&v)[8], int E, int k, float tau,
                                          const unsigned long long* __restrict__ fps, int lane,
                                          TopkList& L) {
  const unsigned full = 0xFFFFFFFFu;
  uint32_t key[8];
  uint32_t taken = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = slot_expert(lane, j);
    key[j] = logit_order_key(v[j]);
    if (e >= E) taken |= 1u << j;
  }
  L.cidx[0] = L.cidx[1] = 0;
  L.cval[0] = L.cval[1] = 0.f;
  L.m = 0;
  L.refine_m = L.copy_m = 0;
  float kth = 0.f;
  const int maxc = E < 64 ? E : 64;
  const bool refine = tau > 0.f;
  for (int r = 0; r < maxc; ++r) {
    // this lane's best untaken entry, then the warp's: the largest key
    // (redux max), among the lanes holding it the lowest expert (redux min)
    uint32_t bk = 0;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (taken & (1u << j)) continue;
      const int e = slot_expert(lane, j);
      if (bi == 0x7FFFFFFF || key[j] > bk || (key[j] == bk && e < bi)) {
        bk = key[j];
        bi = e;
      }
    }
    const uint32_t top_key = __reduce_max_sync(full, bk);
    bi = static_cast<int>(__reduce_min_sync(
        full, (bi != 0x7FFFFFFF && bk == top_key) ? static_cast<uint32_t>(bi) : 0xFFFFFFFFu));
    const float bv = logit_of_key(top_key);
    // past the k-th: only runners-up within tau of it
    if (r >= k && !(refine && kth - bv <= tau)) break;
    if (((bi & 127) >> 2) == lane) taken |= 1u << (((bi >> 7) << 2) | (bi & 3));
    if (r == k - 1) kth = bv;
    if ((r & 31) == lane) {
      if (r < 32) {
        L.cidx[0] = bi;
        L.cval[0] = bv;
      } else {
        L.cidx[1] = bi;
        L.cval[1] = bv;
      }
    }
    L.m = r + 1;
  }
  const int m = L.m;
  // links between positions p and p + 1: close (gap at most tau) and, among
  // those, copies; fingerprints are read only when some link is close
  float nx0 = __shfl_down_sync(full, L.cval[0], 1);
  const float head1 = __shfl_sync(full, L.cval[1], 0);
  if (lane == 31) nx0 = head1;
  const float nx1 = __shfl_down_sync(full, L.cval[1], 1);
  const bool close0 = refine && lane + 1 < m && L.cval[0] - nx0 <= tau;
  const bool close1 = refine && 33 + lane < m && L.cval[1] - nx1 <= tau;
  const uint64_t close_m = static_cast<uint64_t>(__ballot_sync(full, close0)) |
                           (static_cast<uint64_t>(__ballot_sync(full, close1)) << 32);
  if (close_m) {
    const unsigned long long f0 = lane < m ? __ldg(fps + L.cidx[0]) : 0ull;
    const unsigned long long f1 = 32 + lane < m ? __ldg(fps + L.cidx[1]) : 0ull;
    unsigned long long nf0 = __shfl_down_sync(full, f0, 1);
    const unsigned long long fhead1 = __shfl_sync(full, f1, 0);
    if (lane == 31) nf0 = fhead1;
    const unsigned long long nf1 = __shfl_down_sync(full, f1, 1);
    const uint64_t copy_m =
        static_cast<uint64_t>(__ballot_sync(full, close0 && L.cval[0] == nx0 && f0 == nf0)) |
        (static_cast<uint64_t>(__ballot_sync(full, close1 && L.cval[1] == nx1 && f1 == nf1))
         << 32);
    // both ends of every close link that is not a copy, then whole groups of
    // copies around them
    const uint64_t near_m = close_m & ~copy_m;
    uint64_t rm = near_m | (near_m << 1);
    for (;;) {
      const uint64_t g = rm | ((rm << 1) & (copy_m << 1)) | ((rm >> 1) & copy_m);
      if (g == rm) break;
      rm = g;
    }
    L.refine_m = rm;
    L.copy_m = copy_m;
  }
}

// Entries computed for a refined list: the first entry of each refined group
// of copies (the others take its value).
__device__ __forceinline__ uint64_t topk_refine_starts(const TopkList& L) {
  return L.refine_m & ~(L.copy_m << 1);
}

// Positions pos .. pos + len - 1 of the group that starts at pos.
__device__ __forceinline__ int topk_group_len(const TopkList& L, int pos) {
  return __ffsll(static_cast<long long>(~(L.copy_m >> pos)));
}

// Step 2 by the warp alone: val[slot] becomes the fp64 logit of each refined
// entry (others keep their fp32 value).
__device__ __forceinline__ void topk_refine_warp(const TopkList& L,
                                                 const uint16_t* __restrict__ x_row,
                                                 const float* __restrict__ W_r,
                                                 const float* __restrict__ b_r, int d, int lane,
                                                 double (&val)[2]) {
  const unsigned full = 0xFFFFFFFFu;
  uint64_t pending = topk_refine_starts(L);
  const int d128 = d & ~127;
  while (pending) {
    // up to four refined entries per pass over the x row
    int pos[4], ex[4];
    int ng = 0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      pos[g] = -1;
      ex[g] = 0;
      if (pending) {
        const int p = __ffsll(static_cast<long long>(pending)) - 1;
        pending &= pending - 1;
        const int src = (p >> 5) ? L.cidx[1] : L.cidx[0];
        pos[g] = p;
        ex[g] = __shfl_sync(full, src, p & 31);
        ng = g + 1;
      }
    }
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
    for (int i = 4 * lane; i < d128; i += 128) {
      const uint2 xb = __ldg(reinterpret_cast<const uint2*>(x_row + i));
      const double x0 = __uint_as_float(xb.x << 16), x1 = __uint_as_float(xb.x & 0xFFFF0000u);
      const double x2 = __uint_as_float(xb.y << 16), x3 = __uint_as_float(xb.y & 0xFFFF0000u);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (g < ng) {
          const float4 w =
              __ldg(reinterpret_cast<const float4*>(W_r + static_cast<size_t>(ex[g]) * d + i));
          acc[g] = fma(x0, static_cast<double>(w.x), acc[g]);
          acc[g] = fma(x1, static_cast<double>(w.y), acc[g]);
          acc[g] = fma(x2, static_cast<double>(w.z), acc[g]);
          acc[g] = fma(x3, static_cast<double>(w.w), acc[g]);
        }
      }
    }
    for (int i = d128 + lane; i < d; i += 32) {
      const double xv = __uint_as_float(static_cast<uint32_t>(__ldg(x_row + i)) << 16);
#pragma unroll
      for (int g = 0; g < 4; ++g)
        if (g < ng)
          acc[g] = fma(xv, static_cast<double>(__ldg(W_r + static_cast<size_t>(ex[g]) * d + i)),
                       acc[g]);
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g < ng) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[g] += __shfl_xor_sync(full, acc[g], off);
        const double s = acc[g] + static_cast<double>(__ldg(b_r + ex[g]));
        const int len = topk_group_len(L, pos[g]);
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int q = 32 * sl + lane;
          if (q >= pos[g] && q < pos[g] + len) val[sl] = s;
        }
      }
    }
  }
}

// Step 3: final order (fp64 values where refined), softmax over the k
// winners, stores of their experts and weights.
__device__ __forceinline__ void topk_emit(const TopkList& L, const double (&val)[2], int k,
                                          int lane, int32_t* __restrict__ idx_out,
                                          float* __restrict__ w_out) {
  const unsigned full = 0xFFFFFFFFu;
  const int m = L.m;
  int my_idx;
  double my_val, top;
  if (L.refine_m == 0) {
    my_idx = L.cidx[0];
    my_val = static_cast<double>(L.cval[0]);
    top = static_cast<double>(__shfl_sync(full, L.cval[0], 0));
  } else {
    uint32_t ctaken = 0;
    if (lane >= m) ctaken |= 1u;
    if (32 + lane >= m) ctaken |= 2u;
    const uint64_t vk[2] = {value_order_key(val[0]), value_order_key(val[1])};
    my_idx = 0;
    my_val = 0.0;
    top = 0.0;
    for (int r = 0; r < k; ++r) {
      uint64_t bk = 0;
      double bv = 0.0;
      int bi = 0x7FFFFFFF, bs = -1;
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        if (ctaken & (1u << s2)) continue;
        if (bi == 0x7FFFFFFF || vk[s2] > bk || (vk[s2] == bk && L.cidx[s2] < bi)) {
          bk = vk[s2];
          bv = val[s2];
          bi = L.cidx[s2];
          bs = s2;
        }
      }
      int bl = bs >= 0 ? lane : -1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const uint64_t ok = __shfl_xor_sync(full, bk, off);
        const double ov = __shfl_xor_sync(full, bv, off);
        const int oi = __shfl_xor_sync(full, bi, off);
        const int ol = __shfl_xor_sync(full, bl, off);
        const int os = __shfl_xor_sync(full, bs, off);
        const bool better = (bi == 0x7FFFFFFF) ||
                            (oi != 0x7FFFFFFF && (ok > bk || (ok == bk && oi < bi)));
        if (better) {
          bk = ok;
          bv = ov;
          bi = oi;
          bl = ol;
          bs = os;
        }
      }
      if (bl == lane && bs >= 0) ctaken |= 1u << bs;
      if (r == 0) top = bv;
      if (lane == r) {
        my_idx = bi;
        my_val = bv;
      }
    }
  }
  const float ex = (lane < k) ? expf(static_cast<float>(my_val - top)) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(full, sum, off);
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = ex / sum;
  }
}

}  // namespace moe
