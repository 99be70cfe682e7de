// moe_topk.cuh -- top-k over one token's expert logits and the softmax over
// the selected set, one warp per token ("llm-surgery-dark-arts-gpt-oss-40b-
// 64a8-init", section 2, "Proof": i in top-k(s), p_i = exp(s_i) / sum over
// the selected set). Used by the router kernels of moe_routing.cu and
// moe_router_tc.cu.
#pragma once

#include <float.h>
#include <stdint.h>

namespace moe {

// One warp per token. Lane l holds the logits of experts l, l+32, ...; k rounds
// of a warp arg-max on (logit descending, index ascending). Lane j keeps the
// j-th winner; the softmax runs over the k winners only.
//
// The arg-max compares 32-bit keys that order the logits totally: a float's
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

__device__ __forceinline__ void topk_softmax_warp(const float* s, int E, int k, int lane,
                                                  int32_t* __restrict__ idx_out,
                                                  float* __restrict__ w_out) {
  float v[8];
  uint32_t key[8];
  uint32_t taken = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    v[j] = (e < E) ? s[e] : -FLT_MAX;
    key[j] = logit_order_key(v[j]);
    if (e >= E) taken |= 1u << j;
  }
  int my_idx = 0;
  float my_val = 0.f, top = 0.f;
  for (int r = 0; r < k; ++r) {
    uint32_t bk = 0;
    float bv = 0.f;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (taken & (1u << j)) continue;
      const int e = lane + 32 * j;
      if (bi == 0x7FFFFFFF || key[j] > bk || (key[j] == bk && e < bi)) {
        bk = key[j];
        bv = v[j];
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint32_t ok = __shfl_xor_sync(0xFFFFFFFFu, bk, off);
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
      const bool better = (bi == 0x7FFFFFFF) ||
                          (oi != 0x7FFFFFFF && (ok > bk || (ok == bk && oi < bi)));
      if (better) {
        bk = ok;
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (r == 0) top = bv;
    if (lane == r) {
      my_idx = bi;
      my_val = bv;
    }
  }
  const float ex = (lane < k) ? expf(my_val - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = ex / sum;
  }
}

}  // namespace moe
