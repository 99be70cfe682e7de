// moe_perm_small.cuh -- the stable expert permutation of at most kPermChunk
// tokens by one block of 256 threads: per-warp histograms, a serial scan
// over the experts, and the stable scatter with __match_any_sync ranks in
// pair order; writes counts, offsets, the M-tile prefix and perm exactly as
// the three-launch permutation of moe_routing.cu does. Used by
// perm_small_kernel (moe_routing.cu) and by the last block of the top-k
// kernel (moe_router_tc.cu).
#pragma once

#include <stdint.h>

#include "moe_internal.h"

namespace moe {

struct PermSmallSmem {
  int wbase[8][256];
  int cnt[256];
  int mt[256];
};

// topk_idx is read with ld.global.cg: in the top-k kernel other blocks wrote
// it in the same launch.
__device__ __forceinline__ void perm_small_block(const int32_t* topk_idx, int T, int k, int E,
                                                 int32_t* counts, int32_t* offsets,
                                                 int32_t* mtile_prefix, int32_t* perm,
                                                 PermSmallSmem& sm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 8 * 256; i += blockDim.x) (&sm.wbase[0][0])[i] = 0;
  __syncthreads();
  const int64_t qc1 = (int64_t)min(T, kPermChunk) * k;
  const int64_t seg = (int64_t)(kPermChunk / 8) * k;
  const int64_t q0 = warp * seg;
  const int64_t q1 = min(qc1, q0 + seg);
  for (int64_t q = q0 + lane; q < q1; q += 32) atomicAdd(&sm.wbase[warp][__ldcg(topk_idx + q)], 1);
  __syncthreads();
  const int e = threadIdx.x;
  int total = 0;
  if (e < E)
    for (int w = 0; w < 8; ++w) total += sm.wbase[w][e];
  sm.cnt[e] = (e < E) ? total : 0;
  sm.mt[e] = (e < E) ? (total + kTileM - 1) / kTileM : 0;
  __syncthreads();
  if (e == 0) {  // E <= 256: a serial scan is cheap and plainly ordered
    int a = 0, m = 0;
    for (int i = 0; i < E; ++i) {
      const int c = sm.cnt[i], mt = sm.mt[i];
      sm.cnt[i] = a;
      sm.mt[i] = m;
      a += c;
      m += mt;
    }
    offsets[E] = a;
    mtile_prefix[E] = m;
  }
  __syncthreads();
  if (e < E) {
    offsets[e] = sm.cnt[e];
    mtile_prefix[e] = sm.mt[e];
    if (counts) counts[e] = total;
    int run = sm.cnt[e];
    for (int w = 0; w < 8; ++w) {
      const int c = sm.wbase[w][e];
      sm.wbase[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  for (int64_t qb = q0; qb < q1; qb += 32) {
    const int64_t q = qb + lane;
    const bool valid = q < q1;
    const int ex = valid ? __ldcg(topk_idx + q) : -1 - lane;
    const uint32_t m = __match_any_sync(0xFFFFFFFFu, ex);
    const int rank = __popc(m & lt);
    int pos = 0;
    if (valid) pos = sm.wbase[warp][ex] + rank;
    __syncwarp();
    if (valid && lane == __ffs(m) - 1) sm.wbase[warp][ex] += __popc(m);
    __syncwarp();
    if (valid) perm[pos] = (int32_t)q;
  }
}

}  // namespace moe
