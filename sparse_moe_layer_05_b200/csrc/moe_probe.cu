// moe_probe.cu -- tensor-core rate probe: the UMMA throughput the grouped
// GEMMs can count on, measured on the device the library runs on.
//
// Each CTA (one per SM) has one thread that issues back-to-back UMMAs from
// shared-memory tiles (M = 128, K = 16 for bf16, K = 32 for the block-scaled
// E2M1 x E4M3 kind) into one TMEM accumulator, `per_commit` UMMAs per
// tcgen05.commit, keeping at most eight commits in flight. The operands are
// zero (timing only). The result is MACs per SM clock, from clock64 over the
// issuing loop plus the drain of the last commits, slowest SM. Every wait is
// bounded (the shared mbarrier helper): a probe that cannot complete reports
// a timeout instead of hanging.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {
namespace {

constexpr int kProbeIters = 1024;          // UMMA groups per CTA
constexpr int kProbeSmem = 16384 + 32768 + 1024 + 1024;

template <int KIND>
__global__ void __launch_bounds__(128, 1)
    tensor_rate_probe_kernel(int N, int per_commit, unsigned long long* cycles, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) unsigned long long bars[9];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const uint32_t A = smem_u32(sm), B = A + 16384, SF = A + 49152;
  for (int i = threadIdx.x; i < (49152 + 1024) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 9; ++i) mbar_init(smem_u32(&bars[i]), 1);
    s_abort = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(&s_tmem), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem;
  if (threadIdx.x == 0) {
    const uint32_t sfa = tb + 256, sfb = tb + 264;
    bool ok = true;
    int ncommit = 0;
    const unsigned long long t0 = clock64();
    for (int g = 0; g < kProbeIters && ok; ++g) {
      if (ncommit >= 8) {
        const int j = ncommit - 8;
        ok = mbar_wait(smem_u32(&bars[j & 7]), (j >> 3) & 1, &s_abort, status);
        if (!ok) break;
      }
      tc_fence_after();
      for (int u = 0; u < per_commit; u += 4) {
        if (KIND == 1) {
          tmem_cp_32x128b_x4(sfa, sdesc_k_noswizzle(SF, 128));
          tmem_cp_32x128b_x4(sfb, sdesc_k_noswizzle(SF + 512, 128));
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk)
            umma_mxf8f6f4(tb, sdesc_k_sw128(A + kk * 32), sdesc_k_sw128(B + kk * 32),
                          idesc_mx_e2m1_e4m3(128, N, kk, kk), sfa | (kk << 30), sfb | (kk << 30), 1u);
        } else {
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk)
            umma_bf16(tb, sdesc_k_sw128(A + kk * 32), sdesc_k_sw128(B + kk * 32),
                      idesc_bf16_f32(128, N), 1u);
        }
      }
      umma_commit(smem_u32(&bars[ncommit & 7]));
      ++ncommit;
    }
    for (int j = ncommit > 8 ? ncommit - 8 : 0; j < ncommit && ok; ++j)
      ok = mbar_wait(smem_u32(&bars[j & 7]), (j >> 3) & 1, &s_abort, status);
    const unsigned long long t1 = clock64();
    cycles[blockIdx.x] = ok ? t1 - t0 : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tb, 512);
}

}  // namespace

cudaError_t launch_tensor_rate_probe(int kind, int N, int per_commit, int num_sms,
                                     unsigned long long* cycles, int* status, cudaStream_t st) {
  static bool attr_set[2][64] = {{false}};
  int dev = 0;
  cudaGetDevice(&dev);
  const int kd = kind == 1 ? 1 : 0;
  if (dev >= 0 && dev < 64 && !attr_set[kd][dev]) {
    cudaError_t e = kd ? cudaFuncSetAttribute(tensor_rate_probe_kernel<1>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem)
                       : cudaFuncSetAttribute(tensor_rate_probe_kernel<0>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
    if (e != cudaSuccess) return e;
    attr_set[kd][dev] = true;
  }
  if (kd)
    tensor_rate_probe_kernel<1><<<num_sms, 128, kProbeSmem, st>>>(N, per_commit, cycles, status);
  else
    tensor_rate_probe_kernel<0><<<num_sms, 128, kProbeSmem, st>>>(N, per_commit, cycles, status);
  return cudaGetLastError();
}

int tensor_rate_probe_iters() { return kProbeIters; }

}  // namespace moe
