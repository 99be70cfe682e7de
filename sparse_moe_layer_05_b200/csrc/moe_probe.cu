// moe_probe.cu -- tensor-core rate probe: the UMMA throughput the grouped
// GEMMs can count on, measured on the device it runs on. Built as a library
// of its own (libmoe_b200_probe.so, include/moe_b200_probe.h): it is
// measurement tooling for the benchmark, not part of the layer's interface.
//
// Each CTA (one per SM) has one thread that issues back-to-back UMMAs from
// shared-memory tiles (M = 128; K = 16 for bf16, K = 32 for the block-scaled
// E2M1 x E4M3 kind, K = 64 for the block-scaled E2M1 x E2M1 kind::mxf4) into
// one TMEM accumulator, `per_commit` UMMAs per
// tcgen05.commit, keeping at most eight commits in flight. The operands are
// zero (timing only). The result is MACs per SM clock, from clock64 over the
// issuing loop plus the drain of the last commits, slowest SM. Every wait is
// bounded (the shared mbarrier helper): a probe that cannot complete reports
// a timeout instead of hanging.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_b200_probe.h"
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
        } else if (KIND == 2) {
          // four K = 64 steps: two scale bytes per row and step, two steps per
          // 32-bit scale word, so two scale atoms (4 TMEM columns each) per
          // operand for the 256 K of the four steps
          tmem_cp_32x128b_x4(sfa, sdesc_k_noswizzle(SF, 128));
          tmem_cp_32x128b_x4(sfa + 4, sdesc_k_noswizzle(SF, 128));
          tmem_cp_32x128b_x4(sfb, sdesc_k_noswizzle(SF + 512, 128));
          tmem_cp_32x128b_x4(sfb + 4, sdesc_k_noswizzle(SF + 512, 128));
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk) {
            const uint32_t id = (kk & 1) * 2;
            umma_mxf4(tb, sdesc_k_sw128(A + kk * 32), sdesc_k_sw128(B + kk * 32),
                      idesc_mxf4(128, N, id, id), (sfa + 4 * (kk >> 1)) | (id << 30),
                      (sfb + 4 * (kk >> 1)) | (id << 30), 1u);
          }
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

cudaError_t launch_tensor_rate_probe(int kind, int N, int per_commit, int num_sms,
                                     unsigned long long* cycles, int* status, cudaStream_t st) {
  static bool attr_set[3][64] = {{false}};
  int dev = 0;
  cudaGetDevice(&dev);
  const int kd = kind;
  void (*fn)(int, int, unsigned long long*, int*) =
      kd == 2 ? tensor_rate_probe_kernel<2>
              : (kd == 1 ? tensor_rate_probe_kernel<1> : tensor_rate_probe_kernel<0>);
  if (dev >= 0 && dev < 64 && !attr_set[kd][dev]) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
    if (e != cudaSuccess) return e;
    attr_set[kd][dev] = true;
  }
  fn<<<num_sms, 128, kProbeSmem, st>>>(N, per_commit, cycles, status);
  return cudaGetLastError();
}

}  // namespace
}  // namespace moe

namespace {
// what the last failing CUDA call of this thread returned (moe_probe_error_string)
thread_local const char* g_probe_err = "no error";
thread_local const char* g_probe_where = "";

bool probe_cuda(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return true;
  g_probe_err = cudaGetErrorString(e);
  g_probe_where = where;
  cudaGetLastError();
  return false;
}
}  // namespace

extern "C" {

const char* moe_probe_error_string(void) { return g_probe_err; }
const char* moe_probe_error_site(void) { return g_probe_where; }

moe_status moe_probe_tensor_rate(int kind, int N, int per_commit, double* mac_per_clk_sm,
                                 void* stream) {
  if (!mac_per_clk_sm || kind < 0 || kind > 2 || N < 16 || N > 256 || N % 16 ||
      per_commit < 4 || per_commit > 64 || per_commit % 4)
    return MOE_ERR_INVALID_ARG;
  int dev = -1, major = 0, minor = 0, num_sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  if (major != 10 || minor != 0) return MOE_ERR_NO_DEVICE;
  g_probe_err = "no error";
  g_probe_where = "";
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned long long* d_cycles = nullptr;
  const size_t bytes = static_cast<size_t>(num_sms) * 8 + 16;
  if (!probe_cuda(cudaMalloc(&d_cycles, bytes), "cudaMalloc")) return MOE_ERR_CUDA;
  int* d_status = reinterpret_cast<int*>(d_cycles + num_sms);
  moe_status r = MOE_OK;
  if (!probe_cuda(cudaMemsetAsync(d_cycles, 0, bytes, st), "cudaMemsetAsync") ||
      !probe_cuda(moe::launch_tensor_rate_probe(kind, N, per_commit, num_sms, d_cycles, d_status,
                                                st),
                  "probe launch") ||
      !probe_cuda(cudaStreamSynchronize(st), "cudaStreamSynchronize"))
    r = MOE_ERR_CUDA;
  unsigned long long* h = new unsigned long long[num_sms + 2];
  if (r == MOE_OK && !probe_cuda(cudaMemcpy(h, d_cycles, bytes, cudaMemcpyDeviceToHost), "cudaMemcpy"))
    r = MOE_ERR_CUDA;
  if (r == MOE_OK) {
    const int status = *reinterpret_cast<int*>(h + num_sms);
    unsigned long long worst = 0;
    for (int i = 0; i < num_sms; ++i) worst = h[i] > worst ? h[i] : worst;
    if (status || worst == 0) {
      r = status ? static_cast<moe_status>(status) : MOE_ERR_CUDA;
    } else {
      const double k = kind == 2 ? 64.0 : (kind == 1 ? 32.0 : 16.0);
      const double macs = static_cast<double>(moe::kProbeIters) * per_commit * 128.0 * N * k;
      *mac_per_clk_sm = macs / static_cast<double>(worst);
    }
  }
  delete[] h;
  cudaFree(d_cycles);
  return r;
}

}  // extern "C"
