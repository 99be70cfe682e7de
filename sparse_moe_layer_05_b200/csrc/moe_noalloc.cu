// moe_noalloc.cu -- moe_route_noalloc: the router + permutation entry point
// for callers that cannot allocate device memory.
//
// Some callers of this library are handed only their inputs, their outputs
// and a stream: plugin hooks of inference runtimes, or code on a serving
// thread that must not call the device allocator (cudaMalloc can synchronise
// the device and can fail under memory pressure, and such callers have no
// workspace to offer). This file gives them one entry point whose scratch
// memory lives in a fixed-size array in device global memory that the
// library owns; it calls no allocator.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds it, kNoAllocScratchBytes of device memory, until the process
// exits. Host code cannot use the array's name as a device address, so every
// call looks the address up with cudaGetSymbolAddress on the device that is
// current for the call. Nothing is cached on the host: an address stays
// right after a new primary context or a cudaDeviceReset, and host threads
// making their first calls at the same time share no state here. The lookup
// is a cheap runtime query; the first one on a device also loads the
// library's module there, so make a first call before any stream capture.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace {

// Largest T * E accepted: the fp32 router logits take 4 bytes per
// (token, expert). The router's split weights (three bf16 terms per weight,
// a norm and a fingerprint per expert row) take at most
// 3 * 256 * 16384 * 2 + 256 * 12 bytes, its per-token ||x||^2 at most
// 4 * 2^20 bytes; the rest of the scratch is small tables.
constexpr size_t kNoAllocMaxTE = size_t(1) << 20;
constexpr size_t kNoAllocRouterBytes = size_t(3) * 256 * 16384 * 2 + 4096 + kNoAllocMaxTE * 4;
constexpr size_t kNoAllocScratchBytes =
    kNoAllocMaxTE * 4 + kNoAllocRouterBytes + (size_t(64) << 10);

__device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct ScratchLayout {
  size_t status, logits, router, mprefix, chunk_hist, chunk_base, total;
};

ScratchLayout scratch_layout(int E, int T, int d) {
  const size_t nb = static_cast<size_t>(moe::perm_chunks(T));
  ScratchLayout L;
  size_t off = 0;
  L.status = off;
  off = round256(off + 16);
  L.mprefix = off;
  off = round256(off + static_cast<size_t>(E + 1) * 4);
  L.chunk_hist = off;
  off = round256(off + nb * E * 4);
  L.chunk_base = off;
  off = round256(off + nb * E * 4);
  L.logits = off;
  off = round256(off + static_cast<size_t>(T) * E * 4);
  L.router = off;
  off = round256(off + moe::router_tc_scratch_bytes(E, d, T));
  L.total = off;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Device address of the scratch array on the current device, looked up on
// every call (see the file comment).
moe_status scratch_base(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *out = p;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_route_noalloc(const void* x_dev, const float* W_r_dev, const float* b_r_dev, int E,
                             int k, int T, int d, int32_t* topk_idx_dev, float* topk_w_dev,
                             int32_t* counts_dev, int32_t* offsets_dev, int32_t* perm_dev,
                             void* stream) {
  if (!x_dev || !W_r_dev || !b_r_dev || !topk_idx_dev || !topk_w_dev || !counts_dev ||
      !offsets_dev || !perm_dev)
    return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > 256 || k < 1 || k > E || k > 32 || T < 0 || d < 32 || d > 16384 || d % 32)
    return MOE_ERR_UNSUPPORTED;
  if (static_cast<size_t>(T) * static_cast<size_t>(E) > kNoAllocMaxTE) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x_dev) || !aligned16(W_r_dev) || !aligned16(b_r_dev)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const ScratchLayout L = scratch_layout(E, T, d);
  if (L.total > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* base = nullptr;
  moe_status s = scratch_base(&base);
  if (s != MOE_OK) return s;
  unsigned char* sb = static_cast<unsigned char*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = reinterpret_cast<int*>(sb + L.status);
  float* logits = reinterpret_cast<float*>(sb + L.logits);
  int32_t* mprefix = reinterpret_cast<int32_t*>(sb + L.mprefix);
  int32_t* chunk_hist = reinterpret_cast<int32_t*>(sb + L.chunk_hist);
  int32_t* chunk_base = reinterpret_cast<int32_t*>(sb + L.chunk_base);
  // Every buffer below is fully written before it is read; the status word
  // is cleared by the first kernel. Batches of at most kPermChunk tokens get
  // their permutation from the router's top-k launch (identical results).
  // The launches are the ones moe_route makes, in the same order and
  // configuration.
  const uint16_t* x = static_cast<const uint16_t*>(x_dev);
  moe::pdl_launches() = false;
  const bool small = T <= moe::kPermChunk;
  bool launched =
      moe::launch_router_tc(x, W_r_dev, b_r_dev, T, E, k, d, sb + L.router, logits, topk_idx_dev,
                            topk_w_dev, status, st, small ? counts_dev : nullptr,
                            small ? offsets_dev : nullptr, small ? mprefix : nullptr,
                            small ? perm_dev : nullptr) == cudaSuccess;
  if (launched && !small) {
    launched =
        moe::launch_perm_hist(topk_idx_dev, T, k, E, chunk_hist, st) == cudaSuccess &&
        moe::launch_perm_scan(chunk_hist, moe::perm_chunks(T), E, counts_dev, offsets_dev,
                              chunk_base, mprefix, st) == cudaSuccess &&
        moe::launch_perm_scatter(topk_idx_dev, T, k, E, chunk_base, perm_dev, nullptr, st) ==
            cudaSuccess;
  }
  moe::pdl_launches() = false;
  if (!launched) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // extern "C"
