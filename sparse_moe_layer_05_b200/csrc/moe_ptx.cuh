// moe_ptx.cuh -- sm_100a building blocks used by the MoE kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM allocation,
// UMMA issue/commit, TMEM loads), shared-memory matrix descriptors, and the
// exact MXFP4 -> bf16 decoder.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device status word values (match moe_status in include/moe_b200.h).
constexpr int kStatusTimeout = 5;

// Wall-clock budget of one bounded wait, in nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Programmatic dependent launch. A kernel launched with programmatic stream
// serialization may start while its predecessor on the stream is still
// running; griddepcontrol.wait blocks until that predecessor has completed and
// its memory is visible (a no-op for kernels launched without it). Every
// kernel of the library executes it before its first global-memory access, so
// by induction all earlier kernels of the stream have completed by then. The
// trigger lets the stream's next kernel be scheduled once every CTA of this
// one has started (its CTAs then wait in griddepcontrol.wait).
__device__ __forceinline__ void pdl_wait_and_trigger() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------- mbarrier ----

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete. Gives up after
// kWaitLimitNs (or as soon as another role raised *abort), records a timeout
// in *status and returns false. Never spins without limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        if (status) atomicExch(status, kStatusTimeout);
        return false;
      }
    }
  }
}

// Same as mbar_try_wait, with acquire semantics at cluster scope (for phases
// completed by arrivals from the peer CTA of a cluster).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity,
                                                  volatile int* abort, int* status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        if (status) atomicExch(status, kStatusTimeout);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------- clusters ----

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Arrive on an mbarrier of another CTA of the cluster (release, cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// Same, relaxed (no release fence at cluster scope). Used only to forward a
// completion this thread has already observed with acquire semantics on a
// local barrier: the data it announces is complete in this CTA's shared
// memory before the arrive is issued.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMA ----

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                            int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// -------------------------------------------------------------- tcgen05 ----

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A (M = 128 rows, one per TMEM lane) is read
// from tensor memory, 8 columns (16 bf16 of K) per instruction.
__device__ __forceinline__ void umma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Registers -> TMEM: 16 consecutive 32-bit columns of this thread's lane,
// then wait until the store has completed.
__device__ __forceinline__ void tmem_st16_sync(uint32_t taddr, const uint4 (&v)[4]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(v[0].x), "r"(v[0].y), "r"(v[0].z), "r"(v[0].w), "r"(v[1].x), "r"(v[1].y), "r"(v[1].z),
      "r"(v[1].w), "r"(v[2].x), "r"(v[2].y), "r"(v[2].z), "r"(v[2].w), "r"(v[3].x), "r"(v[3].y),
      "r"(v[3].z), "r"(v[3].w)
      : "memory");
}

// Registers -> TMEM: 4 consecutive 32-bit columns of this thread's lane; no
// wait (tmem_wait_st completes this warp's stores).
__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint4 v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// CTA-pair UMMA (issued by the even CTA of a cluster pair): A rows 0..127 come
// from this CTA's shared memory and rows 128..255 from the peer's at the same
// offsets; B's N columns are split the same way; each CTA's TMEM receives its
// 128 accumulator rows.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at offset `bar` in both CTAs of the pair when
// every CTA-pair tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// TMEM -> registers. tcgen05.ld completes asynchronously: its destination
// registers may be read only after tcgen05.wait::ld. Each helper issues the
// load(s) and the wait in one asm statement, so no instruction that consumes
// the registers can be scheduled between them.

// Two 32-lane x 8-column loads (columns [ta, ta+8) and [tb, tb+8)), then wait.
__device__ __forceinline__ void tmem_ld8x2_sync(uint32_t ta, uint32_t tb, uint32_t (&a)[8],
                                                uint32_t (&b)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%16];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%8,%9,%10,%11,%12,%13,%14,%15}, [%17];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]),
        "=r"(a[7]), "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]),
        "=r"(b[6]), "=r"(b[7])
      : "r"(ta), "r"(tb)
      : "memory");
}

// One 32-lane x 8-column load, then wait.
__device__ __forceinline__ void tmem_ld8_sync(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
}

// One 32-lane x 16-column load, then wait.
__device__ __forceinline__ void tmem_ld16_sync(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15},"
      " [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored in the
// 128-byte swizzled layout: rows of 128 bytes (64 bf16 along K), groups of 8
// rows 1024 bytes apart. The tile base must be 1024-byte aligned; advancing
// along K inside the 128-byte row is done by adding the byte offset to the
// start address.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);        // start address
  d |= static_cast<uint64_t>(1) << 16;                        // leading offset (unused)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;                // stride between 8-row groups
  d |= static_cast<uint64_t>(1) << 46;                        // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                        // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B (both K-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------- block-scaled (MX) tcgen05 ----

// D[tmem] (+)= sum_k (a_mk 2^(sa_m - 127)) (b_nk 2^(sb_n - 127)) over one
// K = 32 step with .kind::mxf8f6f4: A holds E2M1 values in 8-bit containers
// (the layout the 16U4_ALIGN16B tensor maps write), B holds E4M3 values, both
// K-major in 128-byte swizzled tiles. sa / sb are E8M0 scales read from TMEM:
// lane m (A) or n (B) of column sf + m/32 (n/32) within each 32-lane quarter,
// byte given by bits 30-31 of the scale address (and the matching sf-id field
// of the instruction descriptor).
__device__ __forceinline__ void umma_mxf8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor for umma_mxf8f6f4: A E2M1, B of type btype (0 E4M3,
// 5 E2M1 in 8-bit containers), E8M0 scales, both operands K-major, fp32
// accumulator; sfa_id / sfb_id select the scale byte.
__host__ __device__ constexpr uint32_t idesc_mx_e2m1(int M, int N, uint32_t sfa_id,
                                                    uint32_t sfb_id, uint32_t btype) {
  return (sfb_id << 4) | (5u << 7) | (btype << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (1u << 23) | (static_cast<uint32_t>(M >> 4) << 24) | (sfa_id << 29);
}
__host__ __device__ constexpr uint32_t idesc_mx_e2m1_e4m3(int M, int N, uint32_t sfa_id,
                                                         uint32_t sfb_id) {
  return idesc_mx_e2m1(M, N, sfa_id, sfb_id, 0u);
}

// D[tmem] (+)= A B^T over one K = 64 step with .kind::mxf4: A and B hold
// packed E2M1 values (two per byte, 32 bytes of K per row and step), K-major in
// 128-byte swizzled tiles; every 32 elements of K carry an E8M0 scale
// (.scale_vec::2X: two scale bytes per row and step, bytes sf_id and
// sf_id + 1 of the row's 32-bit TMEM scale word, sf_id 0 or 2).
__device__ __forceinline__ void umma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor for umma_mxf4: A and B E2M1 (the .kind::mxf4 type
// code 1), E8M0 scales, both K-major, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, uint32_t sfa_id, uint32_t sfb_id) {
  return (sfb_id << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (1u << 23) | (static_cast<uint32_t>(M >> 4) << 24) | (sfa_id << 29);
}

// Shared memory -> TMEM: 32 lanes x 128 bits, replicated into all four 32-lane
// quarters of the columns [taddr, taddr + 4).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Descriptor of an unswizzled K-major shared-memory tile: rows of 16 bytes,
// 8-row core matrices `sbo` bytes apart (the tcgen05.cp source format).
__device__ __forceinline__ uint64_t sdesc_k_noswizzle(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(16 >> 4) << 16;
  d |= static_cast<uint64_t>(sbo >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Contiguous global -> shared copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned), completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Two fp32 -> two E4M3 (round to nearest even, saturating to +-448): the
// result holds e4m3(a) in bits 0-7 and e4m3(b) in bits 8-15.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// fp32 -> E2M1 code (round to nearest even, saturating to +-6), in bits 0-3.
__device__ __forceinline__ uint32_t f32_to_e2m1(float a) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b16 %0, {t, 0};\n\t}"
      : "=h"(r)
      : "f"(0.f), "f"(a));
  return static_cast<uint32_t>(r) & 0xFu;
}

// Two fp32 -> two E2M1 codes in one byte: e2m1(a) in bits 0-3, e2m1(b) in 4-7.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float a, float b) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b16 %0, {t, 0};\n\t}"
      : "=h"(r)
      : "f"(b), "f"(a));
  return static_cast<uint32_t>(r) & 0xFFu;
}

// Two E4M3 (bits 0-7, 8-15) -> two fp32 (exact).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t v) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(v)));
  uint16_t lo = static_cast<uint16_t>(h2 & 0xFFFFu), hi = static_cast<uint16_t>(h2 >> 16);
  float fa, fb;
  asm("cvt.f32.f16 %0, %1;" : "=f"(fa) : "h"(lo));
  asm("cvt.f32.f16 %0, %1;" : "=f"(fb) : "h"(hi));
  return make_float2(fa, fb);
}

// ------------------------------------------------------------ MXFP4 ----

// bf16x2 product; exact whenever the product is representable.
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Order of the elements inside every 8-element chunk of a GEMM operand row:
// position p holds element kPerm8[p]. Both operands of the grouped GEMMs (the
// activation rows and the decoded weight rows) use it, so each dot product is
// unchanged; it lets the decoder emit bf16 pairs (j, j+4) straight from the
// packed nibbles.
//   kPerm8 = {0, 4, 1, 5, 2, 6, 3, 7}

// 8 bf16 in natural order (4 words) -> chunk order.
__device__ __forceinline__ uint4 chunk8_to_perm(uint4 v) {
  return make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632),
                    __byte_perm(v.y, v.w, 0x5410), __byte_perm(v.y, v.w, 0x7632));
}

// 8 bf16 in chunk order -> natural order.
__device__ __forceinline__ uint4 chunk8_from_perm(uint4 v) {
  return make_uint4(__byte_perm(v.x, v.y, 0x5410), __byte_perm(v.z, v.w, 0x5410),
                    __byte_perm(v.x, v.y, 0x7632), __byte_perm(v.z, v.w, 0x7632));
}

// Decode 32 E2M1 codes (16 bytes; byte b holds element 2b in its low nibble)
// sharing the E8M0 scale byte S into 32 bf16 values: four 16-byte chunks of
// 8 elements, each chunk in kPerm8 order.
//
// An E2M1 code s|e1 e0|m placed in bf16 bits as s<<15 | (e1 e0 m)<<6 is the
// bf16 number whose value is exactly 2^-126 times the E2M1 value, for the
// normal codes and the subnormal alike. Multiplying by 2^(S-1) then yields
// e2m1 * 2^(S-127) exactly (one product for S <= 128, two for larger S,
// NaN for S = 255). Nibbles j and j+4 of a code word sit 16 bits apart, so
// one shift and mask place both in their bf16 halves.
__device__ __forceinline__ void mxfp4x32_to_bf16(uint4 q, uint32_t S, uint4 (&out)[4]) {
  uint32_t m1, m2 = 0;
  bool two = false;
  if (S == 255u) {
    m1 = 0x7FC07FC0u;  // NaN
  } else if (S <= 128u) {
    const uint32_t h = (S - 1u + 127u) << 7;   // 2^(S-1); S = 0 gives 2^-1
    m1 = h | (h << 16);
  } else {
    m1 = 0x7F007F00u;                        // 2^127
    const uint32_t h = (S - 128u + 127u) << 7; // 2^(S-128)
    m2 = h | (h << 16);
    two = true;
  }
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  uint32_t r[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t x = w[i];
    // word j holds (element j, element j+4) of this 8-code word
    const uint32_t b0 = ((x << 6) & 0x01C001C0u) | ((x << 12) & 0x80008000u);
    const uint32_t b1 = ((x << 2) & 0x01C001C0u) | ((x << 8) & 0x80008000u);
    const uint32_t b2 = ((x >> 2) & 0x01C001C0u) | ((x << 4) & 0x80008000u);
    const uint32_t b3 = ((x >> 6) & 0x01C001C0u) | (x & 0x80008000u);
    uint32_t v0 = bf16x2_mul(b0, m1), v1 = bf16x2_mul(b1, m1);
    uint32_t v2 = bf16x2_mul(b2, m1), v3 = bf16x2_mul(b3, m1);
    if (two) {
      v0 = bf16x2_mul(v0, m2);
      v1 = bf16x2_mul(v1, m2);
      v2 = bf16x2_mul(v2, m2);
      v3 = bf16x2_mul(v3, m2);
    }
    r[4 * i + 0] = v0;
    r[4 * i + 1] = v1;
    r[4 * i + 2] = v2;
    r[4 * i + 3] = v3;
  }
  out[0] = make_uint4(r[0], r[1], r[2], r[3]);
  out[1] = make_uint4(r[4], r[5], r[6], r[7]);
  out[2] = make_uint4(r[8], r[9], r[10], r[11]);
  out[3] = make_uint4(r[12], r[13], r[14], r[15]);
}

}  // namespace moe
