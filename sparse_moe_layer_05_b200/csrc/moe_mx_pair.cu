// moe_mx_pair.cu -- CTA-pair block-scaled expert GEMMs for experts with many
// routed rows (prefill): tcgen05.mma.cta_group::2.kind::mxf8f6f4 with M = 256.
//
//   gate/up:  H[r, j] = silu(x_r . Wgate[e][j] + bg[e][j]) * (x_r . Wup[e][j] + bu[e][j])
//   down:     Yw[pair(r), m] = p(pair(r)) * (H[r] . Wdown[e][m] + bd[e][m])
//
// Field guide "gpt-oss 20B", "03 Sparse Mixture of Experts" (SwiGLU experts,
// weighted sum); "gpt-oss-20b and gpt-oss-120b", "Four-bit expert weights"
// (E2M1 codes with one power-of-two scale per 32 weights).
//
// Operands. A is the expert's routed token rows (UMMA M = 256: 128 rows in
// each CTA of the pair), B the expert's weight rows (E2M1 codes that TMA widens
// to 8-bit containers; N = 2 NH, NH rows in each CTA). The tensor core applies
// both E8M0 scale sets. With bf16-precision activations each token row comes as
// two E4M3 terms (hi, lo; the split is exact for every element of at least
// 2^-13 of its group's max) and each K step issues two UMMAs into the same
// accumulator, one per term, over the same weight tile: the accumulator holds
// x . w itself. The quantised modes (one E4M3 or E2M1 term) issue one.
//
// Tiles. 256 token rows x N weight rows, 128 K per shared-memory stage.
//   gate/up: NH = 96: the even CTA holds gate rows j0..j0+95, the odd CTA the
//            matching up rows, so accumulator column c (gate) and 96 + c (up)
//            of a token's TMEM lane meet in one thread, and a tile's 96 H
//            columns are three whole MX groups of 32 (the epilogue converts H
//            for the down GEMM per group).
//   down:    NH = 112 (120 for kind::mxf4): output columns n0..n0+N-1.
// Token rows live in a padded layout (each expert's rows start at a multiple
// of 128), so each CTA's half tile is one contiguous block of rows and its
// scale block one contiguous run of bytes. A tile covers 256 rows of one
// expert; when the expert's rows end inside the even CTA's half, the odd CTA
// loads no token rows (its accumulator rows are never stored).
//
// Scale factors in tensor memory. Each CTA holds the A scales of its own 128
// rows (one 512-byte atom per term: row m's four K-step bytes in lane m % 32
// of column m / 32, the same in all four lane quarters) and the B scales of
// all N columns (two atoms), at the same TMEM columns in both CTAs. For the
// 8-bit kinds each pipeline stage has its own slot of scale columns, which
// four builder warps (one per TMEM lane quarter) fill with tcgen05.st while
// the stage's operands arrive, so that the issuing thread issues only UMMAs
// and commits (a tcgen05.cp costs that thread about as long as a UMMA). For
// kind::mxf4 (six atoms per stage: the slots would not fit beside the two
// accumulators) the atoms are staged in shared memory and the issuing thread
// copies them with tcgen05.cp.cta_group::2 before each stage's UMMAs.
// The gate/up builders form the weight atoms from the tile's scale rows,
// staged in shared memory per tile; the down GEMM's weight atoms are laid
// out in global memory beforehand (pair_weight_atoms_kernel, one 1 KB block
// per tile and k-block) and arrive with the stage, which leaves the down
// GEMM the shared memory for a fourth stage.
//
// Roles (448 threads per CTA; 384 for kind::mxf4):
//   warp 0   TMA producer: token rows (A) and their scale block, weight codes
//            (B); the tile's weight-scale rows into a double buffer
//   warp 1   TMEM allocation; in the even CTA the UMMA issuer, in the odd CTA
//            the relay of "stage full" to the even CTA's issuer
//   warps 2, 3, 12, 13  scale builders, TMEM lane quarters 2, 3, 0, 1: the
//            stage's token scale atoms and the tile's weight scales -> the
//            stage's slot (kind::mxf4: warp 2 alone, B atoms into shared
//            memory)
//   warps 4-11 epilogue: warp w reads TMEM lane quarter w % 4 (one token row
//            per thread); warps 4-7 and 8-11 take alternate column groups
// Every wait is bounded (moe_ptx.cuh): a stuck pipeline records a timeout in
// the status word and the kernel exits.
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {
namespace {

constexpr int kMaxE = 256;
enum PairEpi { PAIR_SWIGLU = 0, PAIR_DOWN = 1 };

// Byte of the scale of row (or column) c, K step kk, in a block of 512-byte
// atoms: word c / 32 of lane c % 32, four words per lane per atom.
__host__ __device__ __forceinline__ int atom_offset(int c, int kk) {
  const int w = c >> 5;
  return (w >> 2) * 512 + (c & 31) * 16 + (w & 3) * 4 + kk;
}

// Groups of 32 along K -> (k-block, K step) with the tail rule of the
// block-scaled path: the last k-block of a K that is 64 mod 128 is [K-128, K).
__host__ __device__ __forceinline__ void pair_group_to_kblock(int g, int G, int KB, int& kb,
                                                              int& kk) {
  if ((G % 4) == 0 || g < 4 * (KB - 1)) {
    kb = g >> 2;
    kk = g & 3;
  } else {
    kb = KB - 1;
    kk = g - (G - 4);
  }
}

constexpr int kPairSmemBudget = 232448 - 1024;   // opt-in maximum less alignment slack

template <int EPI, int ACT>
struct PairCfg {
  // kind::mxf4 (ACT_F4): both operands stay packed (two E2M1 per byte) in
  // shared memory, so a 128-byte row holds 256 elements of K, and each UMMA
  // (K = 64) takes two scale bytes per row: two scale words per k-block
  static constexpr bool F4 = ACT == ACT_F4;
  static constexpr int KBK = F4 ? 256 : 128;              // K elements per stage
  static constexpr int TERMS = ACT == ACT_HILO ? 2 : 1;
  static constexpr int MT = 128;                          // token rows per CTA
  // scale atoms reach TMEM by tcgen05.st into per-stage slots (8-bit kinds)
  // or by tcgen05.cp from shared memory (kind::mxf4)
  static constexpr bool SFST = !F4;
  // down GEMM, 8-bit kinds: weight atoms pre-built in global memory, loaded
  // with each stage (no tile-scale buffers)
  static constexpr bool SFBG = EPI == PAIR_DOWN && SFST;
  // weight rows per CTA; down: two accumulators of N = 224 leave 64 TMEM
  // columns for the scale slots
  static constexpr int NH = EPI == PAIR_SWIGLU ? 96 : (SFST ? 112 : 120);
  static constexpr int N = 2 * NH;                        // UMMA N
  static constexpr int A_PLANE = MT * 128;                // one term: 128-byte rows
  static constexpr int A_BYTES = TERMS * A_PLANE;
  static constexpr int A_TX = ACT == ACT_E2M1 ? MT * 64 : A_BYTES;
  static constexpr int B_BYTES = NH * 128;
  static constexpr int B_TX = F4 ? B_BYTES : NH * 64;     // packed code bytes
  static constexpr int SFA_BYTES = F4 ? 1024 : 512 * TERMS;
  static constexpr int SFB_BYTES = F4 ? 2048 : 1024;      // N <= 256: 2 atoms per word
  static constexpr int OFF_B = A_BYTES;
  static constexpr int OFF_SFA = OFF_B + B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + SFA_BYTES;
  static constexpr int STAGE_BYTES =
      (OFF_SFB + ((SFST && !SFBG) ? 0 : SFB_BYTES) + 1023) / 1024 * 1024;
  static constexpr int TS_BYTES = N * (kMxMaxK / 32);     // a tile's weight-scale rows
  static constexpr int TS_BUFS = SFBG ? 0 : 2;
  static constexpr int FIXED = TS_BUFS * TS_BYTES + 3 * (kMaxE + 1) * 4 + 512;
  static constexpr int STAGES_FIT = (kPairSmemBudget - FIXED) / STAGE_BYTES;
  static constexpr int A_ATOMS = SFA_BYTES / 512;
  static constexpr int B_ATOMS = SFB_BYTES / 512;
  static constexpr int SLOT_COLS = 4 * (A_ATOMS + B_ATOMS);   // one stage's scale columns
  static constexpr int TMEM_COLS = 512;
  static constexpr int STAGES_TMEM = SFST ? (TMEM_COLS - 2 * N) / SLOT_COLS : 6;
  static constexpr int STAGES_CAP = STAGES_TMEM < 6 ? STAGES_TMEM : 6;
  static constexpr int STAGES = STAGES_FIT > STAGES_CAP ? STAGES_CAP : STAGES_FIT;
  static constexpr int OFF_TS = STAGES * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_TS + TS_BUFS * TS_BYTES;
  static constexpr int NUM_BARS = 4 * STAGES + 10;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TAB = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = OFF_TAB + 3 * (kMaxE + 1) * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr int EPI_WARPS = 8;                     // two per TMEM lane quarter
  static constexpr int BUILDERS = SFST ? 4 : 1;           // scale-builder warps
  static constexpr int NUM_THREADS = 128 + 32 * EPI_WARPS + (SFST ? 64 : 0);
  static constexpr int ACC_COLS = N;                      // per accumulator buffer
  static constexpr int SF_COL0 = 2 * N;                   // A scales, then B scales
  static constexpr int SFA_COLS = SFA_BYTES / 128;        // 4 TMEM columns per atom
  static constexpr int SFB_COLS = SFB_BYTES / 128;
  static constexpr int TX_FULL = A_TX + B_TX + (SFST ? 0 : SFA_BYTES);   // a stage with token rows
  static constexpr uint32_t ATYPE = ACT == ACT_E2M1 ? 5u : 0u;   // E2M1 or E4M3
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(SF_COL0 + (SFST ? STAGES * SLOT_COLS : SFA_COLS + SFB_COLS) <= TMEM_COLS,
                "TMEM budget");
  static_assert(NUM_BARS * 8 + 16 <= 512, "barrier space");
  static_assert(SMEM_ALLOC <= 232448, "shared memory");
  static_assert(OFF_B % 1024 == 0 && B_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "swizzle");
  static_assert(N % 16 == 0 && N <= 256, "UMMA N");
};

// Instruction descriptor: block-scaled kind::mxf8f6f4, A type atype (tokens),
// B E2M1 (weights), E8M0 scales, K-major operands, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_pair(int M, int N, uint32_t atype, uint32_t sf_id) {
  return (sf_id << 4) | (atype << 7) | (5u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (1u << 23) | (static_cast<uint32_t>(M >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void umma_mx_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// kind::mxf4 on the pair: A and B packed E2M1 (K = 64 per UMMA), two E8M0
// scale bytes per row (bytes sf_id, sf_id + 1 of the row's scale word).
__device__ __forceinline__ void umma_mxf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t sfa_tmem,
                                               uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared memory -> TMEM in both CTAs of the pair (each CTA's atom at the same
// shared-memory offset into its own TMEM), 32 lanes x 128 bits replicated into
// the four lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_x4_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

struct PairArgs {
  const int32_t* offsets;
  int E, K, I;                // K: contraction; I: intermediate size
  int n_out;                  // I (gate/up) or d (down)
  int n_tiles;                // weight tiles per expert
  int rows_per_expert;        // weight rows of an expert in the scale array (2I or d)
  int KB;                     // k-blocks
  const uint8_t* scales;      // [E][rows_per_expert][K/32] E8M0 weight scales
  const uint8_t* sfa;         // token scale blocks [128-row tile][KB][SFA_BYTES]
  const uint8_t* wsfb;        // SFBG: weight atoms [E][n_tiles][KB][SFB_BYTES]
  // gate/up: converted H rows (h_lo: the lo plane of the bf16 split) and
  // their scale blocks (the down GEMM's A operand)
  uint8_t* h_q;
  uint8_t* h_lo;
  uint8_t* h_sfa;
  int h_kb;
  // down: weighted rows
  float* out_f32;
  const int32_t* perm;
  const float* topk_w;
  int* status;
  const float* bias;          // [E][2I] or [E][d], or nullptr
};

__device__ __forceinline__ float silu_p(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int EPI, int ACT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<EPI, ACT>::NUM_THREADS, 1)
    grouped_mx_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmAt,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmBt, const PairArgs args) {
  pdl_wait_and_trigger();
  using C = PairCfg<EPI, ACT>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (S + s); };
  auto bar_accFull = [&](int b) { return bar0 + 8u * (3 * S + b); };
  auto bar_accEmpty = [&](int b) { return bar0 + 8u * (3 * S + 2 + b); };
  auto bar_peerAcc = [&](int b) { return bar0 + 8u * (3 * S + 4 + b); };
  auto bar_tsFull = [&](int b) { return bar0 + 8u * (3 * S + 6 + b); };
  auto bar_tsEmpty = [&](int b) { return bar0 + 8u * (3 * S + 8 + b); };
  auto bar_sfaFull = [&](int s) { return bar0 + 8u * (3 * S + 10 + s); };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* s_off = reinterpret_cast<int*>(smem + C::OFF_TAB);
  int* s_tp = s_off + (kMaxE + 1);   // prefix of tiles per expert
  int* s_tb = s_tp + (kMaxE + 1);    // prefix of 128-row token tiles per expert

  const int E = args.E;
  for (int i = threadIdx.x; i <= E; i += C::NUM_THREADS) s_off[i] = args.offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    int acc = 0, tb = 0;
    for (int e = 0; e < E; ++e) {
      s_tp[e] = acc;
      s_tb[e] = tb;
      const int cnt = s_off[e + 1] - s_off[e];
      acc += (cnt + 255) / 256 * args.n_tiles;
      tb += (cnt + 127) / 128;
    }
    s_tp[E] = acc;
    s_tb[E] = tb;
    for (int s = 0; s < S; ++s) {
      // producer (with the TMA bytes) + builders; in the even CTA also the
      // odd CTA's relay, so that one wait covers both halves of the stage
      mbar_init(bar_full(s), 1 + C::BUILDERS + (rank == 0 ? 1 : 0));
      mbar_init(bar_sfaFull(s), 1);  // the stage's token scale block (8-bit kinds)
      mbar_init(bar_empty(s), 1);    // the issuer's commit, multicast to both CTAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accFull(b), 1);
      mbar_init(bar_accEmpty(b), C::EPI_WARPS * 32);
      mbar_init(bar_peerAcc(b), 1);
      mbar_init(bar_tsFull(b), 1);
      mbar_init(bar_tsEmpty(b), C::BUILDERS);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmBt);
    if (ACT == ACT_E2M1) tma_prefetch_desc(&tmAt);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(misc), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];

  const int total = s_tp[E];
  const int K = args.K;
  const int G = K / 32;
  const int KB = args.KB;
  // K % 64 == 0: a K that is not a multiple of the k-block ends with a block
  // [K - KBK, K) of which only the steps past the previous block are issued
  const bool tail = (K % C::KBK) != 0;
  // K steps in the tail block past the previous block (a step is 32 elements
  // of K, 64 for F4): 2 for the 8-bit kinds, 1..3 for F4
  const int tail_steps = (K % C::KBK) / (C::F4 ? 64 : 32);
  // tile -> expert, weight tile nt, token pair-tile mt (token tiles fastest, so
  // that neighbouring pairs share a weight tile in L2), rows of this CTA's half
  struct Tile {
    int e, nt, mt, rows;   // rows: valid token rows of this CTA's half (0..128)
    int arow;              // first padded token row of this CTA's half
    int ttile;             // its 128-row token tile
  };
  auto decode = [&](int tile, Tile& t) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_tp[mid] <= tile) lo = mid; else hi = mid;
    }
    t.e = lo;
    const int cnt = s_off[t.e + 1] - s_off[t.e];
    const int mpairs = (cnt + 255) / 256;
    const int local = tile - s_tp[t.e];
    t.nt = local / mpairs;
    t.mt = local % mpairs;
    t.rows = min(128, max(0, cnt - t.mt * 256 - rank * 128));
    t.ttile = s_tb[t.e] + 2 * t.mt + rank;
    t.arow = t.ttile * 128;
  };

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0) {
      // a tile's weight-scale rows (this CTA's B columns and the peer's: all N
      // columns' scales are needed in each CTA) into tile-scale buffer it & 1
      auto load_tile_scales = [&](int tile, int itx) -> bool {
        Tile t;
        decode(tile, t);
        const int b = itx & 1;   // (not reached with SFBG)
        if (!mbar_wait(bar_tsEmpty(b), ((itx >> 1) & 1) ^ 1, abort_flag, args.status)) return false;
        const uint32_t ts = sbase + C::OFF_TS + b * C::TS_BYTES;
        const size_t ebase = static_cast<size_t>(t.e) * args.rows_per_expert;
        if (EPI == PAIR_SWIGLU) {
          const int j0 = t.nt * C::NH;
          const uint32_t half = static_cast<uint32_t>(min(C::NH, args.I - j0)) * G;
          mbar_expect_tx(bar_tsFull(b), 2 * half);
          bulk_load(ts, args.scales + (ebase + j0) * G, half, bar_tsFull(b));
          bulk_load(ts + C::NH * G, args.scales + (ebase + args.I + j0) * G, half, bar_tsFull(b));
        } else {
          const int n0 = t.nt * C::N;
          const uint32_t bytes = static_cast<uint32_t>(min(C::N, args.n_out - n0)) * G;
          mbar_expect_tx(bar_tsFull(b), bytes);
          bulk_load(ts, args.scales + (ebase + n0) * G, bytes, bar_tsFull(b));
        }
        return true;
      };
      int s = 0, ph = 0, it = 0;
      bool ok = pair_id >= total || C::SFBG || load_tile_scales(pair_id, 0);
      const int kb_next = min(3, KB - 1);
      for (int tile = pair_id; tile < total && ok; tile += npairs, ++it) {
        Tile t;
        decode(tile, t);
        const bool has_a = t.rows > 0;
        // weight rows of this CTA's B half
        const int wrow = EPI == PAIR_SWIGLU ? rank * args.I + t.nt * C::NH
                                            : t.nt * C::N + rank * C::NH;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, args.status))) break;
          const uint32_t st = sbase + s * C::STAGE_BYTES;
          const uint32_t fb = bar_full(s);
          mbar_expect_tx(fb, has_a ? C::TX_FULL : C::B_TX);
          if (C::SFST)
            mbar_expect_tx(bar_sfaFull(s),
                           (has_a ? C::SFA_BYTES : 0u) + (C::SFBG ? C::SFB_BYTES : 0u));
          if (C::SFBG)
            bulk_load(st + C::OFF_SFB,
                      args.wsfb + ((static_cast<size_t>(t.e) * args.n_tiles + t.nt) * KB + kb) *
                                      C::SFB_BYTES,
                      C::SFB_BYTES, bar_sfaFull(s));
          const bool last_tail = tail && kb == KB - 1;
          const int kx = last_tail ? K - 128 : kb * 128;
          // F4: byte coordinates in the packed rows (two elements per byte)
          const int kxb = last_tail ? (K - 256) / 2 : kb * 128;
          if (has_a) {
            if (ACT == ACT_HILO)
              tma_load_3d(st, &tmA, kx, t.arow, 0, fb);   // hi rows, then lo rows
            else if (ACT == ACT_E4M3)
              tma_load_2d(st, &tmA, kx, t.arow, fb);
            else if (ACT == ACT_F4)
              tma_load_2d(st, &tmA, kxb, t.arow, fb);
            else
              tma_load_2d(st, last_tail ? &tmAt : &tmA, last_tail ? 0 : kb * 128, t.arow, fb);
            bulk_load(st + C::OFF_SFA,
                      args.sfa + (static_cast<size_t>(t.ttile) * KB + kb) * C::SFA_BYTES,
                      C::SFA_BYTES, C::SFST ? bar_sfaFull(s) : fb);
          }
          if (ACT == ACT_F4)
            tma_load_3d(st + C::OFF_B, &tmB, kxb, wrow, t.e, fb);
          else
            tma_load_3d(st + C::OFF_B, last_tail ? &tmBt : &tmB, last_tail ? 0 : kb * 128, wrow,
                        t.e, fb);
          if (++s == S) { s = 0; ph ^= 1; }
          if (!C::SFBG && kb == kb_next && tile + npairs < total &&
              !(ok = load_tile_scales(tile + npairs, it + 1)))
            break;
        }
      }
    }
  } else if (warp == 2 || (C::SFST && (warp == 3 || warp >= 12))) {
    // ------------------------------------------------------ scale builders --
    // Lane l forms row l of both B atoms: the four scale bytes (K steps 0..3
    // of the k-block) of B columns 32w + l (atom 0) and 128 + 32w + l (atom
    // 1), w = 0..3, read from the tile's scale rows (row c of the tile-scale
    // buffer is B column c; 2-byte aligned rows). 8-bit kinds: each builder
    // stores them, after row l of the stage's token scale atoms, into lane l
    // of its TMEM lane quarter of the stage's slot. Down GEMM (SFBG): the
    // stage brings both weight atoms ready-made, and the builders store row l
    // of each as it is.
    int s = 0, ph = 0, it = 0;
    bool ok = true;
    for (int tile = pair_id; tile < total && ok; tile += npairs, ++it) {
      const int b = it & 1;
      if (!C::SFBG && !(ok = mbar_wait(bar_tsFull(b), (it >> 1) & 1, abort_flag, args.status)))
        break;
      const uint8_t* ts = smem + C::OFF_TS + b * C::TS_BYTES;
      for (int kb = 0; kb < KB; ++kb) {
        // groups of this k-block: 4 (8 for F4); the tail block is [K - KBK, K)
        constexpr int GPB = C::KBK / 32;
        const int gs = (tail && kb == KB - 1) ? G - GPB : GPB * kb;
        uint32_t w[C::F4 ? 16 : 8];
#pragma unroll
        for (int j = 0; j < (C::SFBG ? 0 : 8); ++j) {
          const int c = 32 * j + lane;
#pragma unroll
          for (int q = 0; q < GPB / 4; ++q) {
            // word q of column c: the scale bytes of groups gs + 4q .. + 3
            // (2-byte aligned pairs; a group before the row start, possible
            // only in a tail block whose first steps are not issued, reads 0)
            uint32_t v = 0;
            if (c < C::N) {
              const int g0 = gs + 4 * q;
              const uint16_t* p = reinterpret_cast<const uint16_t*>(ts + c * G);
              const uint32_t lo = g0 >= 0 ? p[g0 >> 1] : 0u;
              const uint32_t hi = g0 + 2 >= 0 ? p[(g0 >> 1) + 1] : 0u;
              v = lo | (hi << 16);
            }
            w[8 * q + j] = v;
          }
        }
        if (C::SFST) {
          // the stage's token scale block has landed; the producer loaded it
          // after "stage empty", so the UMMAs that last read this slot are done
          if (!(ok = mbar_wait(bar_sfaFull(s), ph, abort_flag, args.status))) break;
          tc_fence_after();
          const uint8_t* sfa = smem + s * C::STAGE_BYTES + C::OFF_SFA;
          const uint32_t slot = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                                static_cast<uint32_t>(C::SF_COL0 + s * C::SLOT_COLS);
#pragma unroll
          for (int a = 0; a < C::A_ATOMS; ++a)
            tmem_st4(slot + 4 * a, *reinterpret_cast<const uint4*>(sfa + 512 * a + lane * 16));
          if (C::SFBG) {
            const uint8_t* sfb = smem + s * C::STAGE_BYTES + C::OFF_SFB;
#pragma unroll
            for (int a = 0; a < C::B_ATOMS; ++a)
              tmem_st4(slot + 4 * (C::A_ATOMS + a),
                       *reinterpret_cast<const uint4*>(sfb + 512 * a + lane * 16));
          } else {
            tmem_st4(slot + 4 * C::A_ATOMS, make_uint4(w[0], w[1], w[2], w[3]));
            tmem_st4(slot + 4 * C::A_ATOMS + 4, make_uint4(w[4], w[5], w[6], w[7]));
          }
          tmem_wait_st();
          tc_fence_before();
        } else {
          if (!(ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, args.status))) break;
          uint8_t* sfb = smem + s * C::STAGE_BYTES + C::OFF_SFB;
          // atoms: [word 0: columns 0-127, 128-255][word 1: ...] (F4 has two words)
#pragma unroll
          for (int q = 0; q < GPB / 4; ++q) {
            *reinterpret_cast<uint4*>(sfb + 1024 * q + lane * 16) =
                make_uint4(w[8 * q], w[8 * q + 1], w[8 * q + 2], w[8 * q + 3]);
            *reinterpret_cast<uint4*>(sfb + 1024 * q + 512 + lane * 16) =
                make_uint4(w[8 * q + 4], w[8 * q + 5], w[8 * q + 6], w[8 * q + 7]);
          }
        }
        // orders the shared-memory accesses above (tile-scale and scale-block
        // reads, atoms written for tcgen05.cp) before the async-proxy accesses
        // that follow: tcgen05.cp, the next bulk copies into these buffers
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_full(s));
        if (++s == S) { s = 0; ph ^= 1; }
      }
      __syncwarp();
      if (!C::SFBG && lane == 0) mbar_arrive(bar_tsEmpty(b));
    }
  } else if (warp == 1) {
    // ----------------------------------------- UMMA issuer (even CTA) --
    if (rank == 0 && lane == 0) {
      int s = 0, ph = 0, it = 0;
      bool ok = true;
      for (int tile = pair_id; tile < total && ok; tile += npairs, ++it) {
        const int ab = it & 1;
        const uint32_t ap = (it >> 1) & 1;
        if (!(ok = mbar_wait(bar_accEmpty(ab), ap ^ 1, abort_flag, args.status))) break;
        if (!(ok = mbar_wait_cluster(bar_peerAcc(ab), ap ^ 1, abort_flag, args.status))) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * C::ACC_COLS;
        uint32_t accum = 0;   // the tile's first UMMA overwrites the buffer
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait_cluster(bar_full(s), ph, abort_flag, args.status))) break;
          tc_fence_after();
          const uint32_t st = sbase + s * C::STAGE_BYTES;
          // scale atoms (each 4 TMEM columns): A's terms (or F4's two words),
          // then B's (two per word); 8-bit kinds: the stage's slot, filled by
          // the builders; F4: one slot, copied here
          const uint32_t sfa_t =
              tmem_base + static_cast<uint32_t>(C::SF_COL0 + (C::SFST ? s * C::SLOT_COLS : 0));
          const uint32_t sfb_t = sfa_t + 4 * C::A_ATOMS;
          // operand descriptors of the stage; each K step adds its byte
          // offset to the start-address field (addresses stay below 2^18)
          const uint64_t ad0 = sdesc_k_sw128(st), bd0 = sdesc_k_sw128(st + C::OFF_B);
          if (!C::SFST) {
#pragma unroll
            for (int a = 0; a < C::A_ATOMS; ++a)
              tmem_cp_32x128b_x4_pair(sfa_t + 4 * a,
                                      sdesc_k_noswizzle(st + C::OFF_SFA + 512 * a, 128));
#pragma unroll
            for (int a = 0; a < C::B_ATOMS; ++a)
              tmem_cp_32x128b_x4_pair(sfb_t + 4 * a,
                                      sdesc_k_noswizzle(st + C::OFF_SFB + 512 * a, 128));
          }
          // K steps with compile-time indices; a tail k-block issues only its
          // steps past the previous block
          auto step = [&](const int kk) {
            if (C::F4) {
              const uint32_t id = static_cast<uint32_t>(kk & 1) * 2;
              umma_mxf4_pair(d, ad0 + static_cast<uint64_t>(kk * 2), bd0 + static_cast<uint64_t>(kk * 2),
                             idesc_mxf4(256, C::N, id, id), (sfa_t + 4 * (kk >> 1)) | (id << 30),
                             (sfb_t + 8 * (kk >> 1)) | (id << 30), accum);
              accum = 1;
            } else {
#pragma unroll
              for (int h = 0; h < C::TERMS; ++h) {
                umma_mx_pair(d, ad0 + static_cast<uint64_t>((h * C::A_PLANE + kk * 32) >> 4),
                             bd0 + static_cast<uint64_t>(kk * 2),
                             idesc_pair(256, C::N, C::ATYPE, static_cast<uint32_t>(kk)),
                             (sfa_t + 4 * h) | (static_cast<uint32_t>(kk) << 30),
                             sfb_t | (static_cast<uint32_t>(kk) << 30), accum);
                accum = 1;
              }
            }
          };
          if (!(tail && kb == KB - 1)) {
            step(0);
            step(1);
            step(2);
            step(3);
          } else if (tail_steps == 3) {
            step(1);
            step(2);
            step(3);
          } else if (tail_steps == 2) {
            step(2);
            step(3);
          } else {
            step(3);
          }
          umma_commit_pair(bar_empty(s));
          if (++s == S) { s = 0; ph ^= 1; }
        }
        if (ok) umma_commit_pair(bar_accFull(ab));
      }
    } else if (rank == 1 && lane == 0) {
      // ---------------------------------------- stage relay (odd CTA) --
      int s = 0, ph = 0;
      bool ok = true;
      for (int tile = pair_id; tile < total && ok; tile += npairs) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = mbar_wait(bar_full(s), ph, abort_flag, args.status))) break;
          // the stage is complete in this CTA's shared memory and TMEM slot
          // (observed with acquire semantics above: the builders waited for
          // their tcgen05.st to complete before arriving); forward that to the
          // issuer. A release at cluster scope here measured 0.35 us per stage
          // on the issuer's critical path.
          mbar_arrive_remote_relaxed(mapa_shared(bar_full(s), 0));
          if (++s == S) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp >= 4 && warp < 4 + C::EPI_WARPS) {
    // ----------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    const int egrp = (warp - 4) >> 2;   // 0 or 1: alternate column groups
    const int m = quad * 32 + lane;     // token row of this CTA's half
    int it = 0;
    for (int tile = pair_id; tile < total; tile += npairs, ++it) {
      Tile t;
      decode(tile, t);
      const int ab = it & 1;
      const uint32_t ap = (it >> 1) & 1;
      if (!mbar_wait_cluster(bar_accFull(ab), ap, abort_flag, args.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + ab * C::ACC_COLS;
      const bool valid = m < t.rows;
      if (EPI == PAIR_SWIGLU) {
        // columns c < 96: gate row j0 + c, 96 + c: the same up row; three
        // groups of 32 H columns, each converted for the down GEMM
        const int j0 = t.nt * C::NH;
        const float* brow = args.bias ? args.bias + static_cast<int64_t>(t.e) * 2 * args.I : nullptr;
        const size_t hrow = static_cast<size_t>(t.arow) + m;
#pragma unroll 1
        for (int g = egrp; g < C::NH / 32; g += 2) {
          const int jg = j0 + 32 * g;
          float h[32];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t gv[16], uv[16];
            tmem_ld16_sync(taddr + 32 * g + 16 * q, gv);
            tmem_ld16_sync(taddr + C::NH + 32 * g + 16 * q, uv);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int j = jg + 16 * q + i;
              float gg = __uint_as_float(gv[i]), uu = __uint_as_float(uv[i]);
              if (brow && j < args.I) {
                gg += __ldg(brow + j);
                uu += __ldg(brow + args.I + j);
              }
              float hv = silu_p(gg) * uu;
              // bf16 precision: H is a bf16 row, split exactly below; the
              // quantised modes convert the fp32 value itself
              if (ACT == ACT_HILO) hv = __bfloat162float(__float2bfloat16_rn(hv));
              h[16 * q + i] = hv;
            }
          }
          if (!valid || jg >= args.I) continue;
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(h[i]));
          int kb4, kk4;
          uint8_t* blk;
          if (C::F4) {
            // 256-wide k-blocks of the kind::mxf4 down GEMM: group byte b
            // (0..7) of the block in atom b / 4
            const int gI = args.I / 32, g = jg / 32;
            int b;
            if ((gI % 8) == 0 || g < 8 * (args.h_kb - 1)) {
              kb4 = g >> 3;
              b = g & 7;
            } else {
              kb4 = args.h_kb - 1;
              b = g - (gI - 8);
            }
            kk4 = b & 3;
            blk = args.h_sfa + (static_cast<size_t>(t.ttile) * args.h_kb + kb4) * C::SFA_BYTES +
                  512 * (b >> 2);
          } else {
            pair_group_to_kblock(jg / 32, args.I / 32, args.h_kb, kb4, kk4);
            blk = args.h_sfa + (static_cast<size_t>(t.ttile) * args.h_kb + kb4) * C::SFA_BYTES;
          }
          if (ACT == ACT_HILO) {
            int eh = 0;
            if (amax != 0.f) {
              const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127;
              eh = max(ex - 7, -123);
            }
            const float inv = __uint_as_float(static_cast<uint32_t>(127 - eh) << 23);
            uint32_t hw[8], lw[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              uint32_t a = 0, b = 0;
#pragma unroll
              for (int u = 0; u < 4; u += 2) {
                const float x0 = h[4 * q + u] * inv, x1 = h[4 * q + u + 1] * inv;
                const uint32_t h2 = f32x2_to_e4m3x2(x0, x1);
                const float2 hb = e4m3x2_to_f32x2(h2);
                const uint32_t l2 = f32x2_to_e4m3x2((x0 - hb.x) * 16.f, (x1 - hb.y) * 16.f);
                a |= h2 << (8 * u);
                b |= l2 << (8 * u);
              }
              hw[q] = a;
              lw[q] = b;
            }
            const size_t o = hrow * static_cast<size_t>(args.n_out) + jg;   // rows of I bytes
            uint4* dh = reinterpret_cast<uint4*>(args.h_q + o);
            dh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            dh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
            uint4* dl = reinterpret_cast<uint4*>(args.h_lo + o);
            dl[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            dl[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
            blk[atom_offset(m, kk4)] = static_cast<uint8_t>(eh + 127);
            blk[512 + atom_offset(m, kk4)] = static_cast<uint8_t>(eh + 123);
          } else {
            constexpr int emax = (ACT == ACT_E2M1 || ACT == ACT_F4) ? 2 : 8;
            int ex = 0;
            if (amax > 0.f)
              ex = max(static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127 - emax, -127);
            const float inv = __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
            if (ACT == ACT_E4M3) {
              uint32_t w[8];
#pragma unroll
              for (int q = 0; q < 8; ++q)
                w[q] = f32x2_to_e4m3x2(h[4 * q] * inv, h[4 * q + 1] * inv) |
                       (f32x2_to_e4m3x2(h[4 * q + 2] * inv, h[4 * q + 3] * inv) << 16);
              uint4* dq = reinterpret_cast<uint4*>(args.h_q + hrow * args.n_out + jg);
              dq[0] = make_uint4(w[0], w[1], w[2], w[3]);
              dq[1] = make_uint4(w[4], w[5], w[6], w[7]);
            } else {
              uint32_t w[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint32_t a = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b)
                  a |= f32x2_to_e2m1x2(h[8 * q + 2 * b] * inv, h[8 * q + 2 * b + 1] * inv) << (8 * b);
                w[q] = a;
              }
              *reinterpret_cast<uint4*>(args.h_q + hrow * (args.n_out / 2) + jg / 2) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
            blk[atom_offset(m, kk4)] = static_cast<uint8_t>(ex + 127);
          }
        }
      } else {
        // weighted un-permute: fp32 row p * (y + b) of pair perm[row] at yw[pair]
        const int n0 = t.nt * C::N;
        int pr = 0;
        float w = 0.f;
        if (valid) {
          pr = args.perm[s_off[t.e] + t.mt * 256 + rank * 128 + m];
          w = args.topk_w[pr];
        }
        float* orow = args.out_f32 + static_cast<int64_t>(pr) * args.n_out;
        const float* brow = args.bias ? args.bias + static_cast<int64_t>(t.e) * args.n_out : nullptr;
#pragma unroll 1
        for (int c = 16 * egrp; c < C::N; c += 32) {
          uint32_t y[16];
          tmem_ld16_sync(taddr + c, y);
          const int col = n0 + c;
          if (valid && col < args.n_out) {
            float b[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) b[i] = brow ? __ldg(brow + col + i) : 0.f;
            float4* dst = reinterpret_cast<float4*>(orow + col);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(w * (__uint_as_float(y[4 * i]) + b[4 * i]),
                                   w * (__uint_as_float(y[4 * i + 1]) + b[4 * i + 1]),
                                   w * (__uint_as_float(y[4 * i + 2]) + b[4 * i + 2]),
                                   w * (__uint_as_float(y[4 * i + 3]) + b[4 * i + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_accEmpty(ab));
      if (rank == 1 && threadIdx.x == 4 * 32) {
        // accumulator relay: once all epilogue threads of this CTA have
        // released the buffer, tell the even CTA's issuer
        if (!mbar_wait(bar_accEmpty(ab), ap, abort_flag, args.status)) break;
        mbar_arrive_remote(mapa_shared(bar_peerAcc(ab), 0));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// Weight-scale atoms of the down GEMM's tiles: for expert e, weight tile nt
// (B columns c = 0..N-1, output rows nt N + c) and k-block kb, the 1 KB block
// of two 512-byte atoms the builders store into TMEM: word (c / 32) % 4 of
// row c % 32 of atom c / 128 holds the scale bytes of the k-block's four
// groups of 32 (the last block of a K that is not a multiple of 128 takes the
// last four groups), zero for columns past N or past the output rows. One
// CTA per (e, nt): the tile's scale rows (one contiguous run) are staged in
// shared memory with coalesced loads, then each thread forms one word of
// every k-block's block.
constexpr int kAtomRowsMax = 224 * (kMxMaxK / 32);
__global__ void __launch_bounds__(256) pair_weight_atoms_kernel(const uint8_t* __restrict__ scales,
                                                                int rows, int G, int n_out, int N,
                                                                int n_tiles, int KB,
                                                                uint8_t* __restrict__ atoms) {
  __shared__ __align__(16) uint8_t srows[kAtomRowsMax];
  pdl_wait_and_trigger();
  const int e = blockIdx.x / n_tiles, nt = blockIdx.x % n_tiles;
  const int n0 = nt * N;
  const int nrows = min(N, n_out - n0);
  const int bytes = nrows * G;
  const uint8_t* src = scales + (static_cast<size_t>(e) * rows + n0) * G;
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (bytes & 15) == 0) {
    for (int o = 16 * threadIdx.x; o < bytes; o += 16 * 256)
      *reinterpret_cast<uint4*>(srows + o) = __ldg(reinterpret_cast<const uint4*>(src + o));
  } else {
    for (int o = threadIdx.x; o < bytes; o += 256) srows[o] = src[o];
  }
  __syncthreads();
  const int i = threadIdx.x;
  const int c = 32 * (4 * (i >> 7) + (i & 3)) + ((i >> 2) & 31);
  const bool valid = c < nrows;
  const uint8_t* row = srows + (valid ? c : 0) * G;
  uint32_t* dst = reinterpret_cast<uint32_t*>(atoms + static_cast<size_t>(blockIdx.x) * KB * 1024) + i;
  const bool tail = (G % 4) != 0;
  for (int kb = 0; kb < KB; ++kb) {
    const int g0 = (tail && kb == KB - 1) ? G - 4 : 4 * kb;
    uint32_t v = 0;
    if (valid)
      v = static_cast<uint32_t>(row[g0]) | (static_cast<uint32_t>(row[g0 + 1]) << 8) |
          (static_cast<uint32_t>(row[g0 + 2]) << 16) | (static_cast<uint32_t>(row[g0 + 3]) << 24);
    dst[kb * 256] = v;
  }
}

// ----------------------------------------------------------- host side ----

template <int EPI, int ACT>
cudaError_t launch_pair_impl(const MxGemmProblem& p, int num_sms, cudaStream_t st) {
  using C = PairCfg<EPI, ACT>;
  if (p.K % 64 != 0 || p.K < 128 || p.K > kMxMaxK || p.act != ACT) return cudaErrorInvalidValue;
  if (C::F4 && p.K < 256) return cudaErrorInvalidValue;   // a k-block is 256 elements
  if (ACT == ACT_HILO && p.b_lo != p.b_hi + static_cast<size_t>(p.tok_rows) * p.K)
    return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_mx_pair_kernel<EPI, ACT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tmA, tmAt, tmB, tmBt;
  bool ok;
  if (ACT == ACT_HILO) {
    ok = mx_make_tok8_map(&tmA, p.b_hi, p.tok_rows, p.K, C::MT);
    tmAt = tmA;
  } else if (ACT == ACT_E4M3) {
    ok = mx_make_tok8_map1(&tmA, p.b_hi, p.tok_rows, p.K, C::MT);
    tmAt = tmA;
  } else if (ACT == ACT_F4) {
    // packed rows of K/2 bytes, read as bytes: 128 bytes = 256 elements
    ok = mx_make_tok8_map1(&tmA, p.b_hi, p.tok_rows, p.K / 2, C::MT);
    tmAt = tmA;
  } else {
    const cuuint64_t dims[1] = {static_cast<cuuint64_t>(p.tok_rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.K / 2)};
    const cuuint32_t box[1] = {static_cast<cuuint32_t>(C::MT)};
    ok = mx_make_code_maps(&tmA, &tmAt, p.b_hi, p.K, 2, dims, strides, box);
  }
  const int rows = EPI == PAIR_SWIGLU ? 2 * p.I : p.n_out;
  {
    const cuuint64_t rb = static_cast<cuuint64_t>(p.K / 2);
    if (ACT == ACT_F4) {
      const cuuint64_t dims[3] = {rb, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(p.E)};
      const cuuint64_t strides[2] = {rb, rb * static_cast<cuuint64_t>(rows)};
      const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(C::NH), 1};
      ok = ok && mx_make_bytes_map(&tmB, p.codes, 3, dims, strides, box);
      tmBt = tmB;
    } else {
      const cuuint64_t dims[2] = {static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(p.E)};
      const cuuint64_t strides[2] = {rb, rb * static_cast<cuuint64_t>(rows)};
      const cuuint32_t box[2] = {static_cast<cuuint32_t>(C::NH), 1};
      ok = ok && mx_make_code_maps(&tmB, &tmBt, p.codes, p.K, 3, dims, strides, box);
    }
  }
  if (!ok) return cudaErrorInvalidValue;
  PairArgs a;
  a.offsets = p.offsets;
  a.E = p.E;
  a.K = p.K;
  a.I = p.I;
  a.n_out = p.n_out;
  a.n_tiles = EPI == PAIR_SWIGLU ? (p.I + C::NH - 1) / C::NH : (p.n_out + C::N - 1) / C::N;
  a.rows_per_expert = rows;
  a.KB = (p.K + C::KBK - 1) / C::KBK;
  a.scales = p.scales;
  a.sfa = p.b_sfb;
  a.h_q = p.h_hi;
  a.h_lo = p.h_lo;
  a.h_sfa = p.h_sfb;
  a.h_kb = (p.I + C::KBK - 1) / C::KBK;   // the down GEMM's k-blocks
  a.out_f32 = p.out_f32;
  a.perm = p.perm;
  a.topk_w = p.topk_w;
  a.status = p.status;
  a.bias = p.bias;
  a.wsfb = nullptr;
  if (C::SFBG) {
    static_assert(!C::SFBG || C::SFB_BYTES == 1024, "atom block");
    if (p.wsfb == nullptr || C::N > 224) return cudaErrorInvalidValue;
    launch_kernel(pair_weight_atoms_kernel, dim3(p.E * a.n_tiles), dim3(256), 0, st, p.scales,
                  rows, p.K / 32, p.n_out, C::N, a.n_tiles, a.KB, p.wsfb);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    a.wsfb = p.wsfb;
  }
  const int64_t tiles_bound = (static_cast<int64_t>(p.P) / 256 + p.E) * a.n_tiles;
  int64_t pairs = num_sms / 2;
  if (tiles_bound < pairs) pairs = tiles_bound;
  if (pairs < 1) pairs = 1;
  launch_kernel(grouped_mx_pair_kernel<EPI, ACT>, dim3(static_cast<int>(2 * pairs)), dim3(C::NUM_THREADS), C::SMEM_ALLOC, st, 
      tmA, tmAt, tmB, tmBt, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mx_pair_gateup_swiglu(const MxGemmProblem& p, int num_sms, cudaStream_t st) {
  switch (p.act) {
    case ACT_HILO: return launch_pair_impl<PAIR_SWIGLU, ACT_HILO>(p, num_sms, st);
    case ACT_E4M3: return launch_pair_impl<PAIR_SWIGLU, ACT_E4M3>(p, num_sms, st);
    case ACT_E2M1: return launch_pair_impl<PAIR_SWIGLU, ACT_E2M1>(p, num_sms, st);
    case ACT_F4: return launch_pair_impl<PAIR_SWIGLU, ACT_F4>(p, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

size_t mx_pair_down_atom_bytes(int E, int d, int I) {
  // tiles of N = 224 output rows, k-blocks of 128 (the 8-bit kinds' down GEMM)
  return static_cast<size_t>(E) * ((d + 223) / 224) * ((I + 127) / 128) * 1024;
}

cudaError_t launch_mx_pair_down(const MxGemmProblem& p, int num_sms, cudaStream_t st) {
  switch (p.act) {
    case ACT_HILO: return launch_pair_impl<PAIR_DOWN, ACT_HILO>(p, num_sms, st);
    case ACT_E4M3: return launch_pair_impl<PAIR_DOWN, ACT_E4M3>(p, num_sms, st);
    case ACT_E2M1: return launch_pair_impl<PAIR_DOWN, ACT_E2M1>(p, num_sms, st);
    case ACT_F4: return launch_pair_impl<PAIR_DOWN, ACT_F4>(p, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
