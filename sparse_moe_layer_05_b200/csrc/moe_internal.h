// moe_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Launches of a forward pass after its first one are made with programmatic
// stream serialization (each kernel's launch and prologue overlap its
// predecessor's tail; every kernel waits for its predecessor before touching
// global memory, moe_ptx.cuh). The flag is per host thread: the ABI sets it
// once a pass has launched its first kernel and clears it at the pass's end.
bool& pdl_launches();

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_launches() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Same, as clusters of `cluster` CTAs along x (grid.x a multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  int cluster, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_launches() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Token chunk of the permutation kernels (tokens per block).
constexpr int kPermChunk = 256;
// Rows of one M tile of the grouped GEMMs.
constexpr int kTileM = 256;

inline int perm_chunks(int T) { return (T + kPermChunk - 1) / kPermChunk; }

// K2 for T <= kPermChunk in one launch: counts, offsets, M-tile prefix and
// perm, identical to launch_perm_hist + launch_perm_scan + launch_perm_scatter.
cudaError_t launch_perm_small(const int32_t* topk_idx, int T, int k, int E, int32_t* counts,
                              int32_t* offsets, int32_t* mtile_prefix, int32_t* perm,
                              cudaStream_t st);
// K1, the router (moe_router_tc.cu): splits W_r into three bf16 terms, its
// row norms and fingerprints in `scratch` (router_tc_scratch_bytes, which
// also holds ||x_t||^2 per token); then one kernel computes the logits
// (written to `logits`, [T][E] fp32) and one the top-k with near ties settled
// in fp64, and the softmax. Its first launch clears *status.
size_t router_tc_scratch_bytes(int E, int d, int T);
// With perm given and T <= kPermChunk, the top-k kernel's last block also
// builds the permutation (counts may be null), as launch_perm_small would.
cudaError_t launch_router_tc(const uint16_t* x, const float* W_r, const float* b_r, int T, int E,
                             int k, int d, void* scratch, float* logits, int32_t* topk_idx,
                             float* topk_w, int* status, cudaStream_t st,
                             int32_t* counts = nullptr, int32_t* offsets = nullptr,
                             int32_t* mtile_prefix = nullptr, int32_t* perm = nullptr);
// K2: per-chunk expert histograms.
cudaError_t launch_perm_hist(const int32_t* topk_idx, int T, int k, int E, int32_t* chunk_hist,
                             cudaStream_t st);
// K2: counts, offsets, per-chunk bases and the M-tile prefix of each expert.
cudaError_t launch_perm_scan(const int32_t* chunk_hist, int nchunks, int E, int32_t* counts,
                             int32_t* offsets, int32_t* chunk_base, int32_t* mtile_prefix,
                             cudaStream_t st);
// K2: stable scatter of pair ids into expert-contiguous order.
cudaError_t launch_perm_scatter(const int32_t* topk_idx, int T, int k, int E,
                                const int32_t* chunk_base, int32_t* perm, int32_t* inv,
                                cudaStream_t st);
// K2: gather activation rows into permuted order.
cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* perm, int P, int k, int d,
                               uint16_t* xp, cudaStream_t st);
// Per-token sum of the k weighted expert rows (plus the residual row, when
// resid is not null), rounded once to bf16.
cudaError_t launch_combine(const float* yw, int T, int k, int d, const uint16_t* resid,
                           uint16_t* out, cudaStream_t st);
// Pre-MoE RMSNorm: x = bf16((h / sqrt(mean(h^2) + eps)) * g), rows of d.
cudaError_t launch_rms_norm(const uint16_t* h, const float* g, float eps, int T, int d,
                            uint16_t* x, cudaStream_t st);
// E8M0 scales [E][N][G] -> [E][G][N] (the GEMMs load them with TMA per k-block);
// experts with counts[e] == 0 are skipped (counts may be null: all experts).
cudaError_t launch_transpose_scales(const uint8_t* in, int E, int N, int G, const int32_t* counts,
                                    uint8_t* out, cudaStream_t st);
// MXFP4 rows -> bf16 rows (same decoder as the GEMMs).
cudaError_t launch_mxfp4_to_bf16(const uint8_t* codes, const uint8_t* scales, int rows, int K,
                                 uint16_t* out, cudaStream_t st);

// K3/K4: expert-grouped MXFP4 GEMMs on tcgen05.
struct GroupedGemmProblem {
  const uint16_t* A;        // [P][K] bf16 rows in permuted order
  const uint8_t* codes;     // [E][Nrows][K/2]
  const uint8_t* scales_t;  // [E][K/32][Nrows] (transposed E8M0 scales)
  const int32_t* offsets;   // [E+1]
  const int32_t* mprefix;   // [E+1] prefix of M tiles per expert
  int P, E, K, Nrows;
  uint16_t* out;            // SwiGLU: H [P][I] bf16
  float* out_f32;           // down: Yw [T*k][d] fp32, row t*k+j = p_j * y
  const int32_t* perm;      // down: pair id of each permuted row
  const float* topk_w;      // down: weight of each pair
  int n_out;                // output columns (I for SwiGLU, d for down)
  int* status;
  int tiles;                // TILES_SINGLE, TILES_PAIR or TILES_SWAP
  // optional per-expert bias (nullptr: none), added to the fp32 accumulator:
  // SwiGLU [E][2I] (gate 0..I-1, up I..2I-1, before the silu); down [E][d]
  // (before the routing weight)
  const float* bias;
};

// Grouped-GEMM tile shapes.
constexpr int TILES_SINGLE = 1;   // 256 activation rows x 128 weight rows, one CTA
constexpr int TILES_PAIR = 2;     // 256 x 240 on a 2-CTA cluster (cta_group::2)
constexpr int TILES_SWAP = 3;     // 128 weight rows x 64 tokens, weights as UMMA A
cudaError_t launch_gemm_gateup_swiglu(const GroupedGemmProblem& p, int num_sms, cudaStream_t st);
cudaError_t launch_gemm_down_combine(const GroupedGemmProblem& p, int num_sms, cudaStream_t st);

// ---------------------------------------------- block-scaled (MX) path ----
// Largest d or I of the block-scaled path (a tile's weight scales, 128 rows of
// K/32 bytes, are staged in shared memory).
constexpr int kMxMaxK = 3072;
constexpr int TILES_MX = 4;       // block-scaled tcgen05 GEMMs (E2M1 x hi/lo E4M3)
constexpr int TILES_MX_PAIR = 5;  // the same on a CTA pair (cta_group::2, 256-token tiles)
// Tile variants: small (16-token tiles, two CTAs per SM, two UMMA issuers
// each; few rows per expert) and large (120-token tiles, one CTA per SM).
constexpr int kMxSmall = 0;
constexpr int kMxLarge = 1;
// CTA-pair variant (moe_mx_pair.cu): 256-token tiles on a 2-CTA cluster,
// tokens as the UMMA A operand (M = 256); token rows padded to 128.
constexpr int kMxPair = 2;
int mx_tile_tokens(int variant, int act);

// Activation operand of the block-scaled GEMMs (the B operand: token rows of x
// for gate/up, of H for down), per group of 32 along K:
//   ACT_HILO  bf16 precision: two E4M3 terms (hi, lo) with E8M0 scales
//   ACT_E4M3  the w4a8 layer: one E4M3 element, OCP MX scale (emax 8)
//   ACT_E2M1  the w4a4 layer: one E2M1 element, OCP MX scale (emax 2), rows
//             packed two elements per byte (low nibble first)
//   ACT_F4    the w4a4 layer on the CTA-pair kernel with tcgen05 kind::mxf4:
//             rows as ACT_E2M1, both operands read packed (no widening), and
//             the token-side scale blocks laid out per 256-wide k-block
constexpr int ACT_HILO = 0;
constexpr int ACT_E4M3 = 1;
constexpr int ACT_E2M1 = 2;
constexpr int ACT_F4 = 3;

// Rows of the padded token layout (each expert's rows rounded up to a
// multiple of the tile's tokens) and bytes of its B-scale blocks, for either
// variant.
size_t mx_tok_rows(int P, int E);
size_t mx_sfb_bytes(int P, int E, int K);

// K2: gather x rows into the padded token layout as hi/lo E4M3 rows plus the
// B-scale blocks the GEMM loads per (token tile, k-block). With inv (pair id
// -> permuted row) and topk_idx, token-major: each token's groups converted
// once for its k rows (identical results).
cudaError_t launch_mx_quant_gather(int variant, const uint16_t* x, const int32_t* perm,
                                   const int32_t* offsets, int E, int P, int k, int K, uint8_t* qhi,
                                   uint8_t* qlo, uint8_t* sfb, const int32_t* topk_idx,
                                   const int32_t* inv, int T, cudaStream_t st);
// The same for the quantised activation modes (act ACT_E4M3 or ACT_E2M1): one
// MX-converted row per routed pair (K bytes, or K/2 for E2M1) plus its
// B-scale blocks.
cudaError_t launch_mx_act_quant_gather(int variant, int act, const uint16_t* x,
                                       const int32_t* perm, const int32_t* offsets, int E, int P,
                                       int k, int K, uint8_t* q, uint8_t* sfb, cudaStream_t st);
// The MX conversion on plain rows: q [R][K] (E4M3) or [R][K/2] (E2M1, packed),
// scales [R][K/32] E8M0.
cudaError_t launch_mx_act_quant_rows(int act, const uint16_t* x, int R, int K, uint8_t* q,
                                     uint8_t* scales, cudaStream_t st);
// The same split on plain rows, scales as [R][K/32][2] (hi byte, lo byte).
cudaError_t launch_mx_split_rows(const uint16_t* x, int R, int K, uint8_t* qhi, uint8_t* qlo,
                                 uint8_t* scales, cudaStream_t st);

struct MxGemmProblem {
  const uint8_t* codes;     // [E][rows][K/2] E2M1 codes
  const uint8_t* scales;    // [E][rows][K/32] E8M0 scales (row-major, as given)
  const uint8_t* b_hi;      // [tok_rows][K] E4M3 (padded token layout)
  const uint8_t* b_lo;
  const uint8_t* b_sfb;     // B-scale blocks
  const int32_t* offsets;   // [E+1]
  int P, E, K, I;
  int tok_rows;
  // SwiGLU: quantized H (padded layout) and its B-scale blocks
  uint8_t* h_hi;
  uint8_t* h_lo;
  uint8_t* h_sfb;
  // down: weighted rows
  float* out_f32;
  const int32_t* perm;
  const float* topk_w;
  int n_out;                // I for SwiGLU, d for down
  int* status;
  const float* bias;        // optional, as in GroupedGemmProblem
  int act;                  // ACT_HILO, ACT_E4M3 or ACT_E2M1 (b_lo / h_lo unused but HILO)
  // CTA-pair down GEMM with 8-bit activations: room for its weight-scale atoms
  // (mx_pair_down_atom_bytes), written by the launch before the GEMM
  uint8_t* wsfb;
};
cudaError_t launch_mx_gemm_gateup_swiglu(int variant, const MxGemmProblem& p, int num_sms,
                                         cudaStream_t st);
cudaError_t launch_mx_gemm_down(int variant, const MxGemmProblem& p, int num_sms, cudaStream_t st);
// The CTA-pair variant (moe_mx_pair.cu): same problem description; token rows
// and their scale blocks in the 128-row padded layout.
cudaError_t launch_mx_pair_gateup_swiglu(const MxGemmProblem& p, int num_sms, cudaStream_t st);
cudaError_t launch_mx_pair_down(const MxGemmProblem& p, int num_sms, cudaStream_t st);
size_t mx_pair_down_atom_bytes(int E, int d, int I);

// Tensor maps of the block-scaled path (moe_mx_gemm.cu): E2M1 code rows
// (main map over whole 128-element k-blocks plus a tail map for [K-128, K)),
// E4M3 token rows as two planes (hi, lo) or one.
bool mx_make_code_maps(CUtensorMap* main_map, CUtensorMap* tail_map, const uint8_t* codes, int K,
                       int rank, const cuuint64_t* dims_rest, const cuuint64_t* strides,
                       const cuuint32_t* box_rest);
bool mx_make_tok8_map(CUtensorMap* m, const uint8_t* hi, int rows, int K, int nt);
bool mx_make_tok8_map1(CUtensorMap* m, const uint8_t* q, int rows, int K, int nt);
// A byte tensor (rank 1..5, dims/strides/box as cuTensorMapEncodeTiled takes
// them, 128-byte swizzle).
bool mx_make_bytes_map(CUtensorMap* m, const uint8_t* base, int rank, const cuuint64_t* dims,
                       const cuuint64_t* strides, const cuuint32_t* box);
// The same for a bf16 tensor.
bool mx_encode_bf16_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                        const cuuint64_t* strides, const cuuint32_t* box);

// Debug/self-test: one bounded wait on an mbarrier that nothing completes.
cudaError_t launch_wait_timeout_selftest(int* status, cudaStream_t st);

}  // namespace moe
