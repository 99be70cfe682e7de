/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) sparse-MoE layer forward pass.
 *
 * The layer is the gpt-oss-style Mixture-of-Experts feed-forward block:
 *
 *   s_e   = W_r[e] . x_t + b_r[e]                          (router logits)
 *   S_t   = the k largest s_e (ties: lower expert index first)
 *   p_j   = exp(s_j) / sum_{l in S_t} exp(s_l)             (softmax over S_t)
 *   E_e(x)= W_down[e] (silu(W_gate[e] x) * (W_up[e] x))    (SwiGLU expert)
 *   out_t = sum_{j in S_t} p_j E_j(x_t)
 *
 * Sources: "llm-surgery-dark-arts-gpt-oss-40b-64a8-init", section 2, "Proof"
 * (the forward pass, the router logits and the softmax over the selected set);
 * field guide "gpt-oss 20B", "03 Sparse Mixture of Experts" (score all experts,
 * keep the top k, normalise those scores, weighted sum of SwiGLU experts);
 * "gpt-oss-20b and gpt-oss-120b", "Four-bit expert weights" (MXFP4 experts,
 * 4.25 bits per parameter); "shrink/gpt_oss-mic", "Preserved properties"
 * (hidden_act silu).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named *_dev are CUDA device pointers; *_host are host pointers.
 *   Every device pointer must be 16-byte aligned. Inputs are read-only.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream). All device work is enqueued on it; no entry point synchronises
 *   the stream except moe_forward_hostio and moe_sync_status, which say so.
 * - The library allocates no device memory. The caller owns every buffer,
 *   including the workspace, whose size moe_workspace_size() returns.
 *   Concurrent calls must not share a workspace.
 * - Errors are returned as moe_status; nothing is thrown or printed.
 *   Arguments are checked before anything is launched; on an argument error
 *   no work is enqueued. Device-side timeouts (a bounded wait in a kernel
 *   that gave up) are recorded in a status word inside the workspace and
 *   reported by moe_sync_status() or by the next call on that workspace.
 *
 * Data layout (row-major, C order)
 * --------------------------------
 *   x           [T][d]        bf16 (raw 16-bit patterns)
 *   W_r         [E][d]        float32
 *   b_r         [E]           float32
 *   Wgu_codes   [E][2I][d/2]  uint8  MXFP4 E2M1 codes; rows 0..I-1 are the
 *                                    gate projection, rows I..2I-1 the up
 *                                    projection; byte b of a row holds
 *                                    element 2b in its low nibble and
 *                                    element 2b+1 in its high nibble
 *   Wgu_scales  [E][2I][d/32] uint8  E8M0 scale 2^(S-127) of each group of
 *                                    32 consecutive elements along d
 *   Wd_codes    [E][d][I/2]   uint8  down projection codes (contraction on I)
 *   Wd_scales   [E][d][I/32]  uint8
 *   out         [T][d]        bf16
 *   topk_idx    [T][k]        int32  experts of token t, logit descending,
 *                                    then expert index ascending
 *   topk_w      [T][k]        float32 selected-set softmax weights
 *
 * Supported range: 1 <= E <= 256, 1 <= k <= min(E, 32), T >= 0,
 * d and I multiples of 32 with 32 <= d, I <= 16384. Decoded weight
 * magnitudes must be below 2^128 (E8M0 bytes up to 252), the range bf16
 * represents; within it every decoded weight is exact.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, misaligned pointer, bad shape  */
  MOE_ERR_UNSUPPORTED = 2,   /* shape outside the supported range            */
  MOE_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required   */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed            */
  MOE_ERR_TIMEOUT = 5,       /* a kernel's bounded wait expired              */
  MOE_ERR_NO_DEVICE = 6      /* no sm_100 device is current                  */
} moe_status;

/* Human-readable name of a status code (static storage, never NULL). */
MOE_API const char* moe_status_string(moe_status s);

/* Library version as major*10000 + minor*100 + patch. */
MOE_API int moe_version(void);

/*
 * Tile policy of the grouped GEMMs, process-wide: 0 (default) picks by shape
 * from the average number of routed rows per expert, P/E with P = T*k:
 *   P/E < 32        block-scaled tiles (policy 4 below) where the shape allows
 *                   them, else swapped-operand tiles (128 weight rows x 64
 *                   tokens, the decoded weights as the UMMA A operand),
 *   32 <= P/E < 192 single-CTA tiles (256 x 128, the second 128-row half
 *                   skipped for short expert tails),
 *   P/E >= 192      CTA-pair tiles: the block-scaled ones (policy 5 below)
 *                   where the shape allows them, else bf16 CTA-pair tiles (a
 *                   2-CTA cluster computes 256 x 240 tiles with tcgen05
 *                   cta_group::2).
 * 1, 2 and 3 force single-CTA, CTA-pair and swapped-operand tiles; these
 * decode the MXFP4 weights to bf16 in shared memory or TMEM and run bf16
 * UMMAs on bf16 activations.
 * 4 selects the block-scaled tiles: tcgen05.mma .kind::mxf8f6f4 with the E2M1
 * codes widened to 8-bit containers by TMA, the E8M0 weight scales applied by
 * the tensor core, and each bf16 activation (and H) row split per 32 elements
 * into two E4M3 terms (hi and lo) with E8M0 scales; the split is exact for
 * elements of at least 2^-13 of their group's max |x|, smaller ones keep an
 * error below 2^-21 of it. 128 weight rows x 16 tokens per tile, two CTAs
 * per SM with two UMMA-issuing threads each (120-token tiles, one CTA per SM,
 * when experts average 64 rows or more).
 * 5 selects the block-scaled tiles on a CTA pair: a 2-CTA cluster computes
 * 256-token tiles with tcgen05.mma.cta_group::2 (M = 256 token rows, the two
 * E4M3 terms issued as two UMMAs into one accumulator; N = 192 weight rows for
 * gate/up, 240 for down).
 * 4 and 5 need d and I multiples of 64 in [128, 3072] and 32-byte aligned
 * code arrays; otherwise they pick as policy 0 does.
 * All policies compute the same function within the output tolerance.
 * This sets the process default that the entry points without an options
 * argument use; a change takes effect for calls made after it, from any
 * thread. Callers that share a process and want a policy of their own pass
 * it per call through moe_forward_ex instead. MOE_ERR_INVALID_ARG for other
 * values.
 */
MOE_API moe_status moe_set_tile_policy(int policy);

/*
 * Precision of the activations that enter the expert GEMMs (the expert inputs
 * x and the SwiGLU rows H), per call through moe_forward_opts.act_quant.
 *   MOE_ACT_BF16   the layer as the pages define it: bf16 activations used at
 *                  full precision (the block-scaled tiles split each value
 *                  exactly into two E4M3 terms); output within 2e-2 x RMS.
 * The two others change the function ("gpt-oss-20b and gpt-oss-120b",
 * "Four-bit expert weights" puts only the expert weights in MXFP4; field
 * guide "gpt-oss 20B": MXFP4 is "not every path"): the activations are
 * rounded to an MX block format, per group of 32 along the contraction, with
 * the OCP Microscaling conversion (shared scale 2^(floor(log2 max|v|) - emax),
 * elements rounded to nearest even, magnitudes above the largest normal
 * clamped to it):
 *   MOE_ACT_MXFP8  E4M3 elements (emax 8): the w4a8 layer;
 *   MOE_ACT_MXFP4  E2M1 elements (emax 2): the w4a4 layer.
 */
typedef enum { MOE_ACT_BF16 = 0, MOE_ACT_MXFP8 = 1, MOE_ACT_MXFP4 = 2 } moe_act_quant;

/*
 * Per-call options of moe_forward_ex. Zero-initialise and set what you need.
 *   tile_policy    -1: the process default (moe_set_tile_policy); 0: pick by
 *                  shape; 1..5: force a tile family (as moe_set_tile_policy).
 *                  0 is what a zeroed struct asks for.
 *   act_quant      a moe_act_quant value (0 = MOE_ACT_BF16).
 *   gu_bias_dev, down_bias_dev   the experts' biases as in
 *                  moe_forward_biased; NULL for none.
 */
typedef struct {
  int tile_policy;
  int act_quant;
  const float* gu_bias_dev;
  const float* down_bias_dev;
} moe_forward_opts;

/*
 * Bytes of device workspace moe_forward needs for this shape (0 for invalid
 * shapes). The workspace holds the router's logits and top-k, the routing
 * tables, the permuted activations, the SwiGLU hidden rows H [T*k][I] bf16,
 * the weighted per-slot expert outputs [T*k][d] fp32, and the down weights'
 * scale factors re-laid out for the CTA-pair tiles (E * ceil(d/224) *
 * ceil(I/128) KiB).
 */
MOE_API size_t moe_workspace_size(int E, int k, int T, int d, int I);

/*
 * Forward pass of the MoE layer (the whole path: router, top-k, selected-set
 * softmax, permutation, gate/up grouped GEMM with SwiGLU, down grouped GEMM
 * with the weighted un-permute, and the per-token sum).
 * "llm-surgery-dark-arts-gpt-oss-40b-64a8-init", section 2, "Proof".
 *
 * Writes out_dev [T][d] bf16 completely. Asynchronous on `stream`.
 */
MOE_API moe_status moe_forward(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                       const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                       const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev,
                       int E, int k, int T, int d, int I, void* out_dev,
                       void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * moe_forward with per-expert projection biases, as a gpt-oss expert carries
 * them (the parameter totals of "gpt-oss-20b and gpt-oss-120b" count 2I + d
 * bias values per expert):
 *   H = silu(x Wgate^T + b_gate) * (x Wup^T + b_up),  y = H Wdown^T + b_down,
 * and the layer output sum_j p_j y_j as in moe_forward.
 * gu_bias_dev [E][2I] f32: row e holds expert e's gate biases (0..I-1), then
 * its up biases (I..2I-1). down_bias_dev [E][d] f32. Either may be NULL (no
 * bias on that projection; with both NULL this is moe_forward); each given
 * one is 16-byte aligned device memory, read-only and the caller's. The
 * biases are added to the fp32 accumulators in the GEMM epilogues (no extra
 * launches). Errors, workspace and stream semantics are those of moe_forward.
 */
MOE_API moe_status moe_forward_biased(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                                      const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                                      const float* gu_bias_dev, const uint8_t* Wd_codes_dev,
                                      const uint8_t* Wd_scales_dev, const float* down_bias_dev,
                                      int E, int k, int T, int d, int I, void* out_dev,
                                      void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * moe_forward with per-call options (opts may be NULL: the process default
 * tile policy, bf16 activations, no biases). Everything else -- arguments,
 * workspace size (moe_workspace_size), errors, stream semantics -- is as in
 * moe_forward. MOE_ERR_INVALID_ARG for a tile_policy outside -1..5 or an
 * unknown act_quant; MOE_ERR_UNSUPPORTED for an act_quant the shape cannot
 * run (the quantised modes need the block-scaled tiles' shapes: d and I
 * multiples of 64 in [128, 3072], 32-byte aligned code arrays).
 * The quantised modes always run the block-scaled tiles (E2M1 weights x E4M3
 * or E2M1 activations, one term): 16-token tiles when experts average under
 * 64 rows; 256-token tiles on a CTA pair with tile_policy 5, or with 0 when
 * experts average 192 rows or more (w4a4 there runs kind::mxf4 when d and I
 * are at least 256); else 128-token tiles on one CTA.
 * Their intermediates in the workspace: the converted x rows in the xp region
 * and the converted H rows in the h region, in the padded token layout the
 * block-scaled tiles read, their scales at x_scales and h_scales.
 */
MOE_API moe_status moe_forward_ex(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                                  const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                                  const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev,
                                  int E, int k, int T, int d, int I, void* out_dev,
                                  void* workspace_dev, size_t workspace_bytes,
                                  const moe_forward_opts* opts, void* stream);

/*
 * Same as moe_forward, instrumented: records a CUDA event on `stream` at the
 * boundaries of the pass's stages and one after the last, waits for the last
 * event, and writes to stage_ms_host[0..11] (host memory, 12 floats) the
 * device time in milliseconds of each stage, in order -- router (its weight
 * split, logits and top-k/softmax launches; for at most 256 tokens also the
 * permutation), top-k/softmax (0: inside the router stage), expert histogram,
 * scan, scatter, activation gather, the two scale transposes (gate/up, down),
 * gate/up GEMM + SwiGLU, down GEMM + weighted un-permute (on the CTA-pair
 * tiles with the launch before it that lays out the down weights' scale
 * atoms), per-token sum --
 * and in stage_ms_host[11] the span from the first launch to the end of the
 * last. A stage the pass does not launch reads as the cost of its two events.
 * Blocks the calling thread until the pass has finished.
 */
MOE_API moe_status moe_forward_timed(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                                     const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                                     const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev,
                                     int E, int k, int T, int d, int I, void* out_dev,
                                     void* workspace_dev, size_t workspace_bytes, void* stream,
                                     float* stage_ms_host);

/*
 * moe_forward_timed with only some launch boundaries recorded, for timing
 * with less interference: each event recorded between two launches delays
 * the second by a few microseconds, which is visible on decode-sized steps.
 * Bit i of event_mask (i = 0..11) records boundary i, the event before launch
 * i in the order of moe_forward_timed (bit 11: after the last launch); bits 0
 * and 11 are always recorded, bits above 11 are an error (MOE_ERR_INVALID_ARG).
 * stage_ms_host[i] for a recorded boundary i < 11 is the device time to the
 * next recorded boundary, 0 for the others; stage_ms_host[11] is the whole
 * span. Example: bits 0, 8, 9, 11 give the gate/up GEMM alone in [8] and the
 * whole pass in [11]. Blocks the calling thread until the pass has finished.
 */
MOE_API moe_status moe_forward_timed_events(const void* x_dev, const float* W_r_dev,
                                            const float* b_r_dev, const uint8_t* Wgu_codes_dev,
                                            const uint8_t* Wgu_scales_dev,
                                            const uint8_t* Wd_codes_dev,
                                            const uint8_t* Wd_scales_dev, int E, int k, int T,
                                            int d, int I, void* out_dev, void* workspace_dev,
                                            size_t workspace_bytes, void* stream,
                                            unsigned int event_mask, float* stage_ms_host);

/*
 * moe_forward_timed_events with per-call options (opts as in moe_forward_ex;
 * NULL: the defaults). Same timing semantics, errors and blocking.
 */
MOE_API moe_status moe_forward_timed_ex(const void* x_dev, const float* W_r_dev,
                                        const float* b_r_dev, const uint8_t* Wgu_codes_dev,
                                        const uint8_t* Wgu_scales_dev, const uint8_t* Wd_codes_dev,
                                        const uint8_t* Wd_scales_dev, int E, int k, int T, int d,
                                        int I, void* out_dev, void* workspace_dev,
                                        size_t workspace_bytes, const moe_forward_opts* opts,
                                        void* stream, unsigned int event_mask,
                                        float* stage_ms_host);

/*
 * Same as moe_forward with the activations in host memory: copies x_host
 * (T*d*2 bytes; pinned memory gives asynchronous copies) to the workspace,
 * runs the forward pass and copies the result to out_host, then synchronises
 * `stream`. Expert and router weights stay on the device (the layer's
 * resident parameters). moe_workspace_size_hostio() gives the workspace size.
 * Batches of at least 2048 tokens are processed as 4 chunks of tokens (each
 * token's output depends on that token alone, so the result is the same):
 * the copy in, the forward and the copy out of neighbouring chunks overlap on
 * two copy streams the library creates once per device, ordered after the
 * caller's earlier work on `stream`. Host threads may call it concurrently on
 * one device (with separate workspaces): they take turns at enqueueing and
 * share the copy streams. If a launch or a copy fails, the call waits for the
 * copies it had enqueued before it returns the error. The call returns the
 * device status of the pass itself: each chunk keeps its own status word
 * (chunk c uses 32-bit word c of the 16-byte status block at the workspace's
 * start), so a timeout in any chunk is returned. moe_workspace_size_hostio()
 * is at least moe_workspace_size(), so one workspace serves both calls.
 */
MOE_API size_t moe_workspace_size_hostio(int E, int k, int T, int d, int I);
MOE_API moe_status moe_forward_hostio(const void* x_host, const float* W_r_dev, const float* b_r_dev,
                              const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                              const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev,
                              int E, int k, int T, int d, int I, void* out_host,
                              void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * Router and permutation only (the first two steps of the path): router
 * logits in fp32, top-k with the lower-index tie rule, selected-set softmax
 * ("Proof", s_i and p_i), then the stable grouping of the T*k (token, slot)
 * pairs by expert.
 *
 * Precision of the choice: the logits are fp32 dot products on the tensor
 * cores (the fp32 router weights as three bf16 terms, exactly). Where two
 * neighbouring logits of a token's top-k list, or the k-th and a runner-up,
 * lie within tau_t = 2^-17 ||x_t||_2 max_e ||W_r[e]||_2 of each other, their
 * order is decided on fp64 dot products of the same inputs; so the experts
 * and their order are those of the exact logits, equal exact logits going to
 * the lower index. The softmax uses the fp32 logits (the fp64 ones where
 * they were computed). moe_forward leaves the fp32 logits in its workspace
 * (moe_workspace_layout's logits, [T][E]).
 *
 *   topk_idx_dev [T][k] int32, topk_w_dev [T][k] float32
 *   counts_dev   [E]    int32  pairs routed to each expert
 *   offsets_dev  [E+1]  int32  exclusive prefix sum of counts
 *   perm_dev     [T*k]  int32  pair ids (t*k + j) grouped by expert, in
 *                              ascending pair id inside each expert
 * Any of counts/offsets/perm may be NULL to skip the permutation outputs
 * (all three NULL, or none). workspace size: moe_route_workspace_size().
 */
MOE_API size_t moe_route_workspace_size(int E, int k, int T, int d);
MOE_API moe_status moe_route(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                     int E, int k, int T, int d,
                     int32_t* topk_idx_dev, float* topk_w_dev,
                     int32_t* counts_dev, int32_t* offsets_dev, int32_t* perm_dev,
                     void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * moe_route without a workspace, for callers that cannot allocate device
 * memory: code that is handed only its inputs, outputs and a stream (plugin
 * hooks of inference runtimes, serving threads that must not call cudaMalloc,
 * which can synchronise the device and can fail under memory pressure). The
 * pages have no counterpart to this entry point; it is a deployment aid.
 *
 * Same arguments, outputs and results as moe_route (all five outputs are
 * required here), minus the workspace; it makes the same launches as
 * moe_route, so its results are bit-identical to moe_route's. The scratch it
 * needs (router logits, the router's split weights and small routing tables)
 * lives in one device array owned by the library: 32.1 MiB that every GPU
 * which loads the library holds until the process exits. Limit: T * E <= 1,048,576 (e.g. T = 8192 tokens at E = 128,
 * or T = 4096 at E = 248); larger calls return MOE_ERR_UNSUPPORTED and
 * launch nothing. Every call looks up the array's device address on the
 * current device (cudaGetSymbolAddress; no address is cached, so a new
 * primary context or a device reset needs nothing from the caller); the
 * first call on a device also loads the library's device code there, so
 * make that first call before any stream capture. All calls on a device share the array and
 * it keeps the last call's contents (each call rewrites what it reads), so
 * calls whose device work overlaps -- concurrent streams, or several host
 * threads -- race on it; serialise them.
 */
MOE_API moe_status moe_route_noalloc(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                                     int E, int k, int T, int d, int32_t* topk_idx_dev,
                                     float* topk_w_dev, int32_t* counts_dev,
                                     int32_t* offsets_dev, int32_t* perm_dev, void* stream);

/*
 * Where moe_forward keeps its intermediates inside the workspace (byte
 * offsets from the workspace base), so that a caller can read them after a
 * call for inspection: logits [T][E] f32, topk_idx [T][k] i32, topk_w [T][k]
 * f32, counts [E] i32, offsets [E+1] i32, perm [T*k] i32 (pair id at each
 * permuted row), xp [T*k][d] bf16 (permuted activations), h [T*k][I] bf16
 * (SwiGLU hidden rows in permuted order), yw [T*k][d] fp32 (p-weighted expert
 * outputs in pair order t*k+j). Rows of xp and h keep each run of 8
 * consecutive elements in the order 0,4,1,5,2,6,3,7 (the operand order of the
 * grouped GEMMs). Returns MOE_ERR_INVALID_ARG for bad shapes.
 */
typedef struct {
  size_t logits, topk_idx, topk_w, counts, offsets, perm, xp, h, yw, status, total;
  /* the block-scaled tiles' B-scale blocks of the x rows and of the H rows
   * (E8M0 bytes in the layout the GEMMs copy into tensor memory) */
  size_t x_scales, h_scales;
} moe_ws_layout;
MOE_API moe_status moe_workspace_layout(int E, int k, int T, int d, int I, moe_ws_layout* layout);

/*
 * The activation split of the block-scaled tiles (tile policy 4), on plain
 * rows: x_dev [rows][K] bf16 -> hi_dev, lo_dev [rows][K] E4M3 bytes and
 * scales_dev [rows][K/32][2] E8M0 bytes (hi, lo) such that, per group of 32,
 * x = 2^(s_hi-127) e4m3(hi) + 2^(s_lo-127) e4m3(lo), exactly for every
 * element of at least 2^-13 of the group's max |x| and within 2^-21 of that
 * max otherwise (for groups whose max |x| is at least 2^-116). The pages have no counterpart: the split only lets bf16
 * activations enter the tensor core's block-scaled MMA kind next to E2M1
 * weights ("Four-bit expert weights"). K a multiple of 32; x_dev, hi_dev and
 * lo_dev 16-byte aligned. All buffers are the caller's.
 */
MOE_API moe_status moe_mx_split_e4m3(const void* x_dev, int rows, int K, uint8_t* hi_dev,
                                     uint8_t* lo_dev, uint8_t* scales_dev, void* stream);

/*
 * The activation conversion of the quantised modes (moe_forward_opts.act_quant)
 * on plain rows, with the kernels the layer uses: x_dev [rows][K] bf16 ->
 * q_dev [rows][K] E4M3 bytes (MOE_ACT_MXFP8) or [rows][K/2] packed E2M1 codes
 * (MOE_ACT_MXFP4; byte b holds element 2b in its low nibble, as the weights),
 * and scales_dev [rows][K/32] E8M0 bytes, per group of 32: the OCP
 * Microscaling conversion (v1.0, section 6.3) with shared scale
 * 2^(floor(log2 max|x|) - emax), emax 8 (E4M3) or 2 (E2M1), elements rounded
 * to nearest even and clamped to the largest normal. A group whose max|x| is
 * below 2^(emax - 127) keeps the smallest scale byte, 0; an all-zero group
 * gets byte 127 and zero codes. The pages have no counterpart: they put only
 * the expert weights in MXFP4 ("Four-bit expert weights"). K a multiple of 32;
 * x_dev and q_dev 16-byte aligned; all buffers the caller's.
 */
MOE_API moe_status moe_mx_quantize(const void* x_dev, int rows, int K, int act_quant,
                                   uint8_t* q_dev, uint8_t* scales_dev, void* stream);

/*
 * Decode MXFP4 rows to bf16 on the device with the same decoder the grouped
 * GEMMs use ("Four-bit expert weights"). codes_dev [rows][K/2], scales_dev
 * [rows][K/32] -> out_dev [rows][K] bf16. K must be a multiple of 32.
 */
MOE_API moe_status moe_mxfp4_to_bf16(const uint8_t* codes_dev, const uint8_t* scales_dev,
                             int rows, int K, void* out_dev, void* stream);

/*
 * Synchronise `stream`, then read and clear the device status word in the
 * workspace. Returns MOE_OK, or MOE_ERR_TIMEOUT when a kernel gave up a wait.
 */
MOE_API moe_status moe_sync_status(void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * Failure-detection self-test: enqueues one kernel whose only thread waits,
 * with the same bounded wait the GEMM roles use, on an mbarrier that nothing
 * completes. After about two seconds the wait gives up and stores
 * MOE_ERR_TIMEOUT in the status word at the start of workspace_dev (16 bytes
 * suffice), which moe_sync_status() then returns. Nothing hangs or faults.
 */
MOE_API moe_status moe_selftest_wait_timeout(void* workspace_dev, void* stream);

/*
 * The MoE sublayer of a decoder block with its pre-norm and residual add
 * (field guide "gpt-oss 20B", "04 One decoder block": RMSNorm is applied
 * before the MoE and the sublayer is added back to the residual stream):
 *   x   = bf16((h / sqrt(mean(h^2) + eps)) * g)   per row (moe_rms_norm)
 *   out = bf16(h + sum_j p_j E_j(x))              (one rounding, after the add)
 * h_dev [T][d] bf16 (the residual stream), g_dev [d] f32 (the norm's gain),
 * eps >= 0 (the pages give no value; gpt-oss configurations commonly use
 * 1e-5); gu_bias_dev and down_bias_dev (each may be NULL) are the experts'
 * biases as in moe_forward_biased. All other arguments, the result, the errors
 * and the stream semantics are those of moe_forward; the workspace must hold
 * moe_workspace_size_block(...) bytes (moe_forward's, plus the x rows).
 * moe_forward_launch_count(...) + 1 launches.
 */
MOE_API size_t moe_workspace_size_block(int E, int k, int T, int d, int I);
MOE_API moe_status moe_forward_block(const void* h_dev, const float* g_dev, float eps,
                                     const float* W_r_dev, const float* b_r_dev,
                                     const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                                     const float* gu_bias_dev, const uint8_t* Wd_codes_dev,
                                     const uint8_t* Wd_scales_dev, const float* down_bias_dev,
                                     int E, int k, int T, int d, int I, void* out_dev,
                                     void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * The pre-MoE RMSNorm alone: x_dev[t] = bf16((h[t] / sqrt(mean(h[t]^2) + eps)) * g),
 * h_dev and x_dev [T][d] bf16, g_dev [d] f32; d a multiple of 32; all three
 * 16-byte aligned and the caller's. Per row: fp32 sum of squares (a fixed
 * lane-strided order), IEEE sqrt and division, one rounding to bf16.
 */
MOE_API moe_status moe_rms_norm(const void* h_dev, const float* g_dev, float eps, int T, int d,
                                void* x_dev, void* stream);

/*
 * Number of kernel launches one moe_forward call enqueues for this shape
 * under the current tile policy (0 for T = 0), assuming 32-byte aligned code
 * arrays. Used to count device work per step.
 */
MOE_API int moe_forward_launch_count(int E, int k, int T, int d, int I);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
