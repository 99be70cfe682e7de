// moe_abi.cu -- the extern "C" boundary: argument checks, workspace layout,
// and the launch sequence of the MoE forward pass on the caller's stream.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxDevices = 64;

// Process default of the grouped-GEMM tile policy (moe_set_tile_policy):
// 0 = choose by shape, 1 = single-CTA tiles, 2 = CTA-pair tiles,
// 3 = swapped-operand tiles, 4 = block-scaled tiles. Calls through
// moe_forward_ex carry their own policy and never read it.
std::atomic<int> g_tile_policy{0};

// The block-scaled path reads the codes through 4-bit tensor maps: rows of a
// multiple of 64 elements (at least 128) and 32-byte aligned code arrays.
bool mx_shape_ok(int d, int I) {
  return d % 64 == 0 && I % 64 == 0 && d >= 128 && I >= 128 && d <= moe::kMxMaxK &&
         I <= moe::kMxMaxK;
}
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31) == 0; }

int choose_tiles(int policy, int P, int E, bool mx_ok) {
  if (policy == 4 && mx_ok) return moe::TILES_MX;
  if (policy == 5 && mx_ok) return moe::TILES_MX_PAIR;
  if (policy >= 1 && policy <= 3) return policy;
  const int64_t p = P, e = E;
  // Few routed rows per expert (decode): stream the weights, with the
  // block-scaled tiles where the shape allows (no CUDA-core weight decode),
  // else the swapped-operand kernel. From ~192 rows per expert CTA-pair tiles
  // (the block-scaled ones where the shape allows: 1.79 against 2.10 ms per
  // 20b step at T = 8192); in between the single-CTA bf16 tiles, which skip
  // empty 128-row halves.
  if (p < 32 * e) return mx_ok ? moe::TILES_MX : moe::TILES_SWAP;
  if (p >= 192 * e) return mx_ok ? moe::TILES_MX_PAIR : moe::TILES_PAIR;
  return moe::TILES_SINGLE;
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// The block-scaled path's buffers share regions with the bf16 path's (one
// forward call uses one path): the hi/lo token rows live in the xp region,
// the hi/lo H rows in the h region, the B-scale blocks in the two regions of
// transposed weight scales; each region is sized for the larger use.
struct Layout {
  moe_ws_layout pub;
  size_t mprefix, chunk_hist, chunk_base, x_in, out_buf, gu_scales_t, d_scales_t;
  size_t router_terms;   // the router's bf16 weight terms and row norms
  size_t inv;            // permuted row of each (token, slot) pair
  size_t mx_tok_rows;
  size_t wsfb;     // the CTA-pair down GEMM's weight-scale atoms
  size_t x_norm;   // moe_forward_block: the normalised rows [T][d] bf16
};

bool shape_ok(int E, int k, int T, int d) {
  if (E < 1 || E > 256) return false;
  if (k < 1 || k > E || k > 32) return false;
  if (T < 0) return false;
  if (d < 32 || d > 16384 || d % 32) return false;
  if (static_cast<int64_t>(T) * k >= (static_cast<int64_t>(1) << 31)) return false;
  return true;
}

bool full_shape_ok(int E, int k, int T, int d, int I) {
  return shape_ok(E, k, T, d) && I >= 32 && I <= 16384 && I % 32 == 0;
}

void make_layout(int E, int k, int T, int d, int I, bool hostio, Layout* L, bool block = false) {
  const size_t P = static_cast<size_t>(T) * k;
  const size_t NB = static_cast<size_t>(moe::perm_chunks(T));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + (bytes ? bytes : 1));
    return o;
  };
  memset(L, 0, sizeof(*L));
  L->pub.status = take(16);
  L->pub.logits = take(static_cast<size_t>(T) * E * 4);
  L->pub.topk_idx = take(P * 4);
  L->pub.topk_w = take(P * 4);
  L->pub.counts = take(static_cast<size_t>(E) * 4);
  L->pub.offsets = take(static_cast<size_t>(E + 1) * 4);
  L->mprefix = take(static_cast<size_t>(E + 1) * 4);
  L->chunk_hist = take(NB * E * 4);
  L->chunk_base = take(NB * E * 4);
  L->pub.perm = take(P * 4);
  L->inv = take(P * 4);
  L->router_terms = take(moe::router_tc_scratch_bytes(E, d, T));
  const size_t tr = moe::mx_tok_rows(static_cast<int>(P), E);
  L->mx_tok_rows = tr;
  auto larger = [](size_t a, size_t b) { return a > b ? a : b; };
  L->pub.xp = take(larger(P * d * 2, 2 * tr * d));
  L->pub.h = take(larger(P * static_cast<size_t>(I) * 2, 2 * tr * I));
  L->pub.yw = take(P * d * 4);
  L->gu_scales_t = take(larger(static_cast<size_t>(E) * 2 * I * (d / 32),
                               moe::mx_sfb_bytes(static_cast<int>(P), E, d)));
  L->d_scales_t = take(larger(static_cast<size_t>(E) * d * (I / 32),
                              moe::mx_sfb_bytes(static_cast<int>(P), E, I)));
  L->wsfb = take(moe::mx_pair_down_atom_bytes(E, d, I));
  if (hostio) {
    L->x_in = take(static_cast<size_t>(T) * d * 2);
    L->out_buf = take(static_cast<size_t>(T) * d * 2);
  }
  if (block) L->x_norm = take(static_cast<size_t>(T) * d * 2);
  L->pub.total = off;
  L->pub.x_scales = L->gu_scales_t;
  L->pub.h_scales = L->d_scales_t;
}

void make_route_layout(int E, int k, int T, int d, Layout* L) {
  const size_t NB = static_cast<size_t>(moe::perm_chunks(T));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + (bytes ? bytes : 1));
    return o;
  };
  (void)k;
  (void)d;
  memset(L, 0, sizeof(*L));
  L->pub.status = take(16);
  L->pub.logits = take(static_cast<size_t>(T) * E * 4);
  L->mprefix = take(static_cast<size_t>(E + 1) * 4);
  L->chunk_hist = take(NB * E * 4);
  L->chunk_base = take(NB * E * 4);
  L->pub.offsets = take(static_cast<size_t>(E + 1) * 4);  // used when the caller passes none
  L->router_terms = take(moe::router_tc_scratch_bytes(E, d, T));
  L->pub.total = off;
}

// Host-buffer calls on batches of at least kHostioChunkMin tokens split the
// tokens into kHostioChunks chunks (each token's output depends on that token
// alone, so the result is the same): the copy in of one chunk, the forward of
// another and the copy out of a third overlap. Two chunk workspaces alternate;
// the input and output rows of the whole batch are staged in the workspace.
constexpr int kHostioChunks = 4;
constexpr int kHostioChunkMin = 2048;

struct HostioPlan {
  int chunks, Tc;
  Layout sub;          // layout of one chunk workspace (Tc tokens)
  size_t sub_stride;   // bytes between the two chunk workspaces
  size_t x_in, out_buf, total;
};

void make_hostio_plan(int E, int k, int T, int d, int I, HostioPlan* hp) {
  memset(hp, 0, sizeof(*hp));
  hp->chunks = T >= kHostioChunkMin ? kHostioChunks : 1;
  if (hp->chunks == 1) {
    make_layout(E, k, T, d, I, true, &hp->sub);
    hp->Tc = T;
    hp->x_in = hp->sub.x_in;
    hp->out_buf = hp->sub.out_buf;
    hp->total = hp->sub.pub.total;
    return;
  }
  hp->Tc = (T + hp->chunks - 1) / hp->chunks;
  make_layout(E, k, hp->Tc, d, I, false, &hp->sub);
  hp->sub_stride = align256(hp->sub.pub.total);
  const size_t rows = static_cast<size_t>(T) * d * 2;
  hp->x_in = 2 * hp->sub_stride;
  hp->out_buf = align256(hp->x_in + rows);
  hp->total = align256(hp->out_buf + rows);
  // a workspace sized for host-buffer calls also serves moe_forward
  Layout full;
  make_layout(E, k, T, d, I, false, &full);
  if (hp->total < full.pub.total) hp->total = full.pub.total;
}

// Status word of host-buffer chunk c: word c of the 16-byte status block at
// the start of the workspace (chunk 0's workspace), one word per chunk.
int* chunk_status(void* ws, const HostioPlan& hp, int c) {
  static_assert(kHostioChunks * sizeof(int) <= 16, "chunk status words fit the status block");
  return reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + hp.sub.pub.status) + c;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Device capability and SM count, cached per device.
moe_status device_info(int* num_sms) {
  static int sms[kMaxDevices] = {0};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  if (dev < kMaxDevices && sms[dev] > 0) {
    *num_sms = sms[dev];
    return MOE_OK;
  }
  int major = 0, minor = 0, n = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  if (major != 10 || minor != 0) return MOE_ERR_NO_DEVICE;  // built for sm_100a only
  if (dev < kMaxDevices) sms[dev] = n;
  *num_sms = n;
  return MOE_OK;
}

#define MOE_CUDA(call)                        \
  do {                                        \
    if ((call) != cudaSuccess) {              \
      cudaGetLastError();                     \
      return MOE_ERR_CUDA;                    \
    }                                         \
  } while (0)

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

moe_status check_forward_args(const void* x, const float* W_r, const float* b_r,
                              const uint8_t* gc, const uint8_t* gs, const uint8_t* dc,
                              const uint8_t* ds, int E, int k, int T, int d, int I,
                              const void* out, const void* ws) {
  if (!x || !W_r || !b_r || !gc || !gs || !dc || !ds || !out || !ws) return MOE_ERR_INVALID_ARG;
  if (E < 1 || k < 1 || T < 0 || d < 1 || I < 1) return MOE_ERR_INVALID_ARG;
  if (!full_shape_ok(E, k, T, d, I)) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(W_r) || !aligned16(b_r) || !aligned16(gc) || !aligned16(gs) ||
      !aligned16(dc) || !aligned16(ds) || !aligned16(out) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Optional per-launch event recording (moe_forward_timed): ev[i] is recorded
// before launch i, ev[kStages] after the last one; a null ev[i] is skipped.
constexpr int kStages = 11;

struct StageEvents {
  cudaEvent_t ev[kStages + 1];
  cudaStream_t st;
  void mark(int i) const {
    if (ev[i]) cudaEventRecord(ev[i], st);
  }
};

// Launches of the router (logits, top-k, softmax) and, when perm is given, the
// permutation (counts, offsets, M-tile prefix, perm). Batches of at most
// kPermChunk tokens take one fused launch for the permutation (identical
// results). ev marks launches 0..5 of moe_forward_timed.
// The launches of one pass: the first is ordered after everything earlier on
// the stream as usual; the rest use programmatic dependent launch (see
// moe::launch_kernel). Cleared again when the pass's launches are done.
struct PdlPass {
  PdlPass() { moe::pdl_launches() = false; }
  ~PdlPass() { moe::pdl_launches() = false; }
};

moe_status launch_routing(const uint16_t* x, const float* W_r, const float* b_r, int E, int k,
                          int T, int d, float* logits, void* router_terms, int32_t* topk_idx,
                          float* topk_w, int32_t* counts, int32_t* offsets, int32_t* mprefix,
                          int32_t* chunk_hist, int32_t* chunk_base, int32_t* perm, int* status,
                          cudaStream_t st, const StageEvents& ev, int32_t* inv = nullptr) {
  const bool small = T <= moe::kPermChunk;
  ev.mark(0);
  {
    // the router: weight split, tensor-core logits, top-k and softmax (its
    // stage time covers all three launches; the top-k stage reads 0); for
    // at most kPermChunk tokens the top-k kernel's last block also builds the
    // permutation
    moe::pdl_launches() = false;
    cudaError_t e = moe::launch_router_tc(x, W_r, b_r, T, E, k, d, router_terms, logits, topk_idx,
                                          topk_w, status, st, small ? counts : nullptr,
                                          small ? offsets : nullptr, small ? mprefix : nullptr,
                                          small ? perm : nullptr);
    moe::pdl_launches() = true;
    MOE_CUDA(e);
    ev.mark(1);
  }
  ev.mark(2);
  if (!perm) return MOE_OK;
  if (small) {
    ev.mark(3);
    ev.mark(4);
  } else {
    MOE_CUDA(moe::launch_perm_hist(topk_idx, T, k, E, chunk_hist, st));
    ev.mark(3);
    MOE_CUDA(moe::launch_perm_scan(chunk_hist, moe::perm_chunks(T), E, counts, offsets, chunk_base,
                                   mprefix, st));
    ev.mark(4);
    MOE_CUDA(moe::launch_perm_scatter(topk_idx, T, k, E, chunk_base, perm, inv, st));
  }
  ev.mark(5);
  return MOE_OK;
}

// The forward pass on the caller's stream. resid (optional, [T][d] bf16) is
// added to the layer output before its rounding to bf16; gu_bias ([E][2I]) and
// dn_bias ([E][d]), each optional, are the experts' projection biases.
// What a forward call may choose besides its tensors: the tile policy (as
// moe_set_tile_policy; the process default for the entry points without
// options), the experts' optional biases, and where the status word lives
// (null: the workspace's own).
struct FwdOpts {
  int policy;
  int act;                 // moe::ACT_HILO (bf16 precision), ACT_E4M3 or ACT_E2M1
  const float* gu_bias;
  const float* dn_bias;
  int* status;
};

FwdOpts default_opts() {
  FwdOpts o;
  o.policy = g_tile_policy.load(std::memory_order_relaxed);
  o.act = moe::ACT_HILO;
  o.gu_bias = nullptr;
  o.dn_bias = nullptr;
  o.status = nullptr;
  return o;
}

// Per-call options -> FwdOpts (NULL: the defaults), checked before any launch.
moe_status parse_opts(const moe_forward_opts* opts, int d, int I, const uint8_t* gc,
                      const uint8_t* dc, FwdOpts* out) {
  FwdOpts o = default_opts();
  if (opts) {
    if (opts->tile_policy < -1 || opts->tile_policy > 5) return MOE_ERR_INVALID_ARG;
    if (opts->act_quant < MOE_ACT_BF16 || opts->act_quant > MOE_ACT_MXFP4)
      return MOE_ERR_INVALID_ARG;
    if (opts->act_quant != MOE_ACT_BF16) {
      // the quantised modes run on the block-scaled tiles only
      if (!mx_shape_ok(d, I) || !aligned32(gc) || !aligned32(dc)) return MOE_ERR_UNSUPPORTED;
      o.act = opts->act_quant == MOE_ACT_MXFP8 ? moe::ACT_E4M3 : moe::ACT_E2M1;
    }
    if (opts->tile_policy >= 0) o.policy = opts->tile_policy;
    o.gu_bias = opts->gu_bias_dev;
    o.dn_bias = opts->down_bias_dev;
  }
  if (!aligned16(o.gu_bias) || !aligned16(o.dn_bias)) return MOE_ERR_INVALID_ARG;
  *out = o;
  return MOE_OK;
}

moe_status run_forward(const uint16_t* x, const float* W_r, const float* b_r, const uint8_t* gc,
                       const uint8_t* gs, const uint8_t* dc, const uint8_t* ds, int E, int k,
                       int T, int d, int I, uint16_t* out, void* ws, const Layout& L,
                       cudaStream_t st, int num_sms, const FwdOpts& opt,
                       const StageEvents* tev = nullptr, const uint16_t* resid = nullptr) {
  StageEvents none;
  memset(&none, 0, sizeof(none));
  const StageEvents& E_ = tev ? *tev : none;
  PdlPass pdl_pass;
  const float* gu_bias = opt.gu_bias;
  const float* dn_bias = opt.dn_bias;
  const int P = T * k;
  int* status = opt.status ? opt.status : at<int>(ws, L.pub.status);
  float* logits = at<float>(ws, L.pub.logits);
  int32_t* topk_idx = at<int32_t>(ws, L.pub.topk_idx);
  float* topk_w = at<float>(ws, L.pub.topk_w);
  int32_t* counts = at<int32_t>(ws, L.pub.counts);
  int32_t* offsets = at<int32_t>(ws, L.pub.offsets);
  int32_t* mprefix = at<int32_t>(ws, L.mprefix);
  int32_t* chunk_hist = at<int32_t>(ws, L.chunk_hist);
  int32_t* chunk_base = at<int32_t>(ws, L.chunk_base);
  int32_t* perm = at<int32_t>(ws, L.pub.perm);
  uint16_t* xp = at<uint16_t>(ws, L.pub.xp);
  uint16_t* h = at<uint16_t>(ws, L.pub.h);
  float* yw = at<float>(ws, L.pub.yw);
  uint8_t* gst = at<uint8_t>(ws, L.gu_scales_t);
  uint8_t* dst_ = at<uint8_t>(ws, L.d_scales_t);

  moe_status rs = launch_routing(x, W_r, b_r, E, k, T, d, logits, at<void>(ws, L.router_terms),
                                 topk_idx, topk_w, counts, offsets, mprefix, chunk_hist,
                                 chunk_base, perm, status, st, E_, at<int32_t>(ws, L.inv));
  if (rs != MOE_OK) return rs;
  const int tiles = opt.act != moe::ACT_HILO
                        ? moe::TILES_MX
                        : choose_tiles(opt.policy, P, E,
                                       mx_shape_ok(d, I) && aligned32(gc) && aligned32(dc));
  if (opt.act != moe::ACT_HILO) {
    // quantised activations (w4a8, w4a4): one MX-converted row per routed
    // pair, the same block-scaled kernels with a one-term B operand
    uint8_t* qx = at<uint8_t>(ws, L.pub.xp);
    uint8_t* qh = at<uint8_t>(ws, L.pub.h);
    uint8_t* sfbx = at<uint8_t>(ws, L.gu_scales_t);
    uint8_t* sfbh = at<uint8_t>(ws, L.d_scales_t);
    // few rows per expert: 16-token tiles; else 128-token tiles, on a CTA
    // pair when the policy asks for it
    const int variant =
        P < 64 * E ? moe::kMxSmall
                   : ((opt.policy == 5 || (opt.policy == 0 && P >= 192 * E)) ? moe::kMxPair
                                                                              : moe::kMxLarge);
    // E2M1 activations on the CTA pair run the kind::mxf4 kernel (both
    // operands packed, 256-wide k-blocks) where d and I allow it
    const int act = (opt.act == moe::ACT_E2M1 && variant == moe::kMxPair && d >= 256 && I >= 256)
                        ? moe::ACT_F4
                        : opt.act;
    MOE_CUDA(moe::launch_mx_act_quant_gather(variant, act, x, perm, offsets, E, P, k, d, qx, sfbx,
                                             st));
    E_.mark(6);
    E_.mark(7);
    E_.mark(8);
    moe::MxGemmProblem m1;
    memset(&m1, 0, sizeof(m1));
    m1.codes = gc;
    m1.scales = gs;
    m1.b_hi = qx;
    m1.b_sfb = sfbx;
    m1.offsets = offsets;
    m1.P = P;
    m1.E = E;
    m1.K = d;
    m1.I = I;
    m1.tok_rows = static_cast<int>(L.mx_tok_rows);
    m1.h_hi = qh;
    m1.h_sfb = sfbh;
    m1.n_out = I;
    m1.status = status;
    m1.bias = gu_bias;
    m1.act = act;
    MOE_CUDA(variant == moe::kMxPair ? moe::launch_mx_pair_gateup_swiglu(m1, num_sms, st)
                                     : moe::launch_mx_gemm_gateup_swiglu(variant, m1, num_sms, st));
    E_.mark(9);
    moe::MxGemmProblem m2 = m1;
    m2.codes = dc;
    m2.scales = ds;
    m2.b_hi = qh;
    m2.b_sfb = sfbh;
    m2.K = I;
    m2.h_hi = nullptr;
    m2.h_sfb = nullptr;
    m2.out_f32 = yw;
    m2.wsfb = at<uint8_t>(ws, L.wsfb);   // CTA pair, 8-bit activations
    m2.perm = perm;
    m2.topk_w = topk_w;
    m2.n_out = d;
    m2.bias = dn_bias;
    MOE_CUDA(variant == moe::kMxPair ? moe::launch_mx_pair_down(m2, num_sms, st)
                                     : moe::launch_mx_gemm_down(variant, m2, num_sms, st));
    E_.mark(10);
    MOE_CUDA(moe::launch_combine(yw, T, k, d, resid, out, st));
    E_.mark(11);
    return MOE_OK;
  }
  if (tiles == moe::TILES_MX || tiles == moe::TILES_MX_PAIR) {
    // block-scaled path: hi/lo token rows, no scale transposes
    const size_t tr = L.mx_tok_rows;
    uint8_t* qx = at<uint8_t>(ws, L.pub.xp);
    uint8_t* qh = at<uint8_t>(ws, L.pub.h);
    uint8_t* sfbx = at<uint8_t>(ws, L.gu_scales_t);
    uint8_t* sfbh = at<uint8_t>(ws, L.d_scales_t);
    // 16-token tiles while experts average under 64 rows, else 120-token
    // tiles, or 256-token tiles on a CTA pair
    const int variant = tiles == moe::TILES_MX_PAIR ? moe::kMxPair
                                                    : (P < 64 * E ? moe::kMxSmall : moe::kMxLarge);
    // token-major when the three-launch permutation wrote the inverse (more
    // than kPermChunk tokens), else row-major
    const bool inv_ok = T > moe::kPermChunk;
    MOE_CUDA(moe::launch_mx_quant_gather(variant, x, perm, offsets, E, P, k, d, qx, qx + tr * d,
                                         sfbx, inv_ok ? topk_idx : nullptr,
                                         inv_ok ? at<int32_t>(ws, L.inv) : nullptr, T, st));
    E_.mark(6);
    E_.mark(7);
    E_.mark(8);
    moe::MxGemmProblem m1;
    memset(&m1, 0, sizeof(m1));
    m1.codes = gc;
    m1.scales = gs;
    m1.b_hi = qx;
    m1.b_lo = qx + tr * d;
    m1.b_sfb = sfbx;
    m1.offsets = offsets;
    m1.P = P;
    m1.E = E;
    m1.K = d;
    m1.I = I;
    m1.tok_rows = static_cast<int>(tr);
    m1.h_hi = qh;
    m1.h_lo = qh + tr * I;
    m1.h_sfb = sfbh;
    m1.n_out = I;
    m1.status = status;
    m1.bias = gu_bias;
    MOE_CUDA(variant == moe::kMxPair ? moe::launch_mx_pair_gateup_swiglu(m1, num_sms, st)
                                     : moe::launch_mx_gemm_gateup_swiglu(variant, m1, num_sms, st));
    E_.mark(9);
    moe::MxGemmProblem m2 = m1;
    m2.codes = dc;
    m2.scales = ds;
    m2.b_hi = qh;
    m2.b_lo = qh + tr * I;
    m2.b_sfb = sfbh;
    m2.K = I;
    m2.h_hi = nullptr;
    m2.h_lo = nullptr;
    m2.h_sfb = nullptr;
    m2.out_f32 = yw;
    m2.wsfb = at<uint8_t>(ws, L.wsfb);   // CTA pair, 8-bit activations
    m2.perm = perm;
    m2.topk_w = topk_w;
    m2.n_out = d;
    m2.bias = dn_bias;
    MOE_CUDA(variant == moe::kMxPair ? moe::launch_mx_pair_down(m2, num_sms, st)
                                     : moe::launch_mx_gemm_down(variant, m2, num_sms, st));
    E_.mark(10);
    MOE_CUDA(moe::launch_combine(yw, T, k, d, resid, out, st));
    E_.mark(11);
    return MOE_OK;
  }
  MOE_CUDA(moe::launch_gather_rows(x, perm, P, k, d, xp, st));
  E_.mark(6);
  MOE_CUDA(moe::launch_transpose_scales(gs, E, 2 * I, d / 32, counts, gst, st));
  E_.mark(7);
  MOE_CUDA(moe::launch_transpose_scales(ds, E, d, I / 32, counts, dst_, st));
  E_.mark(8);

  moe::GroupedGemmProblem g1;
  g1.A = xp;
  g1.codes = gc;
  g1.scales_t = gst;
  g1.offsets = offsets;
  g1.mprefix = mprefix;
  g1.P = P;
  g1.E = E;
  g1.K = d;
  g1.Nrows = 2 * I;
  g1.out = h;
  g1.out_f32 = nullptr;
  g1.perm = nullptr;
  g1.topk_w = nullptr;
  g1.n_out = I;
  g1.status = status;
  g1.tiles = tiles;
  g1.bias = gu_bias;
  MOE_CUDA(moe::launch_gemm_gateup_swiglu(g1, num_sms, st));
  E_.mark(9);

  moe::GroupedGemmProblem g2 = g1;
  g2.A = h;
  g2.codes = dc;
  g2.scales_t = dst_;
  g2.K = I;
  g2.Nrows = d;
  g2.out = nullptr;
  g2.out_f32 = yw;
  g2.perm = perm;
  g2.topk_w = topk_w;
  g2.n_out = d;
  g2.bias = dn_bias;
  MOE_CUDA(moe::launch_gemm_down_combine(g2, num_sms, st));
  E_.mark(10);
  MOE_CUDA(moe::launch_combine(yw, T, k, d, resid, out, st));
  E_.mark(11);
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_NO_DEVICE: return "MOE_ERR_NO_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

int moe_version(void) { return kVersion; }

moe_status moe_set_tile_policy(int policy) {
  if (policy < 0 || policy > 5) return MOE_ERR_INVALID_ARG;
  g_tile_policy.store(policy, std::memory_order_relaxed);
  return MOE_OK;
}

size_t moe_workspace_size(int E, int k, int T, int d, int I) {
  if (!full_shape_ok(E, k, T, d, I)) return 0;
  Layout L;
  make_layout(E, k, T, d, I, false, &L);
  return L.pub.total;
}

size_t moe_workspace_size_hostio(int E, int k, int T, int d, int I) {
  if (!full_shape_ok(E, k, T, d, I)) return 0;
  HostioPlan hp;
  make_hostio_plan(E, k, T, d, I, &hp);
  return hp.total;
}

moe_status moe_workspace_layout(int E, int k, int T, int d, int I, moe_ws_layout* layout) {
  if (!layout || !full_shape_ok(E, k, T, d, I)) return MOE_ERR_INVALID_ARG;
  Layout L;
  make_layout(E, k, T, d, I, false, &L);
  *layout = L.pub;
  return MOE_OK;
}

int moe_forward_launch_count(int E, int k, int T, int d, int I) {
  if (!full_shape_ok(E, k, T, d, I) || T == 0) return 0;
  int n = 12;
  // small batches: the permutation inside the router's top-k launch
  if (T <= moe::kPermChunk) n -= 3;
  // the block-scaled path launches no scale transposes
  const int tiles =
      choose_tiles(g_tile_policy.load(std::memory_order_relaxed), T * k, E, mx_shape_ok(d, I));
  if (tiles == moe::TILES_MX || tiles == moe::TILES_MX_PAIR) n -= 2;
  // the CTA-pair down GEMM lays out its weight-scale atoms first
  if (tiles == moe::TILES_MX_PAIR) n += 1;
  return n;
}

moe_status moe_forward(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                       const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                       const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev, int E, int k,
                       int T, int d, int I, void* out_dev, void* workspace_dev,
                       size_t workspace_bytes, void* stream) {
  return moe_forward_biased(x_dev, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev, nullptr,
                            Wd_codes_dev, Wd_scales_dev, nullptr, E, k, T, d, I, out_dev,
                            workspace_dev, workspace_bytes, stream);
}

moe_status moe_forward_biased(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                              const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                              const float* gu_bias_dev, const uint8_t* Wd_codes_dev,
                              const uint8_t* Wd_scales_dev, const float* down_bias_dev, int E,
                              int k, int T, int d, int I, void* out_dev, void* workspace_dev,
                              size_t workspace_bytes, void* stream) {
  moe_forward_opts o;
  memset(&o, 0, sizeof(o));
  o.tile_policy = -1;
  o.gu_bias_dev = gu_bias_dev;
  o.down_bias_dev = down_bias_dev;
  return moe_forward_ex(x_dev, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev, Wd_codes_dev,
                        Wd_scales_dev, E, k, T, d, I, out_dev, workspace_dev, workspace_bytes, &o,
                        stream);
}

moe_status moe_forward_ex(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                          const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                          const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev, int E, int k,
                          int T, int d, int I, void* out_dev, void* workspace_dev,
                          size_t workspace_bytes, const moe_forward_opts* opts, void* stream) {
  moe_status s = check_forward_args(x_dev, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev,
                                    Wd_codes_dev, Wd_scales_dev, E, k, T, d, I, out_dev,
                                    workspace_dev);
  if (s != MOE_OK) return s;
  FwdOpts o;
  if ((s = parse_opts(opts, d, I, Wgu_codes_dev, Wd_codes_dev, &o)) != MOE_OK) return s;
  Layout L;
  make_layout(E, k, T, d, I, false, &L);
  if (workspace_bytes < L.pub.total) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  int num_sms = 0;
  if ((s = device_info(&num_sms)) != MOE_OK) return s;
  return run_forward(static_cast<const uint16_t*>(x_dev), W_r_dev, b_r_dev, Wgu_codes_dev,
                     Wgu_scales_dev, Wd_codes_dev, Wd_scales_dev, E, k, T, d, I,
                     static_cast<uint16_t*>(out_dev), workspace_dev, L,
                     static_cast<cudaStream_t>(stream), num_sms, o);
}

size_t moe_workspace_size_block(int E, int k, int T, int d, int I) {
  if (!full_shape_ok(E, k, T, d, I)) return 0;
  Layout L;
  make_layout(E, k, T, d, I, false, &L, true);
  return L.pub.total;
}

moe_status moe_rms_norm(const void* h_dev, const float* g_dev, float eps, int T, int d,
                        void* x_dev, void* stream) {
  if (!h_dev || !g_dev || !x_dev || T < 0 || d < 32 || d % 32 || !(eps >= 0.f))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(h_dev) || !aligned16(g_dev) || !aligned16(x_dev)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  int num_sms = 0;
  moe_status s = device_info(&num_sms);
  if (s != MOE_OK) return s;
  MOE_CUDA(moe::launch_rms_norm(static_cast<const uint16_t*>(h_dev), g_dev, eps, T, d,
                                static_cast<uint16_t*>(x_dev), static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_forward_block(const void* h_dev, const float* g_dev, float eps, const float* W_r_dev,
                             const float* b_r_dev, const uint8_t* Wgu_codes_dev,
                             const uint8_t* Wgu_scales_dev, const float* gu_bias_dev,
                             const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev,
                             const float* down_bias_dev, int E, int k, int T, int d, int I,
                             void* out_dev, void* workspace_dev, size_t workspace_bytes,
                             void* stream) {
  moe_status s = check_forward_args(h_dev, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev,
                                    Wd_codes_dev, Wd_scales_dev, E, k, T, d, I, out_dev,
                                    workspace_dev);
  if (s != MOE_OK) return s;
  if (!g_dev || !aligned16(g_dev) || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(gu_bias_dev) || !aligned16(down_bias_dev)) return MOE_ERR_INVALID_ARG;
  Layout L;
  make_layout(E, k, T, d, I, false, &L, true);
  if (workspace_bytes < L.pub.total) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  int num_sms = 0;
  if ((s = device_info(&num_sms)) != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint16_t* h = static_cast<const uint16_t*>(h_dev);
  uint16_t* x = at<uint16_t>(workspace_dev, L.x_norm);
  MOE_CUDA(moe::launch_rms_norm(h, g_dev, eps, T, d, x, st));
  FwdOpts o = default_opts();
  o.gu_bias = gu_bias_dev;
  o.dn_bias = down_bias_dev;
  return run_forward(x, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev, Wd_codes_dev,
                     Wd_scales_dev, E, k, T, d, I, static_cast<uint16_t*>(out_dev), workspace_dev,
                     L, st, num_sms, o, nullptr, h);
}

moe_status moe_forward_hostio(const void* x_host, const float* W_r_dev, const float* b_r_dev,
                              const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                              const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev, int E,
                              int k, int T, int d, int I, void* out_host, void* workspace_dev,
                              size_t workspace_bytes, void* stream) {
  moe_status s = check_forward_args(x_host, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev,
                                    Wd_codes_dev, Wd_scales_dev, E, k, T, d, I, out_host,
                                    workspace_dev);
  if (s != MOE_OK) return s;
  HostioPlan hp;
  make_hostio_plan(E, k, T, d, I, &hp);
  if (workspace_bytes < hp.total) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  int num_sms = 0;
  if ((s = device_info(&num_sms)) != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint16_t* x_in = at<uint16_t>(workspace_dev, hp.x_in);
  uint16_t* out_buf = at<uint16_t>(workspace_dev, hp.out_buf);
  const uint16_t* xh = static_cast<const uint16_t*>(x_host);
  uint16_t* oh = static_cast<uint16_t*>(out_host);
  const FwdOpts o = default_opts();
  if (hp.chunks == 1) {
    const size_t bytes = static_cast<size_t>(T) * d * 2;
    MOE_CUDA(cudaMemcpyAsync(x_in, xh, bytes, cudaMemcpyHostToDevice, st));
    s = run_forward(x_in, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev, Wd_codes_dev,
                    Wd_scales_dev, E, k, T, d, I, out_buf, workspace_dev, hp.sub, st, num_sms, o);
    if (s != MOE_OK) return s;
    MOE_CUDA(cudaMemcpyAsync(oh, out_buf, bytes, cudaMemcpyDeviceToHost, st));
  } else {
    // copy streams and events, created once per device. Calls from several
    // host threads take turns at enqueueing (the events are shared: a wait
    // must see the record of its own call); their copies then share the two
    // copy streams in that order.
    struct CopyRes {
      cudaStream_t h2d, d2h;
      cudaEvent_t start, in[kHostioChunks], fwd[kHostioChunks], done;
    };
    static CopyRes res[kMaxDevices];
    static bool have[kMaxDevices] = {false};
    static std::mutex lock[kMaxDevices];
    int dev = 0;
    MOE_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> guard(lock[dev]);
    CopyRes& r = res[dev];
    if (!have[dev]) {
      MOE_CUDA(cudaStreamCreateWithFlags(&r.h2d, cudaStreamNonBlocking));
      MOE_CUDA(cudaStreamCreateWithFlags(&r.d2h, cudaStreamNonBlocking));
      MOE_CUDA(cudaEventCreateWithFlags(&r.start, cudaEventDisableTiming));
      MOE_CUDA(cudaEventCreateWithFlags(&r.done, cudaEventDisableTiming));
      for (int c = 0; c < kHostioChunks; ++c) {
        MOE_CUDA(cudaEventCreateWithFlags(&r.in[c], cudaEventDisableTiming));
        MOE_CUDA(cudaEventCreateWithFlags(&r.fwd[c], cudaEventDisableTiming));
      }
      have[dev] = true;
    }
    // Every error exit below first waits for the copies already enqueued on
    // the copy streams, so that none lands in the caller's host buffers after
    // the call has returned.
    auto drained = [&](moe_status err) {
      cudaGetLastError();
      cudaStreamSynchronize(r.h2d);
      cudaStreamSynchronize(r.d2h);
      cudaGetLastError();
      return err;
    };
#define MOE_CUDA_CHUNKED(call) \
  do {                                          \
    if ((call) != cudaSuccess) return drained(MOE_ERR_CUDA); \
  } while (0)
    // nothing of this call touches the workspace before the caller's earlier work on st
    MOE_CUDA_CHUNKED(cudaEventRecord(r.start, st));
    MOE_CUDA_CHUNKED(cudaStreamWaitEvent(r.h2d, r.start, 0));
    for (int c = 0; c < hp.chunks; ++c) {
      const int t0 = c * hp.Tc;
      const int tn = T - t0 < hp.Tc ? T - t0 : hp.Tc;
      if (tn <= 0) break;
      const size_t off = static_cast<size_t>(t0) * d;
      const size_t bytes = static_cast<size_t>(tn) * d * 2;
      MOE_CUDA_CHUNKED(cudaMemcpyAsync(x_in + off, xh + off, bytes, cudaMemcpyHostToDevice, r.h2d));
      MOE_CUDA_CHUNKED(cudaEventRecord(r.in[c], r.h2d));
      MOE_CUDA_CHUNKED(cudaStreamWaitEvent(st, r.in[c], 0));
      // chunks c and c+2 share a workspace (both run in order on st), but
      // each chunk records its device status in a word of its own, so that a
      // later chunk's router, which clears its word, cannot erase an earlier
      // chunk's timeout before the host reads it
      void* ws = static_cast<uint8_t*>(workspace_dev) + (c & 1) * hp.sub_stride;
      FwdOpts oc = o;
      oc.status = chunk_status(workspace_dev, hp, c);
      s = run_forward(x_in + off, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev, Wd_codes_dev,
                      Wd_scales_dev, E, k, tn, d, I, out_buf + off, ws, hp.sub, st, num_sms, oc);
      if (s != MOE_OK) return drained(s);
      MOE_CUDA_CHUNKED(cudaEventRecord(r.fwd[c], st));
      MOE_CUDA_CHUNKED(cudaStreamWaitEvent(r.d2h, r.fwd[c], 0));
      MOE_CUDA_CHUNKED(
          cudaMemcpyAsync(oh + off, out_buf + off, bytes, cudaMemcpyDeviceToHost, r.d2h));
    }
    MOE_CUDA_CHUNKED(cudaEventRecord(r.done, r.d2h));
    MOE_CUDA_CHUNKED(cudaStreamWaitEvent(st, r.done, 0));
#undef MOE_CUDA_CHUNKED
  }
  MOE_CUDA(cudaStreamSynchronize(st));
  // the status word of every chunk (one for an unchunked call); a timeout in
  // any chunk is the call's result
  int words[kHostioChunks] = {0, 0, 0, 0};
  MOE_CUDA(cudaMemcpy(words, chunk_status(workspace_dev, hp, 0), sizeof(int) * hp.chunks,
                      cudaMemcpyDeviceToHost));
  for (int c = 0; c < hp.chunks; ++c)
    if (words[c]) return static_cast<moe_status>(words[c]);
  return MOE_OK;
}

moe_status moe_forward_timed(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                             const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                             const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev, int E,
                             int k, int T, int d, int I, void* out_dev, void* workspace_dev,
                             size_t workspace_bytes, void* stream, float* stage_ms_host) {
  return moe_forward_timed_events(x_dev, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev,
                                  Wd_codes_dev, Wd_scales_dev, E, k, T, d, I, out_dev,
                                  workspace_dev, workspace_bytes, stream,
                                  (1u << (kStages + 1)) - 1u, stage_ms_host);
}

moe_status moe_forward_timed_events(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                                    const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                                    const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev,
                                    int E, int k, int T, int d, int I, void* out_dev,
                                    void* workspace_dev, size_t workspace_bytes, void* stream,
                                    unsigned int event_mask, float* stage_ms_host) {
  return moe_forward_timed_ex(x_dev, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev, Wd_codes_dev,
                              Wd_scales_dev, E, k, T, d, I, out_dev, workspace_dev,
                              workspace_bytes, nullptr, stream, event_mask, stage_ms_host);
}

moe_status moe_forward_timed_ex(const void* x_dev, const float* W_r_dev, const float* b_r_dev,
                                const uint8_t* Wgu_codes_dev, const uint8_t* Wgu_scales_dev,
                                const uint8_t* Wd_codes_dev, const uint8_t* Wd_scales_dev, int E,
                                int k, int T, int d, int I, void* out_dev, void* workspace_dev,
                                size_t workspace_bytes, const moe_forward_opts* opts, void* stream,
                                unsigned int event_mask, float* stage_ms_host) {
  if (!stage_ms_host) return MOE_ERR_INVALID_ARG;
  if (event_mask >> (kStages + 1)) return MOE_ERR_INVALID_ARG;
  moe_status s = check_forward_args(x_dev, W_r_dev, b_r_dev, Wgu_codes_dev, Wgu_scales_dev,
                                    Wd_codes_dev, Wd_scales_dev, E, k, T, d, I, out_dev,
                                    workspace_dev);
  if (s != MOE_OK) return s;
  FwdOpts o;
  if ((s = parse_opts(opts, d, I, Wgu_codes_dev, Wd_codes_dev, &o)) != MOE_OK) return s;
  Layout L;
  make_layout(E, k, T, d, I, false, &L);
  if (workspace_bytes < L.pub.total) return MOE_ERR_WORKSPACE;
  for (int i = 0; i <= kStages; ++i) stage_ms_host[i] = 0.f;
  if (T == 0) return MOE_OK;
  int num_sms = 0;
  if ((s = device_info(&num_sms)) != MOE_OK) return s;
  // the first and the last boundary are always recorded (the whole span)
  event_mask |= 1u | (1u << kStages);
  StageEvents tev;
  tev.st = static_cast<cudaStream_t>(stream);
  for (int i = 0; i <= kStages; ++i) tev.ev[i] = nullptr;
  for (int i = 0; i <= kStages; ++i) {
    if (!((event_mask >> i) & 1u)) continue;
    if (cudaEventCreate(&tev.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j)
        if (tev.ev[j]) cudaEventDestroy(tev.ev[j]);
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
  }
  s = run_forward(static_cast<const uint16_t*>(x_dev), W_r_dev, b_r_dev, Wgu_codes_dev,
                  Wgu_scales_dev, Wd_codes_dev, Wd_scales_dev, E, k, T, d, I,
                  static_cast<uint16_t*>(out_dev), workspace_dev, L, tev.st, num_sms, o, &tev);
  if (s == MOE_OK && cudaEventSynchronize(tev.ev[kStages]) == cudaSuccess) {
    // a recorded boundary's entry spans to the next recorded boundary
    for (int i = 0; i < kStages; ++i) {
      if (!tev.ev[i]) continue;
      int j = i + 1;
      while (!tev.ev[j]) ++j;
      cudaEventElapsedTime(&stage_ms_host[i], tev.ev[i], tev.ev[j]);
    }
    cudaEventElapsedTime(&stage_ms_host[kStages], tev.ev[0], tev.ev[kStages]);
  } else if (s == MOE_OK) {
    s = MOE_ERR_CUDA;
  }
  for (int i = 0; i <= kStages; ++i)
    if (tev.ev[i]) cudaEventDestroy(tev.ev[i]);
  cudaGetLastError();
  return s;
}

size_t moe_route_workspace_size(int E, int k, int T, int d) {
  if (!shape_ok(E, k, T, d)) return 0;
  Layout L;
  make_route_layout(E, k, T, d, &L);
  return L.pub.total;
}

moe_status moe_route(const void* x_dev, const float* W_r_dev, const float* b_r_dev, int E, int k,
                     int T, int d, int32_t* topk_idx_dev, float* topk_w_dev, int32_t* counts_dev,
                     int32_t* offsets_dev, int32_t* perm_dev, void* workspace_dev,
                     size_t workspace_bytes, void* stream) {
  if (!x_dev || !W_r_dev || !b_r_dev || !topk_idx_dev || !topk_w_dev || !workspace_dev)
    return MOE_ERR_INVALID_ARG;
  const int nperm = (counts_dev != nullptr) + (offsets_dev != nullptr) + (perm_dev != nullptr);
  if (nperm != 0 && nperm != 3) return MOE_ERR_INVALID_ARG;
  if (E < 1 || k < 1 || T < 0 || d < 1) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(E, k, T, d)) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x_dev) || !aligned16(W_r_dev) || !aligned16(b_r_dev) ||
      !aligned16(workspace_dev))
    return MOE_ERR_INVALID_ARG;
  Layout L;
  make_route_layout(E, k, T, d, &L);
  if (workspace_bytes < L.pub.total) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  int num_sms = 0;
  moe_status s = device_info(&num_sms);
  if (s != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  StageEvents none;
  memset(&none, 0, sizeof(none));
  PdlPass pdl_pass;
  return launch_routing(static_cast<const uint16_t*>(x_dev), W_r_dev, b_r_dev, E, k, T, d,
                        at<float>(workspace_dev, L.pub.logits),
                        at<void>(workspace_dev, L.router_terms), topk_idx_dev, topk_w_dev,
                        counts_dev, offsets_dev, at<int32_t>(workspace_dev, L.mprefix),
                        at<int32_t>(workspace_dev, L.chunk_hist),
                        at<int32_t>(workspace_dev, L.chunk_base), nperm == 3 ? perm_dev : nullptr,
                        at<int>(workspace_dev, L.pub.status), st, none);
}

moe_status moe_mxfp4_to_bf16(const uint8_t* codes_dev, const uint8_t* scales_dev, int rows, int K,
                             void* out_dev, void* stream) {
  if (!codes_dev || !scales_dev || !out_dev || rows < 0 || K < 32 || K % 32)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(codes_dev) || !aligned16(out_dev)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  int num_sms = 0;
  moe_status s = device_info(&num_sms);
  if (s != MOE_OK) return s;
  MOE_CUDA(moe::launch_mxfp4_to_bf16(codes_dev, scales_dev, rows, K,
                                     static_cast<uint16_t*>(out_dev),
                                     static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_mx_split_e4m3(const void* x_dev, int rows, int K, uint8_t* hi_dev,
                             uint8_t* lo_dev, uint8_t* scales_dev, void* stream) {
  if (!x_dev || !hi_dev || !lo_dev || !scales_dev || rows < 0 || K < 32 || K % 32)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_dev) || !aligned16(hi_dev) || !aligned16(lo_dev)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  int num_sms = 0;
  moe_status s = device_info(&num_sms);
  if (s != MOE_OK) return s;
  MOE_CUDA(moe::launch_mx_split_rows(static_cast<const uint16_t*>(x_dev), rows, K, hi_dev, lo_dev,
                                     scales_dev, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_mx_quantize(const void* x_dev, int rows, int K, int act_quant, uint8_t* q_dev,
                           uint8_t* scales_dev, void* stream) {
  if (!x_dev || !q_dev || !scales_dev || rows < 0 || K < 32 || K % 32) return MOE_ERR_INVALID_ARG;
  if (act_quant != MOE_ACT_MXFP8 && act_quant != MOE_ACT_MXFP4) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_dev) || !aligned16(q_dev)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  int num_sms = 0;
  moe_status s = device_info(&num_sms);
  if (s != MOE_OK) return s;
  MOE_CUDA(moe::launch_mx_act_quant_rows(act_quant == MOE_ACT_MXFP8 ? moe::ACT_E4M3 : moe::ACT_E2M1,
                                         static_cast<const uint16_t*>(x_dev), rows, K, q_dev,
                                         scales_dev, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_sync_status(void* workspace_dev, size_t workspace_bytes, void* stream) {
  if (!workspace_dev || workspace_bytes < 16) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  MOE_CUDA(cudaStreamSynchronize(st));
  MOE_CUDA(cudaMemcpy(&v, workspace_dev, sizeof(int), cudaMemcpyDeviceToHost));
  MOE_CUDA(cudaMemsetAsync(workspace_dev, 0, sizeof(int), st));
  MOE_CUDA(cudaStreamSynchronize(st));
  return v ? static_cast<moe_status>(v) : MOE_OK;
}

// Runs one bounded wait that nothing completes; on return the status word at
// the start of `workspace_dev` holds MOE_ERR_TIMEOUT. Exercises the
// failure-detection path of the kernels without hanging the device.
moe_status moe_selftest_wait_timeout(void* workspace_dev, void* stream) {
  if (!workspace_dev || !aligned16(workspace_dev)) return MOE_ERR_INVALID_ARG;
  int num_sms = 0;
  moe_status s = device_info(&num_sms);
  if (s != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_CUDA(cudaMemsetAsync(workspace_dev, 0, sizeof(int), st));
  MOE_CUDA(moe::launch_wait_timeout_selftest(static_cast<int*>(workspace_dev), st));
  return MOE_OK;
}

}  // extern "C"
