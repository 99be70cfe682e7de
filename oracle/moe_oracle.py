"""CPU oracle for the sparse-MoE layer forward pass (test infrastructure only).

This module is the checker, not the product. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. It shares no code with the CUDA path and
imports nothing from the package under test; it receives plain numpy arrays.

Everything is fp64, in the order the pages state the method, with numpy's
matmul as the only library primitive. Sources (page title, section):

* "llm-surgery-dark-arts-gpt-oss-40b-64a8-init", section 2 "Mathematical
  Foundation: Silent Init", "Proof": FFN(h) = sum over i in top-k(s) of
  p_i(h) E_i(h); s_i = W_r[i].h + b_r[i]; p_i = exp(s_i) / sum over the
  selected set S of exp(s_j).
* field guide "gpt-oss 20B", "03 Sparse Mixture of Experts": the router scores
  every expert, keeps the top k, normalises only those scores and forms the
  weighted sum of SwiGLU experts of intermediate width 2,880.
* "shrink/gpt_oss-mic", "Preserved properties": hidden_act is silu.
* "gpt-oss-20b and gpt-oss-120b", "Four-bit expert weights": MXFP4, 4.25 bits
  per parameter counting the shared scales, to be decoded exactly.
* field guide "gpt-oss 20B", "04 One decoder block": RMSNorm before the MoE,
  the sublayer added back to the residual stream (``rms_norm``, ``moe_block``).

Readings where the pages are silent (each also listed in the design notes):

* ties in top-k go to the lower expert index;
* SwiGLU is silu(gate) * up with no clamp and no extra constants; per-expert
  gate/up and down biases are optional (the pages' parameter totals count
  them; their formulas omit them);
* gate and up rows are stacked [gate; up] in one packed tensor;
* MX groups run along the contraction dimension, 32 elements per E8M0 scale
  (bias 127, 0xFF is NaN); byte b holds element 2b in its low nibble;
* E2M1 is 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit, with a
  subnormal at exponent 0 (OCP Microscaling definition);
* RMSNorm is g * h / sqrt(mean(h^2) + eps) with a caller-chosen eps, and its
  output enters the layer rounded to bf16; the residual add is unrounded.

The activation-quantised modes (``mx_quantize``, ``act_quant`` of
``moe_forward``) are not the pages' method: they simulate what rounding the
expert inputs to MXFP8 (E4M3) or MXFP4 (E2M1) blocks would cost, following the
conversion of the OCP Microscaling Formats specification (v1.0, section 6.3).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force, the silent-init identity, and the pages' printed
routing-space and parameter-count tables).
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Tuple

import numpy as np

# --------------------------------------------------------------------------
# Input format: bf16 bit patterns -> float64 (exact)
# --------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to float64; every bf16 value is exact in fp64."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# MXFP4 decode ("Four-bit expert weights"; OCP MX E2M1 + E8M0)
# --------------------------------------------------------------------------

# Magnitudes of the eight non-negative E2M1 codes: exponent field e (2 bits,
# bias 1) and mantissa bit m give 2^(e-1) * (1 + m/2) for e > 0 and m * 0.5
# for the subnormal e = 0.
E2M1_MAGNITUDE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_value(code: np.ndarray) -> np.ndarray:
    """Value of 4-bit E2M1 codes (0..15); bit 3 is the sign, code 8 is -0."""
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_MAGNITUDE[code & 7]
    return np.where(code & 8, -mag, mag)


def e8m0_value(scale: np.ndarray) -> np.ndarray:
    """Value of E8M0 scale bytes: 2^(S-127), with S = 255 meaning NaN."""
    s = np.asarray(scale, dtype=np.int64)
    v = np.ldexp(1.0, s - 127)
    return np.where(s == 255, np.nan, v)


def _byte_table() -> np.ndarray:
    """[256, 2] values of the two E2M1 codes in each byte (low nibble first)."""
    b = np.arange(256, dtype=np.uint8)
    return np.stack([e2m1_value(b & 0x0F), e2m1_value(b >> 4)], axis=1)


def mxfp4_decode(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Decode packed MXFP4 rows to float64.

    codes  [..., K/2] uint8: byte b holds element 2b (low nibble) and 2b+1
    scales [..., K/32] uint8: one E8M0 scale per 32 consecutive elements.
    Returns [..., K] float64: e2m1(code) * 2^(S-127), exact.
    """
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    K = codes.shape[-1] * 2
    if scales.shape[-1] * 32 != K:
        raise ValueError("scales must hold one byte per 32 elements")
    vals = _byte_table()[codes].reshape(*codes.shape[:-1], K // 32, 32)
    out = vals * e8m0_value(scales)[..., None]
    return out.reshape(*codes.shape[:-1], K)


def mxfp4_bits_per_param(group: int = 32, element_bits: int = 4,
                         scale_bits: int = 8) -> float:
    """Storage cost of one MX element including its share of the block scale."""
    return (group * element_bits + scale_bits) / group


# --------------------------------------------------------------------------
# Router ("Silent Init" proof: s_i = W_r[i].h + b_r[i])
# --------------------------------------------------------------------------


def router_logits(x: np.ndarray, W_r: np.ndarray, b_r: np.ndarray) -> np.ndarray:
    """s[t, e] = sum_i x[t, i] * W_r[e, i] + b_r[e], in fp64.

    x is [T, d] float64 (already decoded from bf16); W_r is [E, d]; b_r is [E].
    The sum runs in increasing i for every (t, e), so identical router rows
    give identical logits.
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W_r, dtype=np.float64)
    b = np.asarray(b_r, dtype=np.float64)
    T, d = x.shape
    E = W.shape[0]
    if W.shape != (E, d) or b.shape != (E,):
        raise ValueError("W_r must be [E, d] and b_r [E]")
    s = np.zeros((T, E), dtype=np.float64)
    # one column per expert, accumulated in increasing contraction index
    for e in range(E):
        acc = np.zeros(T, dtype=np.float64)
        for i0 in range(0, d, 256):
            acc = acc + x[:, i0:i0 + 256] @ W[e, i0:i0 + 256]
        s[:, e] = acc + b[e]
    return s


def topk_select(s: np.ndarray, k: int) -> np.ndarray:
    """Top-k experts per token ("Proof": i in top-k(s)).

    Experts are ordered by logit descending, then expert index ascending (the
    pages give no tie rule; the lower index wins). Returns idx [T, k] int32 in
    that order.
    """
    s = np.asarray(s, dtype=np.float64)
    T, E = s.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    idx = np.empty((T, k), dtype=np.int32)
    experts = np.arange(E)
    for t in range(T):
        order = np.lexsort((experts, -s[t]))  # primary key last: -s, then e
        idx[t] = order[:k]
    return idx


def selected_softmax(s: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """p_j = exp(s_j) / sum over the selected set of exp(s_l) ("Proof").

    Evaluated as exp(s_j - m) / sum exp(s_l - m) with m the largest selected
    logit, which is the same quantity. Returns p [T, k] float64.
    """
    sel = np.take_along_axis(np.asarray(s, dtype=np.float64), idx.astype(np.int64), axis=1)
    m = sel.max(axis=1, keepdims=True)
    w = np.exp(sel - m)
    return w / w.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------
# Permutation into expert-contiguous order (implied by the fused packed
# expert tensors: each expert's tokens form one dense block)
# --------------------------------------------------------------------------


def routing_tables(idx: np.ndarray, E: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """Stable grouping of (token, slot) pairs by expert.

    Pair q = t*k + j. counts[e] = number of pairs routed to e; offsets is the
    exclusive prefix sum (E+1 entries); perm lists pair ids grouped by expert,
    ascending pair id within an expert; inv[q] = position of pair q in perm.
    """
    idx = np.asarray(idx, dtype=np.int64)
    flat = idx.reshape(-1)
    P = flat.size
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    fill = offsets[:-1].copy()
    perm = np.empty(P, dtype=np.int64)
    inv = np.empty(P, dtype=np.int64)
    for q in range(P):  # ascending pair id => stable
        e = flat[q]
        perm[fill[e]] = q
        inv[q] = fill[e]
        fill[e] += 1
    return (counts.astype(np.int32), offsets.astype(np.int32),
            perm.astype(np.int32), inv.astype(np.int32))


# --------------------------------------------------------------------------
# SwiGLU expert (field guide "03 Sparse Mixture of Experts"; hidden_act silu)
# --------------------------------------------------------------------------


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_hidden(xe: np.ndarray, Wgu: np.ndarray, I: int,
                  bias: Optional[np.ndarray] = None) -> np.ndarray:
    """H = silu(xe Wgate^T + b_gate) * (xe Wup^T + b_up); Wgu is the decoded
    [2I, d] matrix, bias (optional) the [2I] gate-then-up bias row."""
    g = xe @ Wgu[:I].T
    u = xe @ Wgu[I:].T
    if bias is not None:
        b = np.asarray(bias, dtype=np.float64)
        g = g + b[None, :I]
        u = u + b[None, I:]
    return silu(g) * u


def expert_out(h: np.ndarray, Wd: np.ndarray, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """y = H Wdown^T + b_down; Wd is the decoded [d, I] matrix, bias (optional) [d]."""
    y = h @ Wd.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------


class Routing:
    """Router outputs for a batch (fp64 logits, chosen experts, weights)."""

    def __init__(self, s: np.ndarray, idx: np.ndarray, p: np.ndarray):
        self.s, self.idx, self.p = s, idx, p

    def near_tie(self, tol: float = 1e-5) -> np.ndarray:
        """Tokens whose k-th and (k+1)-th largest logits lie within ``tol``."""
        T, E = self.s.shape
        k = self.idx.shape[1]
        if k == E:
            return np.zeros(T, dtype=bool)
        srt = -np.sort(-self.s, axis=1)
        return (srt[:, k - 1] - srt[:, k]) < tol


def route(x_bits: np.ndarray, W_r: np.ndarray, b_r: np.ndarray, k: int) -> Routing:
    s = router_logits(bf16_to_f64(x_bits), W_r, b_r)
    idx = topk_select(s, k)
    p = selected_softmax(s, idx)
    return Routing(s, idx, p)


def moe_forward(x_bits, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales,
                k: int, tokens: Optional[Iterable[int]] = None,
                return_hidden: bool = False, Bgu: Optional[np.ndarray] = None,
                Bd: Optional[np.ndarray] = None, act_quant: Optional[str] = None):
    """FFN(h) = sum_{i in top-k(s)} p_i(h) E_i(h) for each token, in fp64.

    ``Bgu`` [E, 2I] and ``Bd`` [E, d] (optional) are per-expert biases of the
    gate/up and down projections (the parameter totals of "gpt-oss-20b and
    gpt-oss-120b" and the fixture page count them).

    ``act_quant`` ("e4m3" or "e2m1", default None) simulates an activation-
    quantised mode: each expert's input rows and its H rows pass through
    ``mx_quantize`` (groups of 32 along the contraction) before the matmuls.

    ``tokens`` restricts the computation to a subset of rows (each token's
    output depends on that token alone). Returns out [T', d] float64, and with
    ``return_hidden`` also the Routing and a dict (expert -> (token ids,
    hidden rows H)) for kernel-level checks.
    """
    x_all = np.asarray(x_bits)
    tok = np.arange(x_all.shape[0]) if tokens is None else np.asarray(list(tokens), dtype=np.int64)
    xs = x_all[tok]
    r = route(xs, W_r, b_r, k)
    xf = bf16_to_f64(xs)
    T, d = xf.shape
    E, twoI, _ = Wgu_codes.shape
    I = twoI // 2
    out = np.zeros((T, d), dtype=np.float64)
    hidden = {}
    contrib = np.zeros((T, k, d), dtype=np.float64)
    for e in range(E):
        rows, slots = np.nonzero(r.idx == e)
        if rows.size == 0:
            continue
        Wgu = mxfp4_decode(Wgu_codes[e], Wgu_scales[e])
        Wd = mxfp4_decode(Wd_codes[e], Wd_scales[e])
        xe = xf[rows] if act_quant is None else mx_quantize(xf[rows], act_quant)
        h = expert_hidden(xe, Wgu, I, None if Bgu is None else Bgu[e])
        he = h if act_quant is None else mx_quantize(h, act_quant)
        y = expert_out(he, Wd, None if Bd is None else Bd[e])
        contrib[rows, slots] = r.p[rows, slots][:, None] * y
        if return_hidden:
            hidden[e] = (tok[rows], h)
    for j in range(k):  # weighted sum over the selected set, slot order
        out += contrib[:, j]
    if return_hidden:
        return out, r, hidden
    return out


# --------------------------------------------------------------------------
# Around the layer: the pre-MoE RMSNorm and the residual add
# --------------------------------------------------------------------------


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest, ties to even), returned as bf16 bit
    patterns. A bf16 value has 8 significant bits; below 2^-126 the quantum
    stays 2^-133 (bf16 subnormals). Finite inputs within the bf16 range."""
    a = np.asarray(a, dtype=np.float64)
    _, e = np.frexp(a)                                  # a = m 2^e, 0.5 <= |m| < 1
    q = np.exp2(np.maximum(e - 8, -133).astype(np.float64))
    r = np.rint(a / q) * q                              # rint rounds halves to even
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def rms_norm(h: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm(h)_i = g_i h_i / sqrt(mean_j h_j^2 + eps), row by row, fp64.

    Field guide "gpt-oss 20B", "04 One decoder block": RMSNorm is applied
    before the MoE. The pages give no formula or epsilon; the standard form
    with a per-channel gain g and a caller-chosen eps is the reading taken.
    """
    h = np.asarray(h, dtype=np.float64)
    ms = np.mean(h * h, axis=1, keepdims=True)
    return h / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)[None, :]


def moe_block(h_bits, g, eps, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, k: int,
              x_bits: Optional[np.ndarray] = None, tokens: Optional[Iterable[int]] = None,
              Bgu: Optional[np.ndarray] = None, Bd: Optional[np.ndarray] = None):
    """h + FFN(RMSNorm(h)) per token, in fp64: the MoE sublayer with its
    pre-norm and residual add (field guide "gpt-oss 20B", "04 One decoder
    block": each sublayer is added back to the residual stream).

    The normalised rows enter the layer in its activation format, bf16:
    x = bf16(RMSNorm(h)), unless ``x_bits`` supplies them. The layer output is
    added to h before any rounding. Returns [T', d] float64.
    """
    h_all = np.asarray(h_bits)
    tok = np.arange(h_all.shape[0]) if tokens is None else np.asarray(list(tokens), dtype=np.int64)
    hf = bf16_to_f64(h_all[tok])
    if x_bits is None:
        xb = f64_to_bf16_bits(rms_norm(hf, g, eps))
    else:
        xb = np.asarray(x_bits)[tok]
    return hf + moe_forward(xb, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, k=k,
                            Bgu=Bgu, Bd=Bd)


# --------------------------------------------------------------------------
# Activation quantisation (a simulated mode, not the pages' method)
# --------------------------------------------------------------------------

# element formats: (exponent bits, mantissa bits, exponent bias, largest normal,
# emax = exponent of the largest normal)
MX_ELEMENTS = {
    "e4m3": (4, 3, 7, 448.0, 8),   # OCP FP8 E4M3 (no infinities; S.1111.111 is NaN)
    "e2m1": (2, 1, 1, 6.0, 2),     # OCP FP4 E2M1
}


def minifloat_round(v: np.ndarray, ebits: int, mbits: int, bias: int,
                    max_normal: float) -> np.ndarray:
    """Round v to the nearest value of a sign/exponent/mantissa format with
    subnormals (ties to the even mantissa), clamping magnitudes above the
    largest normal to it. fp64 in and out."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    emin = 1 - bias
    # floor(log2 a), exactly: a = m 2^x with m in [0.5, 1)
    e = np.frexp(np.where(a > 0, a, 1.0))[1] - 1
    e = np.maximum(e, emin)
    quantum = np.exp2(e - mbits)
    r = np.round(a / quantum) * quantum          # numpy rounds halves to even
    r = np.minimum(r, max_normal)
    return np.copysign(np.where(a > 0, r, 0.0), v)


def mx_quantize(x: np.ndarray, elem: str, group: int = 32) -> np.ndarray:
    """One MX block conversion along the last axis, returned dequantised.

    Per group of ``group`` values: shared scale X = 2^(floor(log2 max|x|) - emax)
    (a power of two, as an E8M0 byte holds), elements = minifloat_round(x / X);
    the result is X * element. An all-zero group stays zero.
    """
    ebits, mbits, bias, max_normal, emax = MX_ELEMENTS[elem]
    x = np.asarray(x, dtype=np.float64)
    K = x.shape[-1]
    if K % group:
        raise ValueError("the last axis must hold whole groups")
    g = x.reshape(*x.shape[:-1], K // group, group)
    amax = np.abs(g).max(axis=-1, keepdims=True)
    X = np.exp2((np.frexp(np.where(amax > 0, amax, 1.0))[1] - 1) - emax)
    q = minifloat_round(g / X, ebits, mbits, bias, max_normal) * X
    return np.where(amax > 0, q, 0.0).reshape(x.shape)


# --------------------------------------------------------------------------
# Accounting facts the pages print
# --------------------------------------------------------------------------


def routing_subsets(E: int, k: int) -> int:
    """Distinct expert subsets per token per layer, C(E, k) (section 3)."""
    return math.comb(E, k)


def routing_space_log10(E: int, k: int, L: int) -> float:
    """log10 of C(E, k)^L, the network-wide routing space ("Over L Layers")."""
    return L * math.log10(math.comb(E, k))


def expert_params(d: int, I: int, bias: bool = False) -> int:
    """Parameters of one SwiGLU expert: gate and up (d -> I each), down (I -> d).

    3*d*I weights; with biases, 2I (gate, up) + d (down) more.
    """
    return 3 * d * I + ((2 * I + d) if bias else 0)


def gpt_oss_layer_params(d: int, I: int, E: int, n_q: int, n_kv: int,
                         head_dim: int, expert_bias: bool = True) -> int:
    """Parameters of one gpt-oss decoder layer (attention + MoE + norms).

    Attention: q/k/v/o projections with biases and one learned sink logit per
    query head; router [E, d] plus bias; E experts; two RMSNorm weights.
    """
    q = d * n_q * head_dim + n_q * head_dim
    kv = 2 * (d * n_kv * head_dim + n_kv * head_dim)
    o = n_q * head_dim * d + d
    sinks = n_q
    router = E * d + E
    experts = E * expert_params(d, I, bias=expert_bias)
    norms = 2 * d
    return q + kv + o + sinks + router + experts + norms


def gpt_oss_model_params(d: int, I: int, E: int, k: int, n_q: int, n_kv: int,
                         head_dim: int, layers: int, vocab: int) -> Tuple[int, int, int]:
    """(total, active per token, decoder-layer total) for a gpt-oss model.

    Untied embedding and lm_head of vocab x d each plus a final RMSNorm.
    Active leaves out the E-k unselected experts of every layer and the
    embedding table (a token reads one row of it; it is not multiplied).
    """
    layer = gpt_oss_layer_params(d, I, E, n_q, n_kv, head_dim)
    inactive_experts = (E - k) * expert_params(d, I, bias=True)
    total = layers * layer + 2 * vocab * d + d
    active = total - layers * inactive_experts - vocab * d
    return total, active, layers * layer
