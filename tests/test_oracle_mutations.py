"""Plant plausible mistakes in the oracle (CPU only) and check that the pins
catch each one. A pin set that lets a mutation through would not pin much.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
import tests.test_oracle_pins as P

PIN_TESTS = [
    (P.test_e2m1_matches_generic_minifloat, {}),
    (P.test_e8m0_scale_bias_and_nan, {}),
    (P.test_mxfp4_nibble_order_and_group_axis, {}),
    (P.test_router_bias_and_orientation, {}),
    (P.test_all_ones_expert_closed_form, {}),
    (P.test_gate_up_not_swapped_and_silu_sign, {}),
    (P.test_down_projection_orientation, {}),
    (P.test_weighted_combine_two_experts, {}),
    (P.test_selected_softmax_properties, {}),
    (P.test_routing_tables_match_stable_sort, {}),
    (P.test_k_equals_E_is_dense_mixture, {}),
    (P.test_f64_to_bf16_rounding, {}),
    (P.test_rms_norm_closed_forms, {}),
    (P.test_moe_block_residual_and_norm, {}),
    (P.test_expert_biases_closed_form, {}),
    (P.test_silent_init_reduced_active_count, {"M": 3, "k2": 4}),
    (P.test_minifloat_round_on_its_grid, {"fmt": "e4m3", "ebits": 4, "mbits": 3, "bias": 7,
                                          "ncodes": 127}),
    (P.test_mx_quantize_shared_scale, {"fmt": "e4m3", "emax": 8}),
    (P.test_act_quant_applies_to_expert_inputs_and_hidden_rows, {"fmt": "e4m3"}),
]


def _orig(name):
    return getattr(O, name)


def _mut_drop_bias(x, W_r, b_r):
    return _orig_router(x, W_r, np.zeros_like(np.asarray(b_r, dtype=np.float64)))


def _mut_softmax_all(s, idx):
    full = np.exp(s - s.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    return np.take_along_axis(full, idx.astype(np.int64), 1)


def _mut_swap_gate_up(xe, Wgu, I):
    g = xe @ Wgu[:I].T
    u = xe @ Wgu[I:].T
    return g * O.silu(u)


def _mut_nibble_order(codes, scales):
    codes = np.asarray(codes, dtype=np.uint8)
    sw = ((codes & 0x0F) << 4) | (codes >> 4)
    return _orig_decode(sw.astype(np.uint8), scales)


def _mut_scale_bias(scale):
    return _orig_e8m0(np.asarray(scale).astype(np.int64) - 1)


def _mut_silu_sign(z):
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(z))


def _mut_down_transposed(h, Wd):
    return h @ Wd.reshape(Wd.shape[1], Wd.shape[0]).T if Wd.shape[0] != Wd.shape[1] else h @ Wd


def _mut_topk_high_index_ties(s, k):
    s = np.asarray(s, dtype=np.float64)
    T, E = s.shape
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        order = np.lexsort((-np.arange(E), -s[t]))
        out[t] = order[:k]
    return out


def _mut_unstable_tables(idx, E):
    c, o, perm, inv = _orig_tables(idx, E)
    perm = perm.copy()
    for e in range(E):  # reverse the order inside each expert segment
        perm[o[e]:o[e + 1]] = perm[o[e]:o[e + 1]][::-1]
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=perm.dtype)
    return c, o, perm, inv


def _mut_norm_sum_not_mean(h, g, eps):
    h = np.asarray(h, dtype=np.float64)
    ss = np.sum(h * h, axis=1, keepdims=True)
    return h / np.sqrt(ss + eps) * np.asarray(g, dtype=np.float64)[None, :]


def _mut_no_residual(h_bits, g, eps, *args, **kw):
    return _orig_block(h_bits, g, eps, *args, **kw) - O.bf16_to_f64(np.asarray(h_bits))


def _mut_round_toward_zero(a):
    a = np.asarray(a, dtype=np.float64)
    return (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _mut_bias_after_silu(xe, Wgu, I, bias=None):
    h = _orig_hidden(xe, Wgu, I)
    if bias is None:
        return h
    b = np.asarray(bias, dtype=np.float64)
    return (O.silu(xe @ Wgu[:I].T) + b[None, :I]) * (xe @ Wgu[I:].T + b[None, I:])


def _mut_drop_down_bias(h, Wd, bias=None):
    return h @ Wd.T


def _mut_round_half_up(v, ebits, mbits, bias, max_normal):
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), 1 - bias)
    q = np.exp2(e - mbits)
    r = np.minimum(np.floor(a / q + 0.5) * q, max_normal)
    return np.copysign(np.where(a > 0, r, 0.0), v)


def _mut_scale_from_ceil(x, elem, group=32):
    # shared scale from ceil(log2 max|x|): one binade too coarse for most groups
    x = np.asarray(x, dtype=np.float64)
    g = x.reshape(*x.shape[:-1], x.shape[-1] // group, group)
    amax = np.abs(g).max(axis=-1, keepdims=True)
    ebits, mbits, bias, mx, emax = O.MX_ELEMENTS[elem]
    X = np.exp2(np.ceil(np.log2(np.where(amax > 0, amax, 1.0))) - emax)
    return (O.minifloat_round(g / X, ebits, mbits, bias, mx) * X).reshape(x.shape)


def _mut_act_quant_ignored(*args, act_quant=None, **kw):
    return _orig_forward(*args, **kw)


_orig_forward = O.moe_forward
_orig_router = O.router_logits
_orig_block = O.moe_block
_orig_hidden = O.expert_hidden
_orig_decode = O.mxfp4_decode
_orig_e8m0 = O.e8m0_value
_orig_tables = O.routing_tables

MUTATIONS = {
    "drop router bias": ("router_logits", _mut_drop_bias),
    "softmax over all experts": ("selected_softmax", _mut_softmax_all),
    "swap gate and up": ("expert_hidden", _mut_swap_gate_up),
    "high nibble first": ("mxfp4_decode", _mut_nibble_order),
    "scale bias off by one": ("e8m0_value", _mut_scale_bias),
    "silu sign flipped": ("silu", _mut_silu_sign),
    "down projection transposed": ("expert_out", _mut_down_transposed),
    "ties to the higher index": ("topk_select", _mut_topk_high_index_ties),
    "unstable grouping": ("routing_tables", _mut_unstable_tables),
    "norm by the sum of squares": ("rms_norm", _mut_norm_sum_not_mean),
    "residual add dropped": ("moe_block", _mut_no_residual),
    "bf16 truncation": ("f64_to_bf16_bits", _mut_round_toward_zero),
    "gate bias after the silu": ("expert_hidden", _mut_bias_after_silu),
    "down bias dropped": ("expert_out", _mut_drop_down_bias),
    "minifloat ties rounded up": ("minifloat_round", _mut_round_half_up),
    "MX scale from the ceiling": ("mx_quantize", _mut_scale_from_ceil),
    "activation quantisation ignored": ("moe_forward", _mut_act_quant_ignored),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch, golden_dir):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failures = 0
    for test, kw in PIN_TESTS:
        try:
            test(**kw)
        except Exception:
            failures += 1
    # the topk tie rule is pinned by the brute-force test
    if name == "ties to the higher index":
        try:
            P.test_topk_brute_force(8, 2)
        except Exception:
            failures += 1
    assert failures > 0, f"no pin caught the mutation '{name}'"
