"""Pins for the CPU oracle: values the pages print, closed forms, brute force,
and invariants. None of these re-types the oracle's own formula; each is
chosen so that a plausible slip (a dropped bias, a transposed operand, a
swapped gate/up, a wrong nibble order or scale bias, a softmax over the wrong
set) fails at least one test.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O
from sparse_moe_layer_05_b200 import workloads as W


# ---------------------------------------------------------------- MXFP4 ----

def _generic_minifloat(code: int, exp_bits: int, man_bits: int, bias: int) -> float:
    """Textbook decoding of an IEEE-style minifloat with subnormals (no inf/NaN)."""
    sign = (code >> (exp_bits + man_bits)) & 1
    e = (code >> man_bits) & ((1 << exp_bits) - 1)
    m = code & ((1 << man_bits) - 1)
    if e == 0:
        v = (m / (1 << man_bits)) * 2.0 ** (1 - bias)
    else:
        v = (1 + m / (1 << man_bits)) * 2.0 ** (e - bias)
    return -v if sign else v


def test_e2m1_matches_generic_minifloat():
    # E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit
    got = O.e2m1_value(np.arange(16, dtype=np.uint8))
    want = np.array([_generic_minifloat(c, 2, 1, 1) for c in range(16)])
    assert np.array_equal(got, want)
    assert np.signbit(got[8]) and got[8] == 0.0  # code 8 is -0
    assert sorted(set(np.abs(got).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e8m0_scale_bias_and_nan():
    s = O.e8m0_value(np.array([0, 1, 126, 127, 128, 254, 255], dtype=np.uint8))
    assert s[3] == 1.0 and s[4] == 2.0 and s[2] == 0.5
    assert s[0] == math.ldexp(1.0, -127) and s[1] == math.ldexp(1.0, -126)
    assert s[5] == math.ldexp(1.0, 127)
    assert np.isnan(s[6])


def test_mxfp4_nibble_order_and_group_axis():
    # one row of K = 64: two groups with different scales
    codes = np.zeros((1, 32), dtype=np.uint8)
    codes[0, 0] = 0x21      # element 0 -> code 1 (0.5), element 1 -> code 2 (1.0)
    codes[0, 15] = 0xF7     # element 30 -> code 7 (6.0), element 31 -> code 15 (-6.0)
    codes[0, 16] = 0x9A     # element 32 -> code 10 (-1.0), element 33 -> code 9 (-0.5)
    scales = np.array([[127, 130]], dtype=np.uint8)   # group 0 x1, group 1 x8
    v = O.mxfp4_decode(codes, scales)[0]
    assert v.shape == (64,)
    assert v[0] == 0.5 and v[1] == 1.0
    assert v[30] == 6.0 and v[31] == -6.0
    assert v[32] == -8.0 and v[33] == -4.0
    assert np.count_nonzero(v) == 6


def _encode_e2m1(val: float) -> int:
    """Test-side encoder: exact E2M1 value -> code (the inverse map)."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    c = mags.index(abs(val))
    return c | (8 if math.copysign(1.0, val) < 0 else 0)


def test_mxfp4_roundtrip_every_code_and_scale():
    rng = np.random.default_rng(5)
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    for S in range(0, 255):
        vals = rng.choice(mags, size=32) * rng.choice([-1.0, 1.0], size=32)
        nib = np.array([_encode_e2m1(v) for v in vals], dtype=np.uint8)
        codes = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)[None]
        dec = O.mxfp4_decode(codes, np.array([[S]], dtype=np.uint8))[0]
        assert np.array_equal(dec, vals * math.ldexp(1.0, S - 127)), S


def test_bits_per_param_matches_page(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "mxfp4_storage.json")))
    assert O.mxfp4_bits_per_param() == g["bits_per_expert_param_printed"]
    lb = g["lower_bound_printed"]
    assert lb["params"] * 16 / 8 == lb["bytes_16bit"]
    assert lb["params"] * 4 / 8 == lb["bytes_4bit"]


# --------------------------------------------------------------- router ----

def test_router_bias_and_orientation():
    rng = np.random.default_rng(1)
    E, d = 5, 64
    Wr = rng.standard_normal((E, d))
    b = rng.standard_normal(E)
    s0 = O.router_logits(np.zeros((1, d)), Wr, b)
    assert np.array_equal(s0[0], b)                  # x = 0 -> logits are the bias
    x = np.zeros((d, d))
    x[np.arange(d), np.arange(d)] = 1.0              # one-hot rows
    s = O.router_logits(x, Wr, b)
    assert np.allclose(s, Wr.T + b[None], rtol=0, atol=1e-15)   # s[i, e] = W_r[e, i] + b_e


def test_router_duplicate_rows_bitwise_equal():
    rng = np.random.default_rng(2)
    Wr = rng.standard_normal((3, 96))
    b = rng.standard_normal(3)
    Wr2 = np.concatenate([Wr, Wr])
    b2 = np.concatenate([b, b])
    s = O.router_logits(rng.standard_normal((7, 96)), Wr2, b2)
    assert np.array_equal(s[:, :3], s[:, 3:])


def test_bf16_decode_exact():
    bits = np.array([0x3F80, 0xBF80, 0x0000, 0x8000, 0x4049, 0x0001, 0x7F7F], dtype=np.uint16)
    v = O.bf16_to_f64(bits)
    assert v[0] == 1.0 and v[1] == -1.0 and v[2] == 0.0 and np.signbit(v[3])
    assert v[4] == 3.140625
    assert v[5] == math.ldexp(1.0, -133)              # smallest bf16 subnormal
    assert v[6] == (2 - 2 ** -7) * 2.0 ** 127         # largest finite bf16


# ---------------------------------------------------------------- top-k ----

def _dominates(s, i, j):
    return s[i] > s[j] or (s[i] == s[j] and i < j)


@pytest.mark.parametrize("E,k", [(4, 2), (5, 1), (6, 3), (7, 4), (8, 2), (8, 8)])
def test_topk_brute_force(E, k):
    rng = np.random.default_rng(E * 10 + k)
    # coarse values so that exact ties occur often
    s = rng.integers(-3, 4, size=(40, E)).astype(np.float64)
    idx = O.topk_select(s, k)
    for t in range(s.shape[0]):
        winners = [S for S in itertools.combinations(range(E), k)
                   if all(_dominates(s[t], i, j) for i in S for j in range(E) if j not in S)]
        assert len(winners) == 1
        assert set(idx[t].tolist()) == set(winners[0])
        # ordered by logit descending, then index ascending
        key = [(-s[t, e], e) for e in idx[t]]
        assert key == sorted(key)


def test_subset_enumeration_matches_page_table(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "routing_space.json")))
    base = None
    for row in g["per_layer"]:
        n = O.routing_subsets(row["E"], row["k"])
        if row["exact"] is not None:
            assert n == row["exact"], row
        if row["config"] == "gpt-oss-20b":
            base = n
    # brute-force enumeration agrees with the closed form for the small ones
    assert sum(1 for _ in itertools.combinations(range(32), 4)) == 35960
    # the 96a12 entry: the per-layer table misprints it; the L-layer table's
    # base value is the exact one
    exact_96_12 = O.routing_subsets(96, 12)
    assert exact_96_12 == 624668654531480
    assert f"{exact_96_12:.2e}" == "6.25e+14"
    # ratios against gpt-oss-20b
    ratio = {r["config"]: O.routing_subsets(r["E"], r["k"]) / base for r in g["per_layer"]}
    assert round(ratio["gpt-oss-120b"]) == 297
    assert round(ratio["64a4 (post-training)"], 1) == 17.7
    assert round(ratio["96a4 (post-training)"]) == 92
    assert round(ratio["64a8"]) == 123086        # printed 123,091x: page error


def test_routing_space_over_layers(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "routing_space.json")))
    for row in g["over_layers"]:
        assert round(O.routing_space_log10(row["E"], row["k"], row["L"])) == row["printed_log10"], row


# -------------------------------------------------------------- softmax ----

def test_selected_softmax_properties():
    rng = np.random.default_rng(3)
    s = rng.standard_normal((50, 9)) * 3
    idx = O.topk_select(s, 4)
    p = O.selected_softmax(s, idx)
    assert np.all(np.abs(p.sum(1) - 1) < 1e-12) and np.all(p > 0)
    assert np.all(np.diff(p, axis=1) <= 0)          # ordered by logit
    # k = 1: the single expert gets weight exactly 1
    assert np.all(O.selected_softmax(s, O.topk_select(s, 1)) == 1.0)
    # k = 2 reduces to the logistic function of the logit gap
    i2 = O.topk_select(s, 2)
    p2 = O.selected_softmax(s, i2)
    gap = s[np.arange(50), i2[:, 0]] - s[np.arange(50), i2[:, 1]]
    assert np.allclose(p2[:, 0], 1 / (1 + np.exp(-gap)), rtol=1e-14, atol=0)
    # normalised over the selected set, not over all experts
    full = np.exp(s - s.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    assert not np.allclose(p, np.take_along_axis(full, idx, 1))


# ---------------------------------------------------------- permutation ----

def test_routing_tables_match_stable_sort():
    rng = np.random.default_rng(4)
    E, k, T = 9, 3, 200
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    counts, offsets, perm, inv = O.routing_tables(idx, E)
    flat = idx.reshape(-1)
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.array_equal(inv[perm], np.arange(T * k))


# --------------------------------------------------------- expert math ----

def _const_layer(E, d, I, gate_code, up_code, down_code, gate_S=127, up_S=127, down_S=None):
    """Layer whose every weight of a kind is one E2M1 code with one scale."""
    gu = np.zeros((E, 2 * I, d // 2), dtype=np.uint8)
    gu[:, :I] = gate_code | (gate_code << 4)
    gu[:, I:] = up_code | (up_code << 4)
    gus = np.zeros((E, 2 * I, d // 32), dtype=np.uint8)
    gus[:, :I] = gate_S
    gus[:, I:] = up_S
    dc = np.full((E, d, I // 2), down_code | (down_code << 4), dtype=np.uint8)
    ds = np.full((E, d, I // 32), 127, dtype=np.uint8)
    if down_S is not None:
        ds[:] = np.asarray(down_S, dtype=np.uint8)[None, :, None]
    return gu, gus, dc, ds


def _bf16(a):
    return W.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def test_all_ones_expert_closed_form():
    d, I = 64, 96
    rng = np.random.default_rng(6)
    x = _bf16(rng.standard_normal((6, d)) * 0.1)
    gu, gus, dc, ds = _const_layer(1, d, I, 2, 2, 2)            # every weight = 1.0
    out = O.moe_forward(x, np.zeros((1, d), np.float32), np.zeros(1, np.float32),
                        gu, gus, dc, ds, k=1)
    sx = O.bf16_to_f64(x).sum(1)
    a = sx / (1 + np.exp(-sx)) * sx
    assert np.allclose(out, (I * a)[:, None] * np.ones(d), rtol=1e-13, atol=0)


def test_gate_up_not_swapped_and_silu_sign():
    d, I = 64, 64
    x = _bf16(np.array([np.full(d, 0.05), np.full(d, -0.05)]))   # sums +3.2 and -3.2
    # gate weights 1.0 (code 2), up weights 0.5 (code 1)
    gu, gus, dc, ds = _const_layer(1, d, I, 2, 1, 2)
    out = O.moe_forward(x, np.zeros((1, d), np.float32), np.zeros(1, np.float32),
                        gu, gus, dc, ds, k=1)
    sx = O.bf16_to_f64(x).sum(1)
    g, u = sx, 0.5 * sx
    want = I * (g / (1 + np.exp(-g))) * u
    assert np.allclose(out[:, 0], want, rtol=1e-13)
    swapped = I * g * (u / (1 + np.exp(-u)))
    assert not np.allclose(out[:, 0], swapped, rtol=1e-3)


def test_down_projection_orientation():
    d, I = 96, 64
    x = _bf16(np.full((1, d), 0.02))
    # down row m scaled by 2^(m % 3): y_m = 2^(m%3) * I * a
    gu, gus, dc, ds = _const_layer(1, d, I, 2, 2, 2, down_S=127 + (np.arange(d) % 3))
    out = O.moe_forward(x, np.zeros((1, d), np.float32), np.zeros(1, np.float32),
                        gu, gus, dc, ds, k=1)
    sx = O.bf16_to_f64(x).sum()
    a = sx / (1 + np.exp(-sx)) * sx
    assert np.allclose(out[0], I * a * 2.0 ** (np.arange(d) % 3), rtol=1e-13)


def test_weighted_combine_two_experts():
    d, I = 64, 64
    x = _bf16(np.full((1, d), 0.03))
    gu0, gus0, dc0, ds0 = _const_layer(1, d, I, 2, 2, 2)        # expert 0: all 1.0
    gu1, gus1, dc1, ds1 = _const_layer(1, d, I, 2, 2, 4)        # expert 1: down = 2.0
    gu = np.concatenate([gu0, gu1, gu0]); gus = np.concatenate([gus0, gus1, gus0])
    dc = np.concatenate([dc0, dc1, dc0]); ds = np.concatenate([ds0, ds1, ds0])
    b = np.array([0.7, 0.2, -5.0], dtype=np.float32)              # bias decides routing
    out = O.moe_forward(x, np.zeros((3, d), np.float32), b, gu, gus, dc, ds, k=2)
    sx = O.bf16_to_f64(x).sum()
    y0 = I * (sx / (1 + np.exp(-sx))) * sx
    p0 = 1 / (1 + np.exp(-(0.7 - np.float64(np.float32(0.2)))))
    p0 = 1 / (1 + np.exp(-(np.float64(np.float32(0.7)) - np.float64(np.float32(0.2)))))
    want = p0 * y0 + (1 - p0) * 2 * y0
    assert np.allclose(out[0], want, rtol=1e-13)


def test_k_equals_E_is_dense_mixture():
    inp = W.make_custom(64, 64, 3, 3, 5, seed=11)
    out = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                        inp.Wd_codes, inp.Wd_scales, k=3)
    xf = O.bf16_to_f64(inp.x)
    s = xf @ inp.W_r.astype(np.float64).T + inp.b_r
    p = np.exp(s - s.max(1, keepdims=True)); p /= p.sum(1, keepdims=True)
    acc = np.zeros_like(out)
    for e in range(3):
        Wgu = O.mxfp4_decode(inp.Wgu_codes[e], inp.Wgu_scales[e])
        Wd = O.mxfp4_decode(inp.Wd_codes[e], inp.Wd_scales[e])
        acc += p[:, e:e + 1] * O.expert_out(O.expert_hidden(xf, Wgu, 64), Wd)
    assert np.allclose(out, acc, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------ silent init ----

@pytest.mark.parametrize("M", [2, 3])
def test_silent_init_identity(M):
    """Expanded x M with k' = M k reproduces the original layer (section 2)."""
    base = W.make_custom(64, 128, 4, 2, 48, seed=7, scale_lo=121, scale_hi=124)
    exp = W.expand_silent(base, M)
    a = O.moe_forward(base.x, base.W_r, base.b_r, base.Wgu_codes, base.Wgu_scales,
                      base.Wd_codes, base.Wd_scales, k=base.k)
    b, r, _ = O.moe_forward(exp.x, exp.W_r, exp.b_r, exp.Wgu_codes, exp.Wgu_scales,
                            exp.Wd_codes, exp.Wd_scales, k=exp.k, return_hidden=True)
    rms = np.sqrt(np.mean(a ** 2))
    assert np.max(np.abs(a - b)) <= 1e-12 * rms
    # top-k' holds exactly the M copies of each original top-k expert
    ra = O.route(base.x, base.W_r, base.b_r, base.k)
    for t in range(base.T):
        assert sorted(set(e % base.E for e in r.idx[t])) == sorted(ra.idx[t])
        assert all(sum(1 for e in r.idx[t] if e % base.E == o) == M for o in ra.idx[t])


@pytest.mark.parametrize("M,k2", [(2, 4), (3, 4), (2, 3), (3, 5)])
def test_silent_init_reduced_active_count(M, k2):
    """An x M silent-init layer run at k' = q M + r (r < M) routes each token to all
    M copies of its q best original experts and to r copies of the next one (the
    copies tie exactly), so with c_o = M or r its output is
    sum_o c_o e^{s_o} E_o(x) / sum_o c_o e^{s_o} over those originals. The page's
    "64a8 to 64a4, 96a12 to 96a4" is k' = 4 with M = 2 (the original layer at k = 2)
    and M = 3 (three copies of the best expert, one of the second)."""
    base = W.make_custom(64, 128, 6, 2, 40, seed=17, scale_lo=121, scale_hi=124)
    exp = W.expand_silent(base, M)
    got = O.moe_forward(exp.x, exp.W_r, exp.b_r, exp.Wgu_codes, exp.Wgu_scales, exp.Wd_codes,
                        exp.Wd_scales, k=k2)
    xf = O.bf16_to_f64(base.x)
    s = xf @ base.W_r.astype(np.float64).T + base.b_r.astype(np.float64)
    outs = np.stack([O.expert_out(O.expert_hidden(xf, O.mxfp4_decode(base.Wgu_codes[e],
                                                                      base.Wgu_scales[e]), 128),
                                  O.mxfp4_decode(base.Wd_codes[e], base.Wd_scales[e]))
                     for e in range(base.E)], axis=1)             # [T, E, d]
    q, r = divmod(k2, M)
    want = np.zeros_like(got)
    for t in range(base.T):
        order = np.argsort(-s[t], kind="stable")
        c = [M] * q + ([r] if r else [])
        chosen = order[:len(c)]
        w = np.array(c) * np.exp(s[t, chosen] - s[t, chosen].max())
        want[t] = (w / w.sum()) @ outs[t, chosen]
    assert np.max(np.abs(got - want)) <= 1e-12 * np.sqrt(np.mean(want ** 2))


def test_fixture_workload_recipe():
    inp = W.make_inputs("fixture")
    assert (inp.d, inp.I, inp.E, inp.k, inp.T) == (64, 128, 4, 2, 256)
    assert inp.Wgu_scales.min() >= 121 and inp.Wgu_scales.max() <= 124
    out = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                        inp.Wd_codes, inp.Wd_scales, k=2)
    assert out.shape == (256, 64) and np.all(np.isfinite(out))


def test_token_subset_equals_full():
    inp = W.make_custom(64, 64, 6, 2, 40, seed=9)
    full = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                         inp.Wd_codes, inp.Wd_scales, k=2)
    sub = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                        inp.Wd_codes, inp.Wd_scales, k=2, tokens=[3, 17, 39])
    # BLAS blocking may differ with the batch size: equal up to fp64 rounding
    assert np.allclose(sub, full[[3, 17, 39]], rtol=1e-12, atol=1e-15)


# ------------------------------------------------------- accounting ----

def _fmt(n, unit, digits):
    return f"{n / unit:.{digits}f}"


def test_parameter_counts_match_pages(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "param_counts.json")))
    f = g["fixture"]
    tot, act, layers = O.gpt_oss_model_params(f["d"], f["I"], f["E"], f["k"], f["n_q"],
                                               f["n_kv"], f["head_dim"], f["layers"], f["vocab"])
    assert _fmt(layers, 1e3, 1) + "K" == f["printed"]["model.layers"]
    assert _fmt(tot, 1e6, 1) + "M" == f["printed"]["total"]
    assert _fmt(f["vocab"] * f["d"], 1e6, 1) + "M" == f["printed"]["lm_head"]
    assert str(f["d"]) == f["printed"]["model.norm"]
    # the printed 224.9K needs expert biases; without them it would read 222.4K
    no_bias = layers - f["layers"] * f["E"] * (2 * f["I"] + f["d"])
    assert _fmt(no_bias, 1e3, 1) == "222.4"
    t = g["20b"]
    tot, act, layers = O.gpt_oss_model_params(t["d"], t["I"], t["E"], t["k"], t["n_q"],
                                               t["n_kv"], t["head_dim"], t["layers"], t["vocab"])
    assert _fmt(tot, 1e9, 2) + "B" == t["printed"]["total"]
    assert _fmt(act, 1e9, 2) + "B" == t["printed"]["active"]
    assert _fmt(layers, 1e9, 1) + "B" == t["printed"]["model.layers"]
    assert f"{100 * layers / tot:.1f}%" == t["printed"]["model.layers_share"]
    assert _fmt(t["vocab"] * t["d"], 1e6, 1) + "M" == t["printed"]["lm_head"]
    assert _fmt(t["d"], 1e3, 1) + "K" == t["printed"]["model.norm"]
    assert O.expert_params(2880, 2880) == g["expert_weights_per_expert_2880"]


def test_near_tie_detector():
    s = np.array([[3.0, 1.0, 1.0 + 5e-6, 0.0], [3.0, 2.0, 1.0, 0.0]])
    r = O.Routing(s, O.topk_select(s, 2), None)
    assert r.near_tie().tolist() == [True, False]


# --------------------------------------------- pre-norm and residual add ----

def test_f64_to_bf16_rounding():
    """Nearest-even rounding to 8 significant bits, checked on hand-made values."""
    one = 1.0
    cases = {
        one: 0x3F80,
        one + 2.0 ** -7: 0x3F81,            # exactly representable
        one + 2.0 ** -8: 0x3F80,            # halfway: ties to the even mantissa
        one + 3 * 2.0 ** -8: 0x3F82,        # halfway: ties up to the even mantissa
        one + 2.0 ** -8 + 2.0 ** -20: 0x3F81,
        -3.0: 0xC040,
        2.0 ** -130: 0x0008,                # bf16 subnormal
    }
    got = O.f64_to_bf16_bits(np.array(list(cases)))
    assert [int(v) for v in got] == list(cases.values())
    x = np.random.default_rng(1).standard_normal(1000)
    b = O.f64_to_bf16_bits(x)
    back = O.bf16_to_f64(b)
    assert np.all(np.abs(back - x) <= 2.0 ** -8 * np.abs(x))   # half a quantum of 8 bits


def test_rms_norm_closed_forms():
    rng = np.random.default_rng(2)
    h = rng.standard_normal((5, 48)) * rng.uniform(0.1, 10, size=(5, 1))
    one = np.ones(48)
    y = O.rms_norm(h, one, 0.0)
    assert np.allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-13)      # unit mean square
    assert np.allclose(O.rms_norm(7.5 * h, one, 0.0), y, rtol=1e-13)  # scale invariant
    c = np.full((1, 48), -2.0)
    g = rng.uniform(0.5, 2.0, size=48)
    assert np.allclose(O.rms_norm(c, g, 0.25), -2.0 / math.sqrt(4.25) * g[None, :], rtol=1e-14)
    assert np.all(O.rms_norm(np.zeros((1, 48)), g, 1e-5) == 0.0)


def test_moe_block_residual_and_norm():
    """Zero expert weights leave exactly h; the sublayer sees the normalised rows
    (a positive rescale of h changes only the residual term)."""
    d, I, E, k, T = 64, 96, 4, 2, 6
    inp = W.make_custom(d, I, E, k, T, seed=9)
    g = np.random.default_rng(3).uniform(0.5, 1.5, size=d)
    zero_gu = np.zeros_like(inp.Wgu_codes)
    zero_d = np.zeros_like(inp.Wd_codes)
    out0 = O.moe_block(inp.x, g, 1e-5, inp.W_r, inp.b_r, zero_gu, inp.Wgu_scales, zero_d,
                       inp.Wd_scales, k=k)
    assert np.array_equal(out0, O.bf16_to_f64(inp.x))
    # h and 4h (exact in bf16) normalise to the same x when eps = 0
    h4 = O.f64_to_bf16_bits(4.0 * O.bf16_to_f64(inp.x))
    a = O.moe_block(inp.x, g, 0.0, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                    inp.Wd_codes, inp.Wd_scales, k=k)
    b = O.moe_block(h4, g, 0.0, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                    inp.Wd_codes, inp.Wd_scales, k=k)
    hx = O.bf16_to_f64(inp.x)
    assert np.allclose(b - 4.0 * hx, a - hx, rtol=1e-12, atol=1e-12)
    # and the sublayer term is the layer applied to bf16(RMSNorm(h))
    xb = O.f64_to_bf16_bits(O.rms_norm(hx, g, 0.0))
    ff = O.moe_forward(xb, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
                       inp.Wd_scales, k=k)
    assert np.array_equal(a - hx, ff) or np.allclose(a - hx, ff, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------- expert biases ----

def test_expert_biases_closed_form():
    """All-zero weights with biases: H = silu(b_gate) b_up and y = b_down + H Wd^T = b_down,
    so the output is sum_j p_j b_down[e_j]; gate/up biases enter before the silu."""
    d, I, E, k, T = 64, 96, 3, 2, 5
    inp = W.make_custom(d, I, E, k, T, seed=21)
    rng = np.random.default_rng(22)
    Bgu = rng.standard_normal((E, 2 * I))
    Bd = rng.standard_normal((E, d))
    zgu, zd = np.zeros_like(inp.Wgu_codes), np.zeros_like(inp.Wd_codes)
    out, r, hidden = O.moe_forward(inp.x, inp.W_r, inp.b_r, zgu, inp.Wgu_scales, zd,
                                   inp.Wd_scales, k=k, return_hidden=True, Bgu=Bgu, Bd=Bd)
    want = np.einsum("tj,tjd->td", r.p, Bd[r.idx])
    assert np.allclose(out, want, rtol=1e-13, atol=1e-13)
    for e, (toks, h) in hidden.items():
        g, u = Bgu[e, :I], Bgu[e, I:]
        assert np.allclose(h, np.broadcast_to(g / (1 + np.exp(-g)) * u, h.shape), rtol=1e-13)
    # with real weights the gate bias shifts the silu argument, not its output
    full = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
                         inp.Wd_scales, k=k, Bgu=Bgu, Bd=np.zeros((E, d)))
    plain = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
                          inp.Wd_scales, k=k)
    assert not np.allclose(full, plain)


# ------------------------------------- simulated activation quantisation ----

@pytest.mark.parametrize("fmt,ebits,mbits,bias,ncodes", [("e4m3", 4, 3, 7, 127),
                                                        ("e2m1", 2, 1, 1, 8)])
def test_minifloat_round_on_its_grid(fmt, ebits, mbits, bias, ncodes):
    """Every finite non-negative code (textbook decoding; E4M3's code 127 is NaN) is a
    fixed point; a midpoint between neighbours goes to the even code (even mantissa);
    a quarter of the way goes to the nearer one; magnitudes above the largest normal
    clamp to it; signs are symmetric."""
    max_normal = O.MX_ELEMENTS[fmt][3]
    codes = np.arange(ncodes)
    grid = np.array([_generic_minifloat(int(c), ebits, mbits, bias) for c in codes])
    assert np.all(np.diff(grid) > 0) and grid[-1] == max_normal

    def r(v):
        return O.minifloat_round(np.asarray(v, dtype=np.float64), ebits, mbits, bias, max_normal)

    assert np.array_equal(r(grid), grid) and np.array_equal(r(-grid), -grid)
    lo, hi = grid[:-1], grid[1:]
    assert np.array_equal(r((lo + hi) / 2), np.where(codes[:-1] % 2 == 0, lo, hi))
    assert np.array_equal(r(lo + (hi - lo) / 4), lo)
    assert np.array_equal(r(hi - (hi - lo) / 4), hi)
    assert np.array_equal(r([max_normal * 1.01, max_normal * 1e6, -max_normal * 3]),
                          [max_normal, max_normal, -max_normal])


@pytest.mark.parametrize("fmt,emax", [("e4m3", 8), ("e2m1", 2)])
def test_mx_quantize_shared_scale(fmt, emax):
    """Shared scale 2^(floor(log2 max|x|) - emax) per group of 32: grid values times
    that scale pass exactly; the group max lands in [2^emax, 2^(emax+1)) before
    rounding (so 1.9 clamps to max_normal * 2^-emax); all-zero groups stay zero;
    groups are independent; scaling by 2^m commutes."""
    ebits, mbits, bias, max_normal, _ = O.MX_ELEMENTS[fmt]
    rng = np.random.default_rng(11)
    grid = np.array([_generic_minifloat(c, ebits, mbits, bias) for c in range(1 << (ebits + mbits))
                     if _generic_minifloat(c, ebits, mbits, bias) <= max_normal])
    x = rng.choice(grid, size=(3, 64)) * rng.choice([-1.0, 1.0], size=(3, 64))
    x[:, 0] = 2.0 ** emax                              # group max = 2^emax: scale 1
    x[:, 32] = 2.0 ** emax
    for m in (-20, 0, 9):
        xs = x * 2.0 ** m
        assert np.array_equal(O.mx_quantize(xs, fmt), xs)
    g = np.zeros((1, 32))
    g[0, 0], g[0, 1] = 1.9, 1.0
    q = O.mx_quantize(g, fmt)
    assert q[0, 0] == max_normal * 2.0 ** -emax and q[0, 1] == 1.0
    assert np.array_equal(O.mx_quantize(np.zeros((2, 32)), fmt), np.zeros((2, 32)))
    y = rng.standard_normal((4, 96))
    qy = O.mx_quantize(y, fmt)
    y2 = y.copy()
    y2[:, 64:] *= 1000.0
    assert np.array_equal(O.mx_quantize(y2, fmt)[:, :64], qy[:, :64])
    assert np.array_equal(O.mx_quantize(y * 2.0 ** 7, fmt), qy * 2.0 ** 7)


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_act_quant_applies_to_expert_inputs_and_hidden_rows(fmt):
    """All-ones expert, constant input rows: the quantised input is a constant c_q,
    H is the constant a = silu(d c_q) d c_q, its quantised value a_q follows from the
    shared-scale rule on one binade, and out = I a_q."""
    d, I = 64, 96
    ebits, mbits, bias, max_normal, emax = O.MX_ELEMENTS[fmt]

    def q_const(v):          # MX quantisation of a group whose 32 values all equal v > 0
        X = 2.0 ** (math.floor(math.log2(v)) - emax)
        step = 2.0 ** (emax - mbits)  # element spacing on the binade [2^emax, 2^(emax+1))
        return X * min(step * round(v / X / step), max_normal)

    x = _bf16(np.array([np.full(d, 0.05), np.full(d, 0.0071)]))
    gu, gus, dc, ds = _const_layer(1, d, I, 2, 2, 2)            # every weight = 1.0
    args = (x, np.zeros((1, d), np.float32), np.zeros(1, np.float32), gu, gus, dc, ds)
    out = O.moe_forward(*args, k=1, act_quant=fmt)
    for t, c in enumerate(O.bf16_to_f64(x)[:, 0]):
        s = d * q_const(c)
        a = s / (1 + math.exp(-s)) * s
        assert np.allclose(out[t], I * q_const(a), rtol=1e-13, atol=0)
    exact = O.moe_forward(*args, k=1)
    assert not np.allclose(out, exact, rtol=1e-4)
