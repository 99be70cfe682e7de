"""GPU-vs-oracle parity of the CUDA path, called through the C ABI.

Integer outputs (top-k indices outside near-ties, the permutation) must be
bit-exact; floating-point outputs must satisfy max|err| <= 2e-2 * RMS of the
oracle output (bf16 I/O, fp32 accumulation). Sizes span several tiles and
ragged tails; the full bench shapes are checked on sampled tokens.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from sparse_moe_layer_05_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_moe_layer_05_b200 import build
    build.build()


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


# ------------------------------------------------------------ MXFP4 decode --

def test_mxfp4_decode_every_code_and_scale():
    from sparse_moe_layer_05_b200 import binding as B
    K = 512                                    # 256 byte values x 2 nibbles
    scales_list = list(range(0, 253)) + [255]
    rows = len(scales_list)
    codes = np.tile(np.arange(256, dtype=np.uint8), (rows, 1))
    scales = np.repeat(np.array(scales_list, dtype=np.uint8)[:, None], K // 32, axis=1)
    out = torch.empty((rows, K), dtype=torch.uint16, device="cuda")
    B.moe_mxfp4_to_bf16(_t(codes), _t(scales), rows, K, out)
    torch.cuda.synchronize()
    got = O.bf16_to_f64(out.cpu().numpy())
    want = O.mxfp4_decode(codes, scales)
    fin = np.isfinite(want)
    assert np.array_equal(got[fin], want[fin])             # exact, subnormals included
    assert np.array_equal(np.signbit(got[fin]), np.signbit(want[fin]))
    assert np.all(np.isnan(got[-1]))                       # E8M0 0xFF is NaN


# ------------------------------------------------------------------ router --

ROUTER_CASES = [
    ("fixture", None),
    ("20b", 512),
    ("128a4", 512),
    ("248a20", 256),
]


def _route_gpu(inp, T):
    from sparse_moe_layer_05_b200 import binding as B
    ws = torch.empty(B.moe_route_workspace_size(inp.E, inp.k, T, inp.d), dtype=torch.uint8,
                     device="cuda")
    idx = torch.empty((T, inp.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, inp.k), dtype=torch.float32, device="cuda")
    counts = torch.empty(inp.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(inp.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * inp.k, dtype=torch.int32, device="cuda")
    B.moe_route(_t(inp.x[:T]), _t(inp.W_r), _t(inp.b_r), inp.E, inp.k, T, inp.d, idx, w,
                counts, offsets, perm, ws)
    assert B.moe_sync_status(ws) == 0
    return (idx.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy(),
            perm.cpu().numpy())


@pytest.mark.parametrize("name,T", ROUTER_CASES)
def test_router_topk_softmax_and_permutation(name, T):
    inp = W.make_inputs(name, T=T) if T else W.make_inputs(name)
    T = inp.T
    idx, w, counts, offsets, perm = _route_gpu(inp, T)
    r = O.route(inp.x, inp.W_r, inp.b_r, inp.k)
    G.compare_routing(idx, w, r)
    assert np.all(np.abs(w.sum(1) - 1) < 1e-6)
    # the permutation is integer work: bit-exact against the oracle's tables
    # built from the GPU's own selection
    c, o, p, _ = O.routing_tables(idx, inp.E)
    assert np.array_equal(counts, c) and np.array_equal(offsets, o) and np.array_equal(perm, p)


def test_router_silent_init_copies_tie_exactly():
    base = W.make_inputs("20b", T=256)
    exp = W.make_inputs("64a8", T=256)
    i2, w2, *_ = _route_gpu(base, 256)
    i8, w8, *_ = _route_gpu(exp, 256)
    for t in range(256):
        assert sorted(set(e % 32 for e in i8[t])) == sorted(i2[t].tolist())
        # copies get bit-identical logits, so equal weights, and the lower
        # index first (copy e+32 right after its original e)
        for j in range(0, 8, 2):
            assert i8[t, j + 1] == i8[t, j] + 32 and w8[t, j] == w8[t, j + 1]
    G.compare_routing(i8, w8, O.route(exp.x, exp.W_r, exp.b_r, 8), copies_of=32)


@pytest.mark.parametrize("d,E,k,T", [(64, 256, 32, 300), (2880, 248, 20, 512), (64, 4, 2, 1000),
                                     (96, 40, 8, 400), (2880, 128, 4, 257)],
                         ids=["E256_k32", "E248_k20", "E4", "d96", "T257"])
def test_router_tensor_core_path(d, E, k, T):
    """The tensor-core router (fp32 router weights as three bf16 terms, logits
    split over a cluster, top-k with fp64 near-tie refinement) at shapes off the
    workloads: the choice on every token against the oracle, the tables
    bit-exact. Cases: 256 expert columns (two stages, two accumulators), 4
    experts padded to 16, d = 32 mod 64 (a half-empty last k-block), a ragged last
    128-token tile."""
    inp = W.make_custom(d, 64, E, k, T, seed=90 + E)
    idx, w, counts, offsets, perm = _route_gpu(inp, T)
    r = O.route(inp.x, inp.W_r, inp.b_r, k)
    ties = G.compare_routing(idx, w, r)
    G.check_tables_against_oracle(idx, counts, offsets, perm, r, E)
    assert np.all(np.abs(w.sum(1) - 1) < 1e-6)
    print(f"[router] tensor-core path d={d} E={E} k={k} T={T}: near-ties {ties}")


def test_router_silent_init_copies_tie_exactly_tensor_cores():
    """Above 256 tokens (the tensor-core router) duplicated router rows still give
    bit-identical logits: each copy directly follows its original with an equal
    weight."""
    base = W.make_inputs("20b", T=512)
    exp = W.make_inputs("64a8", T=512)
    i2, w2, *_ = _route_gpu(base, 512)
    i8, w8, *_ = _route_gpu(exp, 512)
    for t in range(512):
        assert sorted(set(e % 32 for e in i8[t])) == sorted(i2[t].tolist())
        for j in range(0, 8, 2):
            assert i8[t, j + 1] == i8[t, j] + 32 and w8[t, j] == w8[t, j + 1]


def test_router_max_experts_and_k():
    inp = W.make_custom(64, 64, 256, 32, 100, seed=21)
    idx, w, counts, offsets, perm = _route_gpu(inp, 100)
    G.compare_routing(idx, w, O.route(inp.x, inp.W_r, inp.b_r, 32))
    c, o, p, _ = O.routing_tables(idx, 256)
    assert np.array_equal(perm, p) and np.array_equal(offsets, o)


@pytest.mark.parametrize("case", ["order_and_boundary", "chain_with_copies"])
def test_router_near_ties_settled_exactly(case):
    """Router rows that differ by ~1e-6 in their logits, far below the fp32
    tensor-core error (~1e-5) but far above two fp64 evaluations' (~1e-13):
    the choice and its order must be the exact ones on every token, which only
    the fp64 refinement of near ties can give. order_and_boundary: experts 0/1
    always selected (bias +6) with their order decided by the tiny gap, experts
    2/3 competing for the last slot (bias +3). chain_with_copies: sixteen
    near-identical rows (bias +6, k = 8 of them selected) and exact copies of
    four of them (equal logits: lower index first)."""
    d = 2880
    rng = np.random.default_rng(5)
    if case == "order_and_boundary":
        inp = W.make_custom(d, 64, 8, 3, 512, seed=77)
        for a, b, bias in [(0, 1, 6.0), (2, 3, 3.0)]:
            u = rng.standard_normal(d) / np.sqrt(d)
            inp.W_r[b] = (inp.W_r[a].astype(np.float64) + 1e-6 * u).astype(np.float32)
            inp.b_r[a] = inp.b_r[b] = bias
    else:
        inp = W.make_custom(d, 64, 64, 8, 512, seed=78)
        base = inp.W_r[0].astype(np.float64)
        for j in range(16):
            inp.W_r[j] = (base + 1e-6 * rng.standard_normal(d) / np.sqrt(d)).astype(np.float32)
            inp.b_r[j] = 6.0
        for j in range(4):
            inp.W_r[16 + j] = inp.W_r[j]
            inp.b_r[16 + j] = inp.b_r[j]
    T = inp.T
    idx, w, counts, offsets, perm = _route_gpu(inp, T)
    r = O.route(inp.x, inp.W_r, inp.b_r, inp.k)
    srt = -np.sort(-r.s, axis=1)
    gaps = -np.diff(srt[:, :inp.k + 1], axis=1)
    close = int(np.sum((gaps < 1e-4) & (gaps > 0)))
    assert close > T // 2, close          # the case really is full of near ties
    # copies at the k-th / (k+1)-th boundary tie exactly (an exempt token whose
    # choice is still validated); everything else must be exact
    ties = G.compare_routing(idx, w, r, max_exempt=T if case == "chain_with_copies" else None)
    G.check_tables_against_oracle(idx, counts, offsets, perm, r, inp.E)
    print(f"[router] near ties {case}: {close} gaps below 1e-4 among the top k+1, "
          f"exempt {ties}; every other choice and order exact")


def test_router_total_order_with_nan_and_inf_logits():
    """Logits that are NaN or infinite still give one selection that every lane of
    the warp agrees on, the oracle's: numbers in descending order, then -inf, then
    NaN; equal logits (and -0 against +0) to the lower index. A NaN row (expert 3),
    a -inf bias (expert 5) and a +0/-0 pair of zero rows (experts 6, 7)."""
    for E, k in [(8, 4), (8, 8), (40, 32)]:
        inp = W.make_custom(64, 64, E, k, 70, seed=71)
        inp.W_r[3] = np.nan
        inp.b_r[5] = -np.inf
        inp.W_r[6] = 0.0
        inp.W_r[7] = 0.0
        inp.b_r[6] = -0.0
        inp.b_r[7] = 0.0
        idx, w, counts, offsets, perm = _route_gpu(inp, inp.T)
        r = O.route(inp.x, inp.W_r, inp.b_r, k)
        assert np.array_equal(idx, r.idx)
        fin = np.isfinite(r.p)
        assert np.array_equal(fin, np.isfinite(w))
        assert np.all(np.abs(w[fin] - r.p[fin]) < 1e-5)
        c, o, p, _ = O.routing_tables(r.idx, E)
        assert np.array_equal(counts, c) and np.array_equal(offsets, o) and np.array_equal(perm, p)


# ----------------------------------------------------------------- forward --

FORWARD_CASES = [
    # name, d, I, E, k, T, seed   -- ragged M/N/K tails and several tiles
    ("fixture", 64, 128, 4, 2, 256, 0),
    ("ragged", 352, 224, 8, 2, 1000, 3),
    ("k1", 96, 160, 5, 1, 333, 4),
    ("kE", 128, 96, 4, 4, 130, 5),
    ("E1", 64, 64, 1, 1, 300, 6),
    ("single_token", 256, 256, 16, 4, 1, 7),
    ("wide", 2880, 2880, 32, 4, 192, 8),
]


@pytest.mark.parametrize("case", FORWARD_CASES, ids=[c[0] for c in FORWARD_CASES])
def test_forward_matches_oracle(case):
    from sparse_moe_layer_05_b200 import binding as B
    name, d, I, E, k, T, seed = case
    if name == "fixture":
        inp = W.make_inputs("fixture")
    else:
        inp = W.make_custom(d, I, E, k, T, seed=seed)
    out, layer = G.run_forward(inp)
    want, r, hidden = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                                    inp.Wd_codes, inp.Wd_scales, k=inp.k, return_hidden=True)
    G.assert_out_close(out, want)
    yw = layer.intermediate("yw", T).cpu().numpy().reshape(T, k, d)
    G.check_pre_rounding(out, yw, want, what=name,
                         h_bound=lambda: G.h_rounding_bound(inp, r, hidden))
    # kernel-level checks: routing and the SwiGLU hidden rows H (permuted order)
    idx = layer.intermediate("topk_idx", T).cpu().numpy()
    w = layer.intermediate("topk_w", T).cpu().numpy()
    G.compare_routing(idx, w, r)
    perm = layer.intermediate("perm", T).cpu().numpy()
    c, o, p, _ = O.routing_tables(idx, E)
    assert np.array_equal(perm, p)
    # the block-scaled path (no scale transposes: 2 launches fewer) keeps x and
    # H as hi/lo E4M3 rows, so the bf16 intermediates exist only on the other paths
    fused = 3 if T <= 256 else 0
    bf16_path = B.moe_forward_launch_count(E, k, T, d, I) == 12 - fused
    if np.array_equal(idx, r.idx) and bf16_path:
        H = O.bf16_to_f64(G.unpermute_chunks(layer.intermediate("h", T).cpu().numpy()))
        xp = G.unpermute_chunks(layer.intermediate("xp", T).cpu().numpy())
        assert np.array_equal(xp, inp.x[perm // k])
        for e, (toks, h) in hidden.items():
            rows = H[o[e]:o[e + 1]]
            assert np.array_equal(perm[o[e]:o[e + 1]] // k, toks)
            # H is stored in bf16: each element within one bf16 ulp of the
            # fp64 value, plus a small allowance for fp32 accumulation
            rms = np.sqrt(np.mean(h ** 2))
            bound = 2.0 ** -8 * np.abs(h) + 1e-3 * rms
            assert np.all(np.abs(rows - h) <= bound), (e, np.max(np.abs(rows - h) / (bound)))


PAIR_CASES = [
    # name, d, I, E, k, T, seed -- ragged M/N/K tails, many and few rows per expert
    ("pair_ragged", 352, 224, 4, 2, 1500, 31),
    ("pair_wide", 2880, 2880, 8, 2, 1100, 32),
    ("pair_short_tail", 128, 256, 6, 3, 700, 33),
    ("decode_wide", 2880, 2880, 64, 8, 64, 34),
    ("decode_ragged", 352, 224, 16, 2, 40, 35),
    ("decode_overflow", 256, 192, 4, 2, 150, 36),   # > 64 rows per expert: two token blocks
    ("mx_tails", 448, 320, 6, 2, 500, 37),           # K = 64 mod 128 in both GEMMs
    ("mx_decode_many", 2880, 2880, 128, 4, 32, 38),  # many experts with 0-3 rows
]


@pytest.mark.parametrize("policy", [1, 2, 3, 4, 5], ids=["single", "pair", "swap", "mx", "mx_pair"])
@pytest.mark.parametrize("case", PAIR_CASES, ids=[c[0] for c in PAIR_CASES])
def test_forward_both_tile_policies(case, policy):
    from sparse_moe_layer_05_b200 import binding as B
    name, d, I, E, k, T, seed = case
    inp = W.make_custom(d, I, E, k, T, seed=seed)
    # the policy travels with the call (moe_forward_ex), not through the
    # process default
    layer = B.MoELayer(inp)
    out_t = torch.empty((T, d), dtype=torch.uint16, device="cuda")
    B.moe_forward_ex(_t(inp.x), layer.W_r, layer.b_r, layer.Wgu_codes, layer.Wgu_scales,
                     layer.Wd_codes, layer.Wd_scales, E, k, T, d, I, out_t, layer.workspace,
                     tile_policy=policy)
    assert B.moe_sync_status(layer.workspace) == 0
    out = out_t.cpu().numpy()
    want, r, hidden = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                                    inp.Wd_codes, inp.Wd_scales, k=k, return_hidden=True)
    G.assert_out_close(out, want)
    G.check_pre_rounding(out, layer.intermediate("yw", T).cpu().numpy().reshape(T, k, d), want,
                         what=f"{name} policy {policy}",
                         h_bound=lambda: G.h_rounding_bound(inp, r, hidden))
    idx = layer.intermediate("topk_idx", T).cpu().numpy()
    # the block-scaled tiles keep H as hi/lo E4M3 rows, not bf16
    mx = policy in (4, 5) and d % 64 == 0 and I % 64 == 0 and min(d, I) >= 128
    if np.array_equal(idx, r.idx) and not mx:
        c, o, p, _ = O.routing_tables(idx, E)
        H = O.bf16_to_f64(G.unpermute_chunks(layer.intermediate("h", T).cpu().numpy()))
        for e, (toks, h) in hidden.items():
            rms = np.sqrt(np.mean(h ** 2))
            assert np.all(np.abs(H[o[e]:o[e + 1]] - h) <= 2.0 ** -8 * np.abs(h) + 1e-3 * rms), e


BIAS_CASES = [
    # name, d, I, E, k, T, seed
    ("bias_ragged", 352, 224, 8, 2, 1000, 51),
    ("bias_decode", 2880, 2880, 32, 4, 64, 52),
    ("bias_mx_tails", 448, 320, 6, 2, 500, 53),
]


def _expert_biases(inp, seed, gu=True, down=True):
    """Per-expert biases on the scale of the terms they join: the gate/up
    pre-activations and the expert outputs (RMS estimated from expert 0)."""
    rng = np.random.default_rng(seed)
    xf = O.bf16_to_f64(inp.x[:64])
    pre = xf @ O.mxfp4_decode(inp.Wgu_codes[0], inp.Wgu_scales[0]).T
    y = O.expert_out(O.expert_hidden(xf, O.mxfp4_decode(inp.Wgu_codes[0], inp.Wgu_scales[0]),
                                     inp.I), O.mxfp4_decode(inp.Wd_codes[0], inp.Wd_scales[0]))
    rms = lambda a: float(np.sqrt(np.mean(a ** 2)))
    Bgu = (rng.standard_normal((inp.E, 2 * inp.I)) * rms(pre)).astype(np.float32) if gu else None
    Bd = (rng.standard_normal((inp.E, inp.d)) * rms(y)).astype(np.float32) if down else None
    return Bgu, Bd


@pytest.mark.parametrize("policy", [1, 2, 3, 4, 5], ids=["single", "pair", "swap", "mx", "mx_pair"])
@pytest.mark.parametrize("case", BIAS_CASES, ids=[c[0] for c in BIAS_CASES])
def test_forward_expert_biases(case, policy):
    """Gate/up biases before the silu and down biases before the routing weight,
    in every tile family's epilogue; the output must also move away from the
    unbiased layer by far more than the tolerance."""
    from sparse_moe_layer_05_b200 import binding as B
    name, d, I, E, k, T, seed = case
    inp = W.make_custom(d, I, E, k, T, seed=seed)
    Bgu, Bd = _expert_biases(inp, seed + 100)
    layer = B.MoELayer(inp)
    out = torch.empty((T, d), dtype=torch.uint16, device="cuda")
    B.moe_set_tile_policy(policy)
    try:
        B.moe_forward_biased(_t(inp.x), layer.W_r, layer.b_r, layer.Wgu_codes, layer.Wgu_scales,
                             _t(Bgu), layer.Wd_codes, layer.Wd_scales, _t(Bd), E, k, T, d, I, out,
                             layer.workspace)
        assert B.moe_sync_status(layer.workspace) == 0
    finally:
        B.moe_set_tile_policy(0)
    got = out.cpu().numpy()
    args = (inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes, inp.Wd_scales)
    want = O.moe_forward(*args, k=k, Bgu=Bgu.astype(np.float64), Bd=Bd.astype(np.float64))
    G.assert_out_close(got, want)
    plain = O.moe_forward(*args, k=k)
    assert G.rel_rms_err(O.bf16_to_f64(got), plain)[0] > 10 * G.TOL_REL_RMS


@pytest.mark.parametrize("which", ["gate_up_only", "down_only"])
def test_forward_one_bias_and_block_with_biases(which):
    """Either bias alone (the other NULL), through moe_forward_biased and through
    moe_forward_block (norm, layer with biases, residual)."""
    from sparse_moe_layer_05_b200 import binding as B
    d, I, E, k, T = 2880, 2880, 16, 4, 96
    inp = W.make_custom(d, I, E, k, T, seed=61)
    Bgu, Bd = _expert_biases(inp, 62, gu=which == "gate_up_only", down=which == "down_only")
    tb = lambda a: None if a is None else _t(a)
    f64 = lambda a: None if a is None else a.astype(np.float64)
    layer = B.MoELayer(inp)
    out = torch.empty((T, d), dtype=torch.uint16, device="cuda")
    B.moe_forward_biased(_t(inp.x), layer.W_r, layer.b_r, layer.Wgu_codes, layer.Wgu_scales,
                         tb(Bgu), layer.Wd_codes, layer.Wd_scales, tb(Bd), E, k, T, d, I, out,
                         layer.workspace)
    assert B.moe_sync_status(layer.workspace) == 0
    args = (inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes, inp.Wd_scales)
    G.assert_out_close(out.cpu().numpy(), O.moe_forward(inp.x, *args, k=k, Bgu=f64(Bgu),
                                                        Bd=f64(Bd)))
    rng = np.random.default_rng(63)
    h = W.f32_to_bf16_bits((O.bf16_to_f64(inp.x) * 2.0 - 0.25).astype(np.float32))
    g = rng.uniform(0.5, 1.5, size=d).astype(np.float32)
    ht, gt = _t(h), torch.from_numpy(g).cuda()
    xt = torch.empty_like(ht)
    B.moe_rms_norm(ht, gt, 1e-5, T, d, xt)
    ws = torch.empty(B.moe_workspace_size_block(E, k, T, d, I), dtype=torch.uint8, device="cuda")
    B.moe_forward_block(ht, gt, 1e-5, layer.W_r, layer.b_r, layer.Wgu_codes, layer.Wgu_scales,
                        layer.Wd_codes, layer.Wd_scales, E, k, T, d, I, out, ws,
                        gu_bias=tb(Bgu), down_bias=tb(Bd))
    assert B.moe_sync_status(ws) == 0
    got = O.bf16_to_f64(out.cpu().numpy())
    want = O.moe_block(h, g, 1e-5, *args, k=k, x_bits=xt.cpu().numpy(), Bgu=f64(Bgu), Bd=f64(Bd))
    ff = want - O.bf16_to_f64(h)
    bound = 2e-2 * np.sqrt(np.mean(ff ** 2)) + 2.0 ** -8 * np.abs(want)
    assert np.all(np.abs(got - want) <= bound), np.max(np.abs(got - want) / bound)


def _e4m3_to_f64(b):
    b = b.astype(np.int64)
    e, m = (b >> 3) & 15, b & 7
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * np.exp2(e - 7.0))
    v = np.where((b & 0x7F) == 0x7F, np.nan, v)
    return np.where(b >> 7, -v, v)


def test_mx_split_is_exact_above_the_group_floor():
    """hi/lo E4M3 split of bf16 rows: x = 2^(s_hi-127) hi + 2^(s_lo-127) lo, exact for
    every element of at least 2^-13 of its group's max |x|, within 2^-21 of that max
    otherwise (groups with max |x| >= 2^-116). Groups cover N(0,1), wide exponent
    spreads, zeros and scales near both ends of that range."""
    from sparse_moe_layer_05_b200 import binding as B
    rng = np.random.default_rng(5)
    R, K = 64, 2880
    x = rng.standard_normal((R, K))
    x *= np.exp2(rng.integers(-40, 40, size=(R, K // 32, 1)).astype(float)).repeat(32, 2).reshape(R, K)
    x[1] = rng.standard_normal(K) * np.exp2(rng.uniform(-30, 0, size=K))  # far below the max
    x[2] = 0.0
    x[3, :32] = 0.0
    x[4] = rng.standard_normal(K) * 2.0 ** 100
    x[5] = rng.standard_normal(K) * 2.0 ** -105
    xb = W.f32_to_bf16_bits(x.astype(np.float32))
    hi = torch.empty((R, K), dtype=torch.uint8, device="cuda")
    lo = torch.empty_like(hi)
    sc = torch.empty((R, K // 32, 2), dtype=torch.uint8, device="cuda")
    B.moe_mx_split_e4m3(_t(xb), R, K, hi, lo, sc)
    torch.cuda.synchronize()
    sc = sc.cpu().numpy().astype(np.int64)
    s_hi = np.exp2(sc[..., 0] - 127.0).repeat(32, 1)
    s_lo = np.exp2(sc[..., 1] - 127.0).repeat(32, 1)
    rec = _e4m3_to_f64(hi.cpu().numpy()) * s_hi + _e4m3_to_f64(lo.cpu().numpy()) * s_lo
    xv = O.bf16_to_f64(xb)
    gmax = np.abs(xv).reshape(R, K // 32, 32).max(axis=2).repeat(32, 1)
    big = np.abs(xv) >= 2.0 ** -13 * gmax
    assert np.all(np.isfinite(rec))
    assert np.array_equal(rec[big], xv[big])
    assert np.all(np.abs(rec - xv)[~big] <= 2.0 ** -21 * gmax[~big])
    assert np.all(sc[..., 1] == sc[..., 0] - 4)


@pytest.mark.parametrize("d,I,E,k,T", [(2880, 2880, 32, 4, 64), (352, 224, 8, 2, 500)],
                         ids=["block_scaled_decode", "bf16_tiles"])
def test_forward_block_rms_norm_and_residual(d, I, E, k, T):
    """out = h + MoE(RMSNorm(h)): the norm against the oracle within one bf16 ulp, then
    the block against h + MoE(x) computed by the oracle from the same normalised rows,
    with the layer's tolerance on the sublayer term plus the output's bf16 rounding."""
    from sparse_moe_layer_05_b200 import binding as B
    inp = W.make_custom(d, I, E, k, T, seed=41)
    rng = np.random.default_rng(42)
    h = W.f32_to_bf16_bits((O.bf16_to_f64(inp.x) * 3.0 + 0.5).astype(np.float32))
    g = rng.uniform(0.5, 1.5, size=d).astype(np.float32)
    eps = 1e-5
    layer = B.MoELayer(inp)
    ht, gt = _t(h), torch.from_numpy(g).cuda()
    xt = torch.empty_like(ht)
    B.moe_rms_norm(ht, gt, eps, T, d, xt)
    torch.cuda.synchronize()
    x_gpu = xt.cpu().numpy()
    x_or = O.f64_to_bf16_bits(O.rms_norm(O.bf16_to_f64(h), g.astype(np.float64), eps))
    a, b = O.bf16_to_f64(x_gpu), O.bf16_to_f64(x_or)
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)))
    ws = torch.empty(B.moe_workspace_size_block(E, k, T, d, I), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.uint16, device="cuda")
    B.moe_forward_block(ht, gt, eps, layer.W_r, layer.b_r, layer.Wgu_codes, layer.Wgu_scales,
                        layer.Wd_codes, layer.Wd_scales, E, k, T, d, I, out, ws)
    assert B.moe_sync_status(ws) == 0
    got = O.bf16_to_f64(out.cpu().numpy())
    want = O.moe_block(h, g, eps, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
                       inp.Wd_scales, k=k, x_bits=x_gpu)
    ff = want - O.bf16_to_f64(h)
    bound = 2e-2 * np.sqrt(np.mean(ff ** 2)) + 2.0 ** -8 * np.abs(want)
    assert np.all(np.abs(got - want) <= bound), np.max(np.abs(got - want) / bound)


@pytest.mark.parametrize("T", [600, 4099], ids=["one_piece", "chunked"])
def test_forward_deterministic_and_hostio_equal(T):
    """Repeated forwards agree bit for bit; so does the host-buffer call, which
    processes batches of 2048+ tokens as pipelined chunks (4099: a short last one)."""
    from sparse_moe_layer_05_b200.binding import MoELayer
    inp = W.make_custom(352, 224, 8, 2, T, seed=12)
    out1, layer = G.run_forward(inp)
    out2, _ = G.run_forward(inp, layer=layer)
    assert np.array_equal(out1, out2)
    hl = MoELayer(inp, hostio=True)
    xh = torch.from_numpy(inp.x).pin_memory()
    oh = torch.empty((inp.T, inp.d), dtype=torch.uint16).pin_memory()
    for _ in range(2):          # the second call reuses the copy streams
        oh.zero_()
        hl.forward_hostio(xh, oh)
        assert np.array_equal(oh.numpy(), out1)


def test_hostio_concurrent_threads():
    """Two host threads run chunked host-buffer forwards on one device at once
    (separate layers and workspaces, shared copy streams): every result equals the
    device-buffer forward."""
    import threading
    from sparse_moe_layer_05_b200.binding import MoELayer
    T = 4099
    inp = W.make_custom(352, 224, 8, 2, T, seed=12)
    want, _ = G.run_forward(inp)
    layers = [MoELayer(inp, hostio=True) for _ in range(2)]
    xh = torch.from_numpy(inp.x).pin_memory()
    outs = [torch.empty((T, inp.d), dtype=torch.uint16).pin_memory() for _ in range(2)]
    errors = []

    def work(i):
        try:
            torch.cuda.set_device(0)
            with torch.cuda.stream(torch.cuda.Stream()):
                for _ in range(4):
                    outs[i].zero_()
                    layers[i].forward_hostio(xh, outs[i])
                    if not np.array_equal(outs[i].numpy(), want):
                        errors.append(i)
        except Exception as e:          # reported below, on the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=work, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors


def test_timed_events_sparse_mask():
    """Only the masked boundaries are timed (others read 0; a recorded one spans to
    the next recorded), the output is moe_forward's bit for bit, and mask bits above
    the last boundary are rejected."""
    from sparse_moe_layer_05_b200 import binding as B
    for T in (64, 600):                        # block-scaled and bf16 tiles
        inp = W.make_custom(448, 320, 8, 2, T, seed=17)
        want, layer = G.run_forward(inp)
        x = _t(inp.x)
        out = torch.empty((T, inp.d), dtype=torch.uint16, device="cuda")
        nb = len(B.STAGES)
        dom = B.STAGES.index("gemm_gateup_swiglu")
        ms = layer.forward_timed_events(x, out, (1 << dom) | (1 << (dom + 1)))
        assert np.array_equal(out.cpu().numpy(), want)
        assert all(ms[i] == 0.0 for i in range(nb) if i not in (0, dom, dom + 1))
        assert ms[dom] > 0 and ms[dom + 1] > 0 and ms[0] > 0
        assert abs(ms[0] + ms[dom] + ms[dom + 1] - ms[nb]) <= 1e-3 + 1e-3 * ms[nb]
        full = layer.forward_timed(x, out)
        assert all(v >= 0 for v in full) and full[nb] > 0
        with pytest.raises(B.MoEError):
            layer.forward_timed_events(x, out, 1 << (nb + 1))


def test_skewed_routing_and_empty_experts():
    inp = W.make_custom(128, 128, 16, 2, 700, seed=13)
    inp.b_r[3] += 50.0            # every token picks expert 3
    inp.b_r[[5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15]] -= 50.0   # never chosen
    out, layer = G.run_forward(inp)
    want = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
                         inp.Wd_scales, k=2)
    G.assert_out_close(out, want)
    counts = layer.intermediate("counts", inp.T).cpu().numpy()
    assert counts[3] == 700 and counts[5:].sum() == 0


def test_zero_tokens_is_a_no_op():
    from sparse_moe_layer_05_b200 import binding as B
    inp = W.make_custom(64, 64, 4, 2, 8, seed=1)
    from sparse_moe_layer_05_b200.binding import MoELayer
    layer = MoELayer(inp)
    x = torch.empty((0, 64), dtype=torch.uint16, device="cuda")
    out = torch.empty((1, 64), dtype=torch.uint16, device="cuda")  # non-null, untouched
    B.moe_forward(x if x.numel() else out, layer.W_r, layer.b_r, layer.Wgu_codes,
                  layer.Wgu_scales, layer.Wd_codes, layer.Wd_scales, 4, 2, 0, 64, 64, out,
                  layer.workspace)
    torch.cuda.synchronize()


def test_silent_init_identity_on_gpu():
    """64a8 (x2 silent init) and 96a12 (x3) reproduce 32a4 at T = 64 (decode,
    block-scaled tiles) and T = 512 (bf16 tiles)."""
    for T in (64, 512):
        base = W.make_inputs("20b", T=T)
        o2, _ = G.run_forward(base)
        want = O.bf16_to_f64(o2)
        for name in ("64a8", "96a12"):
            exp = W.make_inputs(name, T=T)
            o8, _ = G.run_forward(exp)
            G.assert_out_close(o8, want, what=f"{name} vs 20b at T={T}")


def test_reduced_active_count_on_gpu():
    """64a4 (the x2 layer at k = 4) reproduces the 20b layer at k = 2; 96a4 (the x3
    layer at k = 4: three copies of the best expert, one of the second) matches the
    oracle on sampled tokens. T = 64 (block-scaled tiles) and 512 (bf16 tiles)."""
    for T in (64, 512):
        base = W.make_inputs("20b", T=T)
        base.k = 2
        o2, _ = G.run_forward(base)
        o4, _ = G.run_forward(W.make_inputs("64a4", T=T))
        G.assert_out_close(o4, O.bf16_to_f64(o2), what=f"64a4 vs 20b at k=2, T={T}")
        inp = W.make_inputs("96a4", T=T)
        o3, _ = G.run_forward(inp)
        toks = np.sort(np.random.default_rng(T).choice(T, size=12, replace=False))
        want = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                             inp.Wd_codes, inp.Wd_scales, k=4, tokens=toks)
        G.assert_out_close(o3[toks], want, what=f"96a4 T={T} sampled")


def test_timeout_path_reports_status_and_device_survives():
    from sparse_moe_layer_05_b200 import binding as B
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    B.moe_selftest_wait_timeout(ws)
    assert B.moe_sync_status(ws) == 5          # MOE_ERR_TIMEOUT
    assert B.moe_sync_status(ws) == 0          # cleared
    inp = W.make_inputs("fixture")
    out, _ = G.run_forward(inp)                # the context is still usable
    want = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
                         inp.Wd_scales, k=2)
    G.assert_out_close(out, want)


# ------------------------------------------------ full sizes, every config ----

# Every workload the benchmark names, at its prefill and decode batch sizes.
FULL_CASES = [
    ("20b", 8192),
    ("64a8", 8192),
    ("64a8", 64),
    ("128a4", 16384),
    ("128a4", 32),
    ("248a20", 4096),
    ("248a20", 16),
]
N_OUT_TOKENS = 256       # tokens whose outputs are compared with the oracle


def _output_tokens(T, k, offsets, perm, seed):
    """All tokens of a small batch; otherwise the first and the last token of
    every expert's segment (so every expert and every segment's last tile is
    checked) plus random tokens, at least N_OUT_TOKENS in all."""
    if T <= N_OUT_TOKENS:
        return np.arange(T)
    chosen = set()
    for e in range(len(offsets) - 1):
        if offsets[e + 1] > offsets[e]:
            chosen.add(int(perm[offsets[e]]) // k)
            chosen.add(int(perm[offsets[e + 1] - 1]) // k)
    rng = np.random.default_rng(seed)
    rest = rng.permutation(T)
    for t in rest:
        if len(chosen) >= N_OUT_TOKENS:
            break
        chosen.add(int(t))
    return np.array(sorted(chosen))


@pytest.mark.parametrize("name,T", FULL_CASES, ids=[f"{n}-T{t}" for n, t in FULL_CASES])
def test_full_size_every_token_routed_and_sampled_outputs(name, T):
    """At the full batch of every configuration: the router's fp32 logits within
    their error bound on every token; top-k indices, weights, counts, offsets
    and the permutation against the oracle on every token (exact ties below
    NEAR_TIE are counted and printed; their choice must still be valid);
    outputs of at least 256 tokens,
    among them every expert's first and last routed token, against the oracle,
    both as the bf16 output (tolerance plus the output's own rounding) and,
    strictly, as the fp32 sum before that rounding."""
    inp = W.make_inputs(name, T=T)
    out, layer = G.run_forward(inp)
    assert G.torch_mod().cuda.is_available()
    from sparse_moe_layer_05_b200 import binding as B
    assert B.moe_sync_status(layer.workspace) == 0
    idx = layer.intermediate("topk_idx", T).cpu().numpy()
    w = layer.intermediate("topk_w", T).cpu().numpy()
    counts = layer.intermediate("counts", T).cpu().numpy()
    offsets = layer.intermediate("offsets", T).cpu().numpy()
    perm = layer.intermediate("perm", T).cpu().numpy()
    r = O.route(inp.x, inp.W_r, inp.b_r, inp.k)
    G.check_router_logits(layer.intermediate("logits", T).cpu().numpy(), r, inp.x, inp.W_r,
                          what=f"{name} T={T}")
    copies = 32 if name == "64a8" else None
    ties = G.compare_routing(idx, w, r, copies_of=copies, max_exempt=max(2, T // 1000))
    same = G.check_tables_against_oracle(idx, counts, offsets, perm, r, inp.E)
    assert np.all(np.abs(w.sum(1) - 1) < 1e-6)
    toks = _output_tokens(T, inp.k, offsets, perm, seed=T)
    want = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
                         inp.Wd_scales, k=inp.k, tokens=toks)
    r_out = G.assert_out_close(out[toks], want, what=f"{name} T={T}")
    tt = torch.from_numpy(toks).cuda()
    rows = (tt[:, None] * inp.k + torch.arange(inp.k, device="cuda")[None, :]).reshape(-1)
    yw = layer.intermediate("yw", T).index_select(0, rows).cpu().numpy()
    r_pre = G.check_pre_rounding(out[toks], yw.reshape(len(toks), inp.k, inp.d), want,
                                 what=f"{name} T={T}")
    print(f"[parity] {name} T={T}: near-ties {ties} of {T} tokens; routing tables "
          f"{'equal the oracle' if same else 'of the GPU choice'}; {len(toks)} tokens vs oracle: "
          f"bf16 out max|err|/RMS {r_out:.3e}, fp32 pre-rounding {r_pre:.3e}")


def test_full_size_silent_init_prefill():
    base = W.make_inputs("20b")
    o2, l2 = G.run_forward(base)
    del l2
    torch.cuda.empty_cache()
    exp = W.make_inputs("64a8")
    o8, _ = G.run_forward(exp)
    G.assert_out_close(o8, O.bf16_to_f64(o2), what="64a8 vs 20b at T=8192")
