"""The activation-quantised layers (w4a8: MXFP8 E4M3 activations, w4a4: MXFP4
E2M1 activations; moe_forward_ex act_quant) against the oracle's simulation of
the same conversion (``moe_forward(act_quant=...)``, the OCP Microscaling
conversion). The quantised function is deterministic, so each step is checked
where its result is unique:

* the conversion of bf16 values (x) is bit-exact: both sides round exact inputs;
* the conversion of H, whose fp32 (GPU) and fp64 (oracle) values differ by
  accumulation order, agrees except where the oracle's H lies at a rounding
  midpoint, within fp32 accumulation error of it; such elements are counted and
  each may take either of the two neighbouring grid values;
* the down projection of the GPU's own converted H matches the fp64 product of
  the same values within fp32 accumulation error (2e-3 x RMS);
* the layer output is reported against the simulated layer (2e-2 x RMS plus the
  bf16 output's rounding, the layer's own tolerance).
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from sparse_moe_layer_05_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MODES = {"mxfp8": "e4m3", "mxfp4": "e2m1"}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_moe_layer_05_b200 import build
    build.build()


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _conversion_inputs(K):
    """bf16 rows that exercise the conversion: N(0,1) groups; groups spread over
    many binades; exact midpoints between neighbouring E4M3 and E2M1 values (ties
    to even), the clamping range just below the next power of two, element
    subnormals, zero groups, and very large and very small groups."""
    rng = np.random.default_rng(11)
    rows = [rng.standard_normal(K)]
    rows.append(rng.standard_normal(K) * np.exp2(rng.integers(-20, 20, size=K)))
    g = K // 32
    # E4M3 midpoints: m/16 + 1/32 over [1, 2) times a power of two, max 2^8 sets X = 1
    mid8 = (1.0 + (np.arange(32) % 8) / 8.0 + 1.0 / 16.0) * np.exp2(np.arange(32) % 9 - 1)
    mid8[0] = 256.0
    rows.append(np.tile(mid8, g) * np.exp2(rng.integers(-6, 6, size=g)).repeat(32))
    # E2M1 midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 with max 4 (X = 1)
    mid4 = np.array([4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4)
    mid4 = mid4 * np.where(np.arange(32) % 3 == 0, -1.0, 1.0)
    mid4[0] = 4.0
    rows.append(np.tile(mid4, g) * np.exp2(rng.integers(-6, 6, size=g)).repeat(32))
    # clamping: magnitudes in [448, 512) and [6, 8) after the scale
    rows.append(np.tile(np.linspace(256.0, 511.0, 32), g))
    rows.append(np.tile(np.linspace(4.0, 7.96875, 32), g))
    # element subnormals: small values next to a large one in each group
    sub = rng.standard_normal(K) * 2.0 ** -12
    sub[::32] = 3.0
    rows.append(sub)
    rows.append(np.zeros(K))
    rows.append(rng.standard_normal(K) * 2.0 ** 60)
    rows.append(rng.standard_normal(K) * 2.0 ** -60)
    x = np.stack(rows)
    return W.f32_to_bf16_bits(x.astype(np.float32))


@pytest.mark.parametrize("mode", list(MODES))
def test_conversion_is_the_oracle_conversion(mode):
    """moe_mx_quantize (the kernels' conversion) equals the oracle's mx_quantize on
    every element, scale bytes included."""
    from sparse_moe_layer_05_b200 import binding as B
    elem = MODES[mode]
    K = 2880
    xb = _conversion_inputs(K)
    R = xb.shape[0]
    qcols = K if elem == "e4m3" else K // 2
    q = torch.empty((R, qcols), dtype=torch.uint8, device="cuda")
    sc = torch.empty((R, K // 32), dtype=torch.uint8, device="cuda")
    B.moe_mx_quantize(_t(xb), R, K, mode, q, sc)
    torch.cuda.synchronize()
    got = G.mx_dequant(q.cpu().numpy(), sc.cpu().numpy(), elem)
    want = O.mx_quantize(O.bf16_to_f64(xb), elem)
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]
    # the shared scale is 2^(floor(log2 max|x|) - emax) for every non-zero group
    xv = O.bf16_to_f64(xb).reshape(R, K // 32, 32)
    amax = np.abs(xv).max(axis=2)
    nz = amax > 0
    emax = 8 if elem == "e4m3" else 2
    want_s = np.frexp(np.where(nz, amax, 1.0))[1] - 1 - emax + 127
    assert np.array_equal(sc.cpu().numpy()[nz].astype(int), want_s[nz])


QUANT_CASES = [
    # name, d, I, E, k, T, seed -- 16-token tiles (few rows per expert), 128-token
    # tiles with ragged tails, and K = 64 mod 128 in both GEMMs
    ("decode", 2880, 2880, 32, 4, 64, 81),
    ("prefill_ragged", 448, 320, 6, 2, 900, 82),
    ("prefill_wide", 2880, 2880, 8, 2, 1200, 83),
]


@pytest.mark.parametrize("policy", [0, 4, 5], ids=["by_shape", "one_cta", "cta_pair"])
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("case", QUANT_CASES, ids=[c[0] for c in QUANT_CASES])
def test_quantised_layer_against_the_simulation(case, mode, policy):
    from sparse_moe_layer_05_b200 import binding as B
    elem = MODES[mode]
    name, d, I, E, k, T, seed = case
    if policy != 0 and T * k < 64 * E:
        pytest.skip("few rows per expert: the 16-token tiles run either way")
    inp = W.make_custom(d, I, E, k, T, seed=seed)
    layer = B.MoELayer(inp)
    out_t = torch.empty((T, d), dtype=torch.uint16, device="cuda")
    B.moe_forward_ex(_t(inp.x), layer.W_r, layer.b_r, layer.Wgu_codes, layer.Wgu_scales,
                     layer.Wd_codes, layer.Wd_scales, E, k, T, d, I, out_t, layer.workspace,
                     tile_policy=policy, act_quant=mode)
    assert B.moe_sync_status(layer.workspace) == 0
    out = out_t.cpu().numpy()
    want, r, hidden = O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales,
                                    inp.Wd_codes, inp.Wd_scales, k=k, act_quant=elem,
                                    return_hidden=True)
    idx = layer.intermediate("topk_idx", T).cpu().numpy()
    G.compare_routing(idx, layer.intermediate("topk_w", T).cpu().numpy(), r)
    assert np.array_equal(idx, r.idx), "near-tie in this seeded case: pick another seed"
    offsets = layer.intermediate("offsets", T).cpu().numpy()
    perm = layer.intermediate("perm", T).cpu().numpy()
    topk_w = layer.intermediate("topk_w", T).cpu().numpy()
    P = T * k
    NT = G.mx_tile_tokens(P, E, elem)
    pr = G.mx_padded_rows(offsets, NT)
    L = layer.layout(T)
    ws = layer.workspace.cpu().numpy()
    qb = 1 if elem == "e4m3" else 2                   # elements per byte

    # the CTA-pair tiles run where forced (policy 5) and, picked by shape, from
    # 192 rows per expert; w4a4 on them runs kind::mxf4 (d, I >= 256), whose
    # scale blocks are laid out per 256-wide k-block
    pair = P >= 64 * E and (policy == 5 or (policy == 0 and P >= 192 * E))
    f4 = mode == "mxfp4" and pair and min(d, I) >= 256

    def rows_of(region, scales, K):
        q = ws[L[region]:L[region] + (int(pr.max()) + 1) * K // qb].reshape(-1, K // qb)[pr]
        s = G.mx_scale_bytes(ws[L[scales]:], pr, K, NT, kb256=f4)
        return G.mx_dequant(q, s, elem)

    # (a) x: bit-exact conversion of each routed token's row
    xq = rows_of("xp", "x_scales", d)
    assert np.array_equal(xq, O.mx_quantize(O.bf16_to_f64(inp.x[perm // k]), elem))
    # (b) H: equal except at rounding midpoints of the fp64 value
    hq = rows_of("h", "h_scales", I)
    flips = total = 0
    wq_of = {}
    for e, (toks, h) in hidden.items():
        got = hq[offsets[e]:offsets[e + 1]]
        wq = O.mx_quantize(h, elem)
        wq_of[e] = wq
        total += got.size
        bad = got != wq
        if not bad.any():
            continue
        gmax = np.abs(h).reshape(h.shape[0], -1, 32).max(axis=2).repeat(32, axis=1)
        # either neighbour of a midpoint is a correct rounding: the fp64 value
        # must lie within fp32 accumulation error of the two values' midpoint
        near = np.abs(h - 0.5 * (got + wq)) <= 1e-5 * gmax
        assert np.all(near[bad]), (e, np.argwhere(bad & ~near)[:3])
        flips += int(bad.sum())
    assert flips <= max(8, total // 10000), (flips, total)
    # (c) the down projection of the GPU's own converted H, weighted and summed
    yw = layer.intermediate("yw", T).cpu().numpy().reshape(T, k, d)
    pre = G.slot_sum_f32(yw)
    exp = np.zeros((T, d))       # the GPU's converted H through the fp64 down projection
    flip = np.zeros((T, d))      # what the H midpoint flips alone contribute
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        wd = O.mxfp4_decode(inp.Wd_codes[e], inp.Wd_scales[e])
        pairs = perm[a:b]
        pw = topk_w.reshape(-1)[pairs][:, None].astype(np.float64)
        np.add.at(exp, pairs // k, pw * (hq[a:b] @ wd.T))
        np.add.at(flip, pairs // k, pw * ((hq[a:b] - wq_of[e]) @ wd.T))
    rd, rms_d, _ = G.rel_rms_err(pre.astype(np.float64), exp)
    assert rd <= 2e-3, rd
    assert np.array_equal(out, G.f32_to_bf16_rne(pre))
    # (d) the layer against the simulated layer: within the layer's tolerance
    # plus the bf16 output's rounding, once the flips' own contribution (either
    # rounding of a midpoint value is correct) is allowed for
    got = O.bf16_to_f64(out)
    r_out, rms, _ = G.rel_rms_err(got, want)
    bound = G.TOL_REL_RMS * rms + G.BF16_REL * np.abs(want) + np.abs(flip)
    excess = np.abs(got - want) / bound
    assert np.all(excess <= 1.0), (mode, name, float(excess.max()), r_out)
    print(f"[act_quant] {mode} {name} policy {policy}: H midpoint flips {flips} of {total} "
          f"(moving the layer by up to {np.abs(flip).max() / rms:.2e} x RMS); down GEMM on the "
          f"GPU's H {rd:.2e} x RMS; layer vs simulation {r_out:.3e} x RMS")
