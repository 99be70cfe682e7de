"""Helpers shared by the GPU parity tests: upload a workload, run the CUDA path
through the C ABI, and compare with the oracle."""
import numpy as np

from oracle import moe_oracle as O

TOL_REL_RMS = 2e-2       # |err| <= 2e-2 * RMS(oracle out) ...
BF16_REL = 2.0 ** -8     # ... + the bf16 output's own rounding, 2^-8 |oracle value|
# The router settles every gap below its refinement margin on fp64 logits, so
# its choice is the exact one; two fp64 evaluations of a logit (the oracle's
# and the router's, summed in different orders) differ by ~1e-13 relative.
# Only gaps below this are exempt from index parity (equal logits, e.g. copied
# router rows, go to the lower index on both sides and need no exemption).
NEAR_TIE = 1e-9          # k-th vs (k+1)-th oracle logit gap exempt from index parity
# The router's fp32 tensor-core logits: each within 2^-20 ||x_t|| max_e ||W_r[e]||
# of the exact value (its refinement margin is 2^-17 of the same scale, so
# every unrefined gap is decided right with a factor 4 to spare).
LOGIT_REL = 2.0 ** -20


def check_router_logits(gpu_logits, routing, x_bits, W_r, what=""):
    """Max |fp32 logit - exact logit| / (||x_t|| max_e ||W_r[e]||) <= LOGIT_REL;
    returns that maximum."""
    x = O.bf16_to_f64(x_bits)
    scale = np.sqrt((x * x).sum(axis=1)) * np.sqrt((W_r.astype(np.float64) ** 2).sum(axis=1)).max()
    fin = np.isfinite(routing.s)
    err = np.where(fin, np.abs(gpu_logits.astype(np.float64) - np.where(fin, routing.s, 0.0)), 0.0)
    rel = (err / np.maximum(scale, 1e-300)[:, None]).max()
    print(f"[router] {what}: fp32 logits max|err| {err.max():.3e}, "
          f"{rel:.3e} x ||x|| max||W_r[e]|| (bound {LOGIT_REL:.3e})")
    assert rel <= LOGIT_REL, (what, rel)
    return rel


def torch_mod():
    import torch
    return torch


def run_forward(inp, T=None, layer=None):
    """Run moe_forward on cuda:0; returns (out uint16 numpy, layer)."""
    torch = torch_mod()
    from sparse_moe_layer_05_b200.binding import MoELayer
    T = inp.T if T is None else T
    if layer is None:
        layer = MoELayer(inp, T_max=max(T, 1))
    x = torch.from_numpy(np.ascontiguousarray(inp.x[:T])).cuda()
    out = layer.forward(x)
    torch.cuda.synchronize()
    return out.cpu().numpy(), layer


def bf16_to_f64(u16):
    return O.bf16_to_f64(u16)


# Inside every 8-element chunk the GEMM operand rows (xp, h) store element
# CHUNK_ORDER[p] at position p.
CHUNK_ORDER = np.array([0, 4, 1, 5, 2, 6, 3, 7])


def unpermute_chunks(a):
    """Natural column order of a [rows, n] array stored in chunk order."""
    a = np.asarray(a)
    n = a.shape[-1]
    out = np.empty_like(a)
    out.reshape(*a.shape[:-1], n // 8, 8)[..., CHUNK_ORDER] = a.reshape(*a.shape[:-1], n // 8, 8)
    return out


def rel_rms_err(got, want):
    rms = float(np.sqrt(np.mean(want ** 2)))
    err = float(np.max(np.abs(got - want))) if want.size else 0.0
    return err / rms if rms > 0 else err, rms, err


def assert_out_close(got_u16, want, tol=TOL_REL_RMS, what="out"):
    """Element-wise |got - want| <= tol * RMS(want) + 2^-8 |want|.

    The second term is the rounding of the bf16 output format itself: the
    exact result rounded to bf16 is off by up to 2^-8 |want|, which for
    heavy-tailed outputs exceeds 2e-2 * RMS on its own."""
    got = bf16_to_f64(got_u16)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    r, rms, err = rel_rms_err(got, want)
    bound = tol * rms + BF16_REL * np.abs(want)
    excess = np.abs(got - want) / bound
    assert np.all(excess <= 1.0), (
        f"{what}: worst element uses {excess.max():.3f} of the bound "
        f"(max|err| {err:.3e} = {r:.3e} x RMS {rms:.3e})")
    return r


def f32_to_bf16_rne(a):
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs): the
    one rounding the layer's last step applies."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def slot_sum_f32(yw_rows):
    """[n, k, d] float32 per-slot weighted expert rows -> their fp32 sum taken
    as the combine takes it: from 0, slot j = 0, 1, ..., k-1, one IEEE add each."""
    acc = np.zeros((yw_rows.shape[0], yw_rows.shape[2]), dtype=np.float32)
    for j in range(yw_rows.shape[1]):
        acc = (acc + yw_rows[:, j]).astype(np.float32)
    return acc


def h_rounding_bound(inp, routing, hidden):
    """Per output element, how far storing H in bf16 can move the layer's fp32
    result: each H value is rounded once to 8 significant bits (unit roundoff
    2^-8), so |delta out[t, m]| <= 2^-8 sum_j p_j sum_n |Wd[e_j][m, n]| |H_j[n]|.
    (The block-scaled tiles split that bf16 H exactly, up to 2^-21 of a group's
    max for its tiniest elements, covered by the 1% margin.)"""
    T = routing.idx.shape[0]
    acc = np.zeros((T, inp.d))
    for e, (_, h) in hidden.items():
        rows, slots = np.nonzero(routing.idx == e)
        wd = np.abs(O.mxfp4_decode(inp.Wd_codes[e], inp.Wd_scales[e]))
        acc[rows] += routing.p[rows, slots][:, None] * (np.abs(h) @ wd.T)
    return 1.01 * 2.0 ** -8 * acc


def check_pre_rounding(out_u16, yw_rows, want, tol=TOL_REL_RMS, what="out", h_bound=None):
    """The stated bound with nothing added for the output format: the layer's
    fp32 result before its one rounding to bf16 (the sum of the per-slot rows
    the down GEMM wrote to the workspace) must lie within tol * RMS(oracle) of
    the fp64 oracle element by element, and the bf16 output must be exactly
    that sum rounded to nearest even. Returns max|err| / RMS of the fp32 sum.

    ``h_bound`` (a callable giving h_rounding_bound's array), for synthetic
    shapes whose outputs are heavy-tailed: if the plain bound fails, each
    element may also carry what H's bf16 storage can move it, and nothing
    more. The pages' shapes (d = I = 2880) are checked without it."""
    s = slot_sum_f32(np.asarray(yw_rows, dtype=np.float32))
    assert np.array_equal(np.asarray(out_u16), f32_to_bf16_rne(s)), \
        f"{what}: bf16 output is not the rounded fp32 sum"
    r, rms, err = rel_rms_err(s.astype(np.float64), want)
    if r <= tol:
        return r
    assert h_bound is not None, \
        f"{what}: pre-rounding max|err| {err:.3e} = {r:.3e} x RMS {rms:.3e} > {tol}"
    bound = tol * rms + h_bound()
    excess = np.abs(s.astype(np.float64) - want) / bound
    assert np.all(excess <= 1.0), (
        f"{what}: pre-rounding error beyond 2e-2 x RMS plus H's bf16 rounding "
        f"(worst element {excess.max():.3f} of the bound; max|err| = {r:.3e} x RMS)")
    print(f"[parity] {what}: fp32 result {r:.3e} x RMS, within 2e-2 x RMS plus the bound of "
          f"H's bf16 rounding (worst element {excess.max():.3f} of it)")
    return r


def compare_routing(gpu_idx, gpu_w, routing, copies_of=None, max_exempt=None):
    """Index parity except near-ties; weights within 1e-5 absolute.

    With ``copies_of`` (silent-init layers) the order inside a group of equal
    copies is a pure tie, so each token's index set and the weight per index
    are compared instead of the ordered list. An exempt token (k-th and
    (k+1)-th oracle logits within NEAR_TIE) must still hold a valid choice: k
    distinct experts, none of them below the oracle's k-th logit by more than
    NEAR_TIE. Returns the number of exempt tokens.
    """
    idx_o, p_o = routing.idx, routing.p
    tie = routing.near_tie(NEAR_TIE)
    T, k = idx_o.shape
    # ties inside the selected list (adjacent logits within NEAR_TIE) make the
    # order ambiguous but not the set
    srt = -np.sort(-routing.s, axis=1)[:, :k]
    inner_tie = np.any(np.abs(np.diff(srt, axis=1)) < NEAR_TIE, axis=1) if k > 1 else np.zeros(T, bool)
    exempt = 0
    for t in range(T):
        if tie[t]:
            exempt += 1
            sel = gpu_idx[t].astype(np.int64)
            assert len(set(sel.tolist())) == k, (t, sel)
            assert np.all(routing.s[t, sel] >= srt[t, k - 1] - NEAR_TIE), (t, sel)
            continue
        if copies_of is not None or inner_tie[t]:
            assert set(gpu_idx[t].tolist()) == set(idx_o[t].tolist()), t
            wo = dict(zip(idx_o[t].tolist(), p_o[t].tolist()))
            for e, w in zip(gpu_idx[t].tolist(), gpu_w[t].tolist()):
                assert abs(w - wo[e]) < 1e-5, (t, e, w, wo[e])
        else:
            assert np.array_equal(gpu_idx[t], idx_o[t]), (t, gpu_idx[t], idx_o[t])
            assert np.max(np.abs(gpu_w[t] - p_o[t])) < 1e-5, t
    limit = max(2, T // 50) if max_exempt is None else max_exempt
    assert exempt <= limit, f"too many near-ties: {exempt}"
    return exempt


def check_tables_against_oracle(gpu_idx, counts, offsets, perm, routing, E):
    """counts, offsets and perm bit-exact: against the oracle's own tables when
    the GPU chose exactly the oracle's experts, else (near-ties) against the
    tables of the GPU's choice, which compare_routing has validated."""
    same = np.array_equal(gpu_idx, routing.idx)
    c, o, p, _ = O.routing_tables(routing.idx if same else gpu_idx, E)
    assert np.array_equal(counts, c) and np.array_equal(offsets, o) and np.array_equal(perm, p)
    return same


# ---------------------------------------- block-scaled workspace readouts ----
# The block-scaled tiles keep their activation operands in a padded token
# layout: expert e's routed rows start at a multiple of the tile's token count
# NT, so a token tile is NT consecutive rows. Their E8M0 scales sit in blocks
# of [token tile][k-block][512-byte tcgen05.cp atoms]; byte
# (w // 4) * 512 + (c % 32) * 16 + (w % 4) * 4 + kk holds the scale of B column
# c (w = c // 32) for K step kk of the k-block.

def mx_tile_tokens(P, E, act, pair=False):
    """Token-row granule of the block-scaled kernels' padded layout: 16 when
    experts average under 64 rows, else 128 on a CTA pair or for the quantised
    modes, 120 for the one-CTA bf16-split tiles."""
    if P < 64 * E:
        return 16
    return 128 if (pair or act != "bf16") else 120


def mx_padded_rows(offsets, NT):
    """Padded-layout row of every permuted position."""
    E = len(offsets) - 1
    pr = np.empty(int(offsets[-1]), dtype=np.int64)
    tb = 0
    for e in range(E):
        n = int(offsets[e + 1] - offsets[e])
        pr[offsets[e]:offsets[e + 1]] = tb * NT + np.arange(n)
        tb += (n + NT - 1) // NT
    return pr


def mx_scale_bytes(sfb, pr, K, NT, terms=1, kb256=False):
    """E8M0 scale bytes [len(pr)][K/32] of the rows at padded positions pr.
    kb256: the kind::mxf4 kernel's blocks, 1024 bytes per 256-wide k-block,
    group byte b (0..7) of a block in atom b // 4."""
    G = K // 32
    n = pr % NT
    w = n // 32
    atom = (w // 4) * 512 + (n % 32) * 16 + (w % 4) * 4
    out = np.empty((len(pr), G), dtype=np.uint8)
    if kb256:
        KB = (K + 255) // 256
        for g in range(G):
            if G % 8 == 0 or g < 8 * (KB - 1):
                kb, b = g // 8, g % 8
            else:
                kb, b = KB - 1, g - (G - 8)
            out[:, g] = sfb[(pr // NT * KB + kb) * 1024 + (b // 4) * 512 + atom + b % 4]
        return out
    KB = (K + 127) // 128
    blk = 512 * ((terms * NT + 127) // 128)
    for g in range(G):
        if G % 4 == 0 or g < 4 * (KB - 1):
            kb, kk = g // 4, g % 4
        else:
            kb, kk = KB - 1, g - (G - 4)
        out[:, g] = sfb[(pr // NT * KB + kb) * blk + atom + kk]
    return out


def e4m3_to_f64(b):
    """OCP E4M3 bytes to float64 (S.1111.111 is NaN; no infinities)."""
    b = np.asarray(b).astype(np.int64)
    e, m = (b >> 3) & 15, b & 7
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * np.exp2(e - 7.0))
    v = np.where((b & 0x7F) == 0x7F, np.nan, v)
    return np.where(b >> 7, -v, v)


def mx_dequant(q, scales, act):
    """Converted rows back to float64: q [n][K] E4M3 bytes or [n][K/2] packed
    E2M1 codes (element 2i in the low nibble of byte i), scales [n][K/32]."""
    q = np.asarray(q)
    if act == "e4m3":
        v = e4m3_to_f64(q)
    else:
        v = np.stack([O.e2m1_value(q & 0x0F), O.e2m1_value(q >> 4)], axis=-1).reshape(
            q.shape[0], -1)
    s = np.exp2(np.asarray(scales, dtype=np.float64) - 127.0)
    return v * np.repeat(s, 32, axis=1)
