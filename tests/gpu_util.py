"""Helpers shared by the GPU parity tests: upload a workload, run the CUDA path
through the C ABI, and compare with the oracle."""
import numpy as np

from oracle import moe_oracle as O

TOL_REL_RMS = 2e-2       # |err| <= 2e-2 * RMS(oracle out) ...
BF16_REL = 2.0 ** -8     # ... + the bf16 output's own rounding, 2^-8 |oracle value|
NEAR_TIE = 1e-5          # k-th vs (k+1)-th oracle logit gap exempt from index parity


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


def compare_routing(gpu_idx, gpu_w, routing, copies_of=None):
    """Index parity except near-ties; weights within 1e-5 absolute.

    With ``copies_of`` (silent-init layers) the order inside a group of equal
    copies is a pure tie, so each token's index set and the weight per index
    are compared instead of the ordered list.
    Returns the number of exempt tokens.
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
            continue
        if copies_of is not None or inner_tie[t]:
            assert set(gpu_idx[t].tolist()) == set(idx_o[t].tolist()), t
            wo = dict(zip(idx_o[t].tolist(), p_o[t].tolist()))
            for e, w in zip(gpu_idx[t].tolist(), gpu_w[t].tolist()):
                assert abs(w - wo[e]) < 1e-5, (t, e, w, wo[e])
        else:
            assert np.array_equal(gpu_idx[t], idx_o[t]), (t, gpu_idx[t], idx_o[t])
            assert np.max(np.abs(gpu_w[t] - p_o[t])) < 1e-5, t
    assert exempt <= max(2, T // 50), f"too many near-ties: {exempt}"
    return exempt
