"""moe_route_noalloc: the router + permutation entry point for callers that
cannot allocate device memory (they get only inputs, outputs and a stream, so
they cannot hand the library a workspace). It must give the same results as
moe_route, which uses a caller-provided workspace, call after call, while its
scratch lives in the library's own fixed device array.

This file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import numpy as np
import pytest

from sparse_moe_layer_05_b200 import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_moe_layer_05_b200 import build
    build.build()


def _outputs(E, k, T):
    dev = "cuda"
    return (torch.empty((T, k), dtype=torch.int32, device=dev),
            torch.empty((T, k), dtype=torch.float32, device=dev),
            torch.empty(E, dtype=torch.int32, device=dev),
            torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(T * k, dtype=torch.int32, device=dev))


def _tables(idx, E):
    """counts, offsets and the stable permutation of a top-k choice (integer
    bookkeeping, written out here so this file needs no oracle for it)."""
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    return counts, offsets, perm, None


def _route_with_workspace(inp, x, W_r, b_r):
    from sparse_moe_layer_05_b200 import binding as B
    E, k, T, d = inp.E, inp.k, inp.T, inp.d
    outs = _outputs(E, k, T)
    ws = torch.empty(B.moe_route_workspace_size(E, k, T, d), dtype=torch.uint8, device="cuda")
    B.moe_route(x, W_r, b_r, E, k, T, d, *outs, workspace=ws)
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in outs]


def _route_noalloc(inp, x, W_r, b_r):
    from sparse_moe_layer_05_b200 import binding as B
    E, k, T, d = inp.E, inp.k, inp.T, inp.d
    outs = _outputs(E, k, T)
    B.moe_route_noalloc(x, W_r, b_r, E, k, T, d, *outs)
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in outs]


def test_noalloc_route_matches_workspace_route_on_consecutive_calls():
    # two calls in a row with different shapes: the second must not see the
    # first call's leftovers in the shared scratch array
    # (the last two take the two permutation paths: several 256-token chunks,
    # and one fused launch for at most 256 tokens)
    cases = [W.make_inputs("248a20", T=4096),      # T * E = 1,015,808, near the limit
             W.make_custom(256, 128, 32, 4, 700, seed=41),
             W.make_custom(2880, 128, 128, 4, 200, seed=42)]
    for inp in cases:
        x = torch.from_numpy(inp.x).cuda()
        W_r = torch.from_numpy(inp.W_r).cuda()
        b_r = torch.from_numpy(inp.b_r).cuda()
        want = _route_with_workspace(inp, x, W_r, b_r)
        got = _route_noalloc(inp, x, W_r, b_r)
        idx, w, counts, offsets, perm = got
        # the same launches on the same inputs: bit-identical outputs
        for g, r in zip(got, want):
            assert np.array_equal(g, r)
        c, o, p, _ = _tables(idx, inp.E)
        assert np.array_equal(counts, c) and np.array_equal(offsets, o)
        assert np.array_equal(perm, p)


def test_noalloc_route_rejects_oversized_calls():
    from sparse_moe_layer_05_b200 import binding as B
    E, k, T, d = 128, 4, 8193, 64                      # T * E = 1,048,704 > 1,048,576
    x = torch.zeros((T, d), dtype=torch.uint16, device="cuda")
    W_r = torch.zeros((E, d), dtype=torch.float32, device="cuda")
    b_r = torch.zeros(E, dtype=torch.float32, device="cuda")
    with pytest.raises(B.MoEError) as ei:
        B.moe_route_noalloc(x, W_r, b_r, E, k, T, d, *_outputs(E, k, T))
    assert ei.value.code == 2                          # MOE_ERR_UNSUPPORTED
