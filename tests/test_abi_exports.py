"""The C-ABI library loads and exports every function include/moe_b200.h
declares; host-side checks (sizes, argument validation) behave without a GPU.
No compute call is made here."""
import ctypes
import os
import re

import pytest

from sparse_moe_layer_05_b200 import binding as B
from sparse_moe_layer_05_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.load()


def declared_functions(header):
    src = open(os.path.join(ROOT, "include", header)).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, re.M)))


def test_every_declared_symbol_is_exported(lib):
    assert sorted(f for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")) == \
        ["moe_b200.h", "moe_b200_probe.h"]
    names = declared_functions("moe_b200.h")
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTS)
    # the measurement tool is a library of its own; the layer's library lacks it
    probe = B.load_probe()
    pnames = declared_functions("moe_b200_probe.h")
    assert set(pnames) == set(B.PROBE_EXPORTS)
    for n in pnames:
        assert hasattr(probe, n), n
        assert not hasattr(lib, n), n


def test_probe_checks_arguments_without_a_device():
    probe = B.load_probe()
    out = ctypes.c_double(0.0)
    assert probe.moe_probe_tensor_rate(3, 256, 16, ctypes.byref(out), None) == 1   # kind
    assert probe.moe_probe_tensor_rate(2, 250, 16, ctypes.byref(out), None) == 1   # N % 16
    assert probe.moe_probe_tensor_rate(0, 256, 6, ctypes.byref(out), None) == 1    # per_commit
    assert probe.moe_probe_tensor_rate(0, 256, 16, None, None) == 1                # no output


def test_forward_ex_checks_options(lib):
    """Per-call options are checked before any launch: the tile policy range, the
    activation mode, the bias alignment; NULL options mean the defaults."""
    good = 0x10000
    fwd = [good] * 7 + [4, 2, 8, 64, 128, good, good, 1 << 30]
    f = lib.moe_forward_ex
    z = fwd[:]
    z[9] = 0                                            # T = 0

    def opts(**kw):
        o = B.ForwardOpts(0, 0, None, None)
        for k_, v in kw.items():
            setattr(o, k_, v)
        return ctypes.byref(o)

    assert f(*(z + [None, None])) == 0                  # NULL options
    assert f(*(z + [opts(), None])) == 0
    assert f(*(z + [opts(tile_policy=-1), None])) == 0
    assert f(*(z + [opts(tile_policy=5), None])) == 0
    assert f(*(fwd + [opts(tile_policy=6), None])) == 1
    assert f(*(fwd + [opts(tile_policy=-2), None])) == 1
    assert f(*(fwd + [opts(act_quant=3), None])) == 1
    assert f(*(fwd + [opts(act_quant=-1), None])) == 1
    assert f(*(fwd + [opts(gu_bias_dev=good + 4), None])) == 1
    # the quantised modes need the block-scaled tiles' shapes (d = 64 is not one)
    assert f(*(fwd + [opts(act_quant=1), None])) == 2
    assert f(*(fwd + [opts(act_quant=2), None])) == 2
    q = lib.moe_mx_quantize
    assert q(good, 4, 40, 1, good, good, None) == 1     # K not a multiple of 32
    assert q(good, 4, 64, 0, good, good, None) == 1     # not a quantised mode
    assert q(good, 4, 64, 3, good, good, None) == 1
    assert q(good + 8, 4, 64, 1, good, good, None) == 1  # misaligned rows
    assert q(good, 0, 64, 2, good, good, None) == 0     # no rows: nothing to do
    a = fwd[:]
    a[14] = 16
    assert f(*(a + [opts(), None])) == 3                # workspace too small


def test_hostio_status_block_holds_a_word_per_chunk():
    """Chunked host-buffer calls (T >= 2048, four chunks on two alternating chunk
    workspaces) give every chunk its own status word inside the 16-byte status
    block at the workspace's start, so no chunk can clear another's timeout."""
    for shape in [(32, 4, 8192, 2880, 2880), (8, 2, 4099, 352, 224), (4, 2, 2048, 64, 128)]:
        E, k, T, d, I = shape
        Tc = (T + 3) // 4
        sub = B.moe_workspace_layout(E, k, Tc, d, I)
        assert sub["status"] == 0
        nxt = min(v for n, v in sub.items() if n not in ("status", "total"))
        assert nxt >= 16                                 # four 32-bit words
        assert B.moe_workspace_size_hostio(E, k, T, d, I) >= 2 * sub["total"]


def test_status_strings_and_version(lib):
    assert lib.moe_status_string(0) == b"MOE_OK"
    assert lib.moe_status_string(5) == b"MOE_ERR_TIMEOUT"
    assert lib.moe_version() == 100


def test_workspace_sizes():
    assert B.moe_workspace_size(32, 4, 8192, 2880, 2880) > 8192 * 4 * 2880 * 2 * 3
    assert B.moe_workspace_size(4, 2, 0, 64, 128) > 0
    assert B.moe_workspace_size(0, 1, 8, 64, 64) == 0        # E < 1
    assert B.moe_workspace_size(4, 5, 8, 64, 64) == 0        # k > E
    assert B.moe_workspace_size(300, 4, 8, 64, 64) == 0      # E > 256
    assert B.moe_workspace_size(64, 33, 8, 64, 64) == 0      # k > 32
    assert B.moe_workspace_size(4, 2, 8, 48, 64) == 0        # d % 32
    assert B.moe_workspace_size(4, 2, 8, 64, 40) == 0        # I % 32
    assert B.moe_workspace_size_hostio(4, 2, 8, 64, 64) > B.moe_workspace_size(4, 2, 8, 64, 64)
    # chunked host-buffer calls (T >= 2048) still fit a device-buffer call
    assert (B.moe_workspace_size_hostio(32, 4, 8192, 2880, 2880)
            >= B.moe_workspace_size(32, 4, 8192, 2880, 2880))
    L = B.moe_workspace_layout(32, 4, 100, 2880, 2880)
    offs = sorted((v, k) for k, v in L.items() if k != "total")
    assert all(v % 256 == 0 for v, _ in offs)
    assert L["status"] == 0 and L["total"] >= L["yw"] + 400 * 2880 * 2
    # the block-scaled paths (decode shapes, and prefill shapes on the CTA
    # pair) launch no scale transposes (-2); the bf16 tiles do
    # 12 launches: the router's three (weight split, logits, top-k), three
    # for the permutation (none of its own for at most 256 tokens: the top-k
    # launch builds it), the gather, two scale transposes (none on the
    # block-scaled tiles), two GEMMs, combine; the CTA-pair tiles add one
    # (the down weights' scale atoms)
    assert B.moe_forward_launch_count(32, 4, 8192, 2880, 2880) == 11
    assert B.moe_forward_launch_count(32, 4, 8192, 352, 224) == 12
    assert B.moe_forward_launch_count(32, 4, 100, 2880, 2880) == 7
    assert B.moe_forward_launch_count(32, 4, 100, 352, 2880) == 9
    assert B.moe_forward_launch_count(128, 4, 300, 2880, 2880) == 10
    assert B.moe_forward_launch_count(32, 4, 0, 2880, 2880) == 0


def test_argument_errors_before_any_launch(lib):
    vp = ctypes.c_void_p
    good = 0x10000  # 16-byte aligned fake address; never dereferenced on error paths
    args = [good] * 7 + [4, 2, 8, 64, 128, good, good, 1 << 30, None]
    f = lib.moe_forward
    a = list(args)
    a[0] = None
    assert f(*a) == 1                                   # null x
    a = list(args)
    a[3] = good + 4
    assert f(*a) == 1                                   # misaligned codes
    a = list(args)
    a[10] = 48
    assert f(*a) == 2                                   # d not a multiple of 32
    a = list(args)
    a[8] = 5
    assert f(*a) == 2                                   # k > E
    a = list(args)
    a[14] = 16
    assert f(*a) == 3                                   # workspace too small
    a = list(args)
    a[9] = 0
    assert f(*a) == 0                                   # T = 0: nothing to do
    r = lib.moe_route
    assert r(good, good, good, 4, 2, 8, 64, good, good, good, None, None, good, 1 << 20, None) == 1
    assert lib.moe_mxfp4_to_bf16(good, good, 4, 40, good, None) == 1


def test_biased_block_and_timed_entries_check_arguments(lib):
    """The entries added for expert biases, the sublayer and sparse timing reject
    bad arguments before any launch; NULL biases are allowed."""
    good = 0x10000
    fwd = [good] * 7 + [4, 2, 8, 64, 128, good, good, 1 << 30, None]
    biased = fwd[:5] + [good] + fwd[5:7] + [good] + fwd[7:]
    f = lib.moe_forward_biased
    a = list(biased)
    a[5] = good + 4
    assert f(*a) == 1                                   # misaligned gate/up bias
    a = list(biased)
    a[8] = good + 8
    assert f(*a) == 1                                   # misaligned down bias
    a = list(biased)
    a[5], a[8], a[11] = None, None, 0
    assert f(*a) == 0                                   # no biases, T = 0
    a = list(biased)
    a[10] = 5
    assert f(*a) == 2                                   # k > E
    blk = [good, good, ctypes.c_float(1e-5)] + biased[1:]
    a = list(blk)
    a[7] = good + 4
    assert lib.moe_forward_block(*a) == 1               # misaligned gate/up bias
    a = list(blk)
    a[2] = ctypes.c_float(-1.0)
    assert lib.moe_forward_block(*a) == 1               # eps < 0
    ms = (ctypes.c_float * 12)()
    t = lib.moe_forward_timed_events
    assert t(*(fwd + [1 << 12, ms])) == 1               # a boundary past the last
    assert t(*(fwd + [0x301, None])) == 1               # no output array
    a = fwd + [0x301, ms]
    a[9] = 0
    assert t(*a) == 0 and list(ms) == [0.0] * 12        # T = 0: zeros, nothing launched


@pytest.mark.parametrize("E,k,T,d,I", [(4, 2, 256, 64, 128), (32, 4, 8192, 2880, 2880),
                                       (128, 4, 32, 2880, 2880), (248, 20, 16, 2880, 2880),
                                       (8, 2, 1000, 352, 224), (1, 1, 1, 32, 32)])
def test_workspace_regions_hold_their_arrays(E, k, T, d, I):
    """Every public workspace region is 256-byte aligned and has room, up to the
    next region, for the array the header says it holds."""
    L = B.moe_workspace_layout(E, k, T, d, I)
    P = T * k
    need = {"status": 4, "logits": T * E * 4, "topk_idx": P * 4, "topk_w": P * 4,
            "counts": E * 4, "offsets": (E + 1) * 4, "perm": P * 4, "xp": P * d * 2,
            "h": P * I * 2, "yw": P * d * 4}
    order = sorted((L[n], n) for n in need)
    ends = [off for off, _ in order[1:]] + [L["total"]]
    for (off, n), end in zip(order, ends):
        assert off % 256 == 0, n
        assert end - off >= need[n], (n, end - off, need[n])
    assert B.moe_workspace_size(E, k, T, d, I) == L["total"]
    assert B.moe_workspace_size_block(E, k, T, d, I) >= L["total"] + T * d * 2
