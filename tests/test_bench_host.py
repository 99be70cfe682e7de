"""Host logic of bench.py that needs no GPU: the tile family and MMA kind a
quantised-activation forward runs (which sets the roofline's peak) and the
kernel launches a step claims."""
import os
import sys
from types import SimpleNamespace

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_moe_layer_05_b200 import binding as B  # noqa: E402

SHAPE_20B = SimpleNamespace(E=32, k=4, d=2880, I=2880)


def _args(act, policy=0):
    return SimpleNamespace(act_quant=act, tile_policy=policy)


def test_bf16_launches_are_the_library_count():
    B.moe_set_tile_policy(0)
    for T in (64, 256, 8192):
        assert bench.forward_launches(_args("bf16"), SHAPE_20B, T) == \
            B.moe_forward_launch_count(32, 4, T, 2880, 2880)
    # prefill on the CTA pair: router 3, permutation 3, gather, gate/up,
    # the down weights' atom pass, down, combine
    assert bench.forward_launches(_args("bf16"), SHAPE_20B, 8192) == 11


def test_quantised_tiles_and_kinds():
    # 20b prefill: 1,024 rows per expert -> the CTA pair by shape
    assert bench.quant_tiles(_args("mxfp8"), SHAPE_20B, 8192) == "pair"
    assert not bench.quant_runs_mxf4(_args("mxfp8"), SHAPE_20B, 8192)
    assert bench.quant_runs_mxf4(_args("mxfp4"), SHAPE_20B, 8192)
    # forced one-CTA tiles: w4a4 stays on kind::mxf8f6f4
    assert bench.quant_tiles(_args("mxfp4", 4), SHAPE_20B, 8192) == "large"
    assert not bench.quant_runs_mxf4(_args("mxfp4", 4), SHAPE_20B, 8192)
    # decode: 8 rows per expert -> 16-token tiles even when the pair is forced
    assert bench.quant_tiles(_args("mxfp4", 5), SHAPE_20B, 64) == "small"
    # between 64 and 192 rows per expert: one CTA by shape, the pair if forced
    assert bench.quant_tiles(_args("mxfp8"), SHAPE_20B, 1024) == "large"
    assert bench.quant_tiles(_args("mxfp8", 5), SHAPE_20B, 1024) == "pair"
    # kind::mxf4 needs d and I of at least 256
    small = SimpleNamespace(E=32, k=4, d=128, I=2880)
    assert not bench.quant_runs_mxf4(_args("mxfp4", 5), small, 8192)


def test_quantised_launches():
    # the down weights' atom pass runs on the pair with 8-bit activations only
    assert bench.forward_launches(_args("mxfp8"), SHAPE_20B, 8192) == 11
    assert bench.forward_launches(_args("mxfp4"), SHAPE_20B, 8192) == 10
    assert bench.forward_launches(_args("mxfp4", 4), SHAPE_20B, 8192) == 10
    # at most 256 tokens the permutation is built inside the router's top-k launch
    assert bench.forward_launches(_args("mxfp8"), SHAPE_20B, 64) == 7
