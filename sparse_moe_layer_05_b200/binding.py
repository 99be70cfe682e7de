"""ctypes binding of ``libmoe_b200.so`` (the C ABI in ``include/moe_b200.h``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. Tensors are torch CUDA tensors (torch provides device memory and
streams); functions keep the C names. There is no CPU fallback: if the
library or a CUDA device is missing, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_b200.so")

STATUS = {
    0: "MOE_OK",
    1: "MOE_ERR_INVALID_ARG",
    2: "MOE_ERR_UNSUPPORTED",
    3: "MOE_ERR_WORKSPACE",
    4: "MOE_ERR_CUDA",
    5: "MOE_ERR_TIMEOUT",
    6: "MOE_ERR_NO_DEVICE",
}

EXPORTS = [
    "moe_status_string", "moe_version", "moe_workspace_size", "moe_forward",
    "moe_workspace_size_hostio", "moe_forward_hostio", "moe_route_workspace_size",
    "moe_route", "moe_workspace_layout", "moe_mxfp4_to_bf16", "moe_mx_split_e4m3", "moe_sync_status",
    "moe_selftest_wait_timeout", "moe_forward_launch_count", "moe_forward_timed",
    "moe_set_tile_policy", "moe_route_noalloc",
    "moe_workspace_size_block", "moe_forward_block", "moe_rms_norm", "moe_forward_biased",
    "moe_forward_timed_events", "moe_forward_ex", "moe_mx_quantize", "moe_forward_timed_ex",
]
# the measurement library (libmoe_b200_probe.so, include/moe_b200_probe.h)
PROBE_EXPORTS = ["moe_probe_tensor_rate", "moe_probe_error_string", "moe_probe_error_site"]
PROBE_LIB_PATH = os.path.join(PKG, "libmoe_b200_probe.so")

# moe_forward_opts.act_quant
ACT_BF16, ACT_MXFP8, ACT_MXFP4 = 0, 1, 2
ACT_MODES = {"bf16": ACT_BF16, "mxfp8": ACT_MXFP8, "mxfp4": ACT_MXFP4}

STAGES = ["router_logits", "topk_softmax", "perm_hist", "perm_scan", "perm_scatter",
          "gather_rows", "transpose_scales_gu", "transpose_scales_d", "gemm_gateup_swiglu",
          "gemm_down_combine", "combine"]


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


class ForwardOpts(ctypes.Structure):
    """moe_forward_opts (include/moe_b200.h)."""
    _fields_ = [("tile_policy", ctypes.c_int), ("act_quant", ctypes.c_int),
                ("gu_bias_dev", ctypes.c_void_p), ("down_bias_dev", ctypes.c_void_p)]


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("logits", "topk_idx", "topk_w", "counts", "offsets", "perm", "xp", "h", "yw",
                 "status", "total", "x_scales", "h_scales")]


_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load the library (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m sparse_moe_layer_05_b200.build`")
    lib = ctypes.CDLL(p)
    vp, sz, i32, u8p, fp = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int,
                            ctypes.c_void_p, ctypes.c_void_p)
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_status_string.argtypes = [i32]
    lib.moe_version.restype = i32
    lib.moe_workspace_size.restype = sz
    lib.moe_workspace_size.argtypes = [i32] * 5
    lib.moe_workspace_size_hostio.restype = sz
    lib.moe_workspace_size_hostio.argtypes = [i32] * 5
    lib.moe_route_workspace_size.restype = sz
    lib.moe_route_workspace_size.argtypes = [i32] * 4
    fwd = [vp, fp, fp, u8p, u8p, u8p, u8p, i32, i32, i32, i32, i32, vp, vp, sz, vp]
    lib.moe_forward.restype = i32
    lib.moe_forward.argtypes = fwd
    lib.moe_forward_hostio.restype = i32
    lib.moe_forward_hostio.argtypes = fwd
    lib.moe_forward_timed.restype = i32
    lib.moe_forward_timed.argtypes = fwd + [ctypes.POINTER(ctypes.c_float)]
    lib.moe_forward_timed_events.restype = i32
    lib.moe_forward_timed_events.argtypes = fwd + [ctypes.c_uint, ctypes.POINTER(ctypes.c_float)]
    lib.moe_route.restype = i32
    lib.moe_route.argtypes = [vp, fp, fp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_route_noalloc.restype = i32
    lib.moe_route_noalloc.argtypes = [vp, fp, fp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.moe_workspace_layout.restype = i32
    lib.moe_workspace_layout.argtypes = [i32] * 5 + [ctypes.POINTER(WsLayout)]
    lib.moe_mxfp4_to_bf16.restype = i32
    lib.moe_mxfp4_to_bf16.argtypes = [u8p, u8p, i32, i32, vp, vp]
    lib.moe_workspace_size_block.restype = sz
    lib.moe_workspace_size_block.argtypes = [i32] * 5
    lib.moe_forward_block.restype = i32
    # the biased forms: gate/up bias after the gate/up weights, down bias after the down ones
    fwd_b = fwd[:5] + [fp] + fwd[5:7] + [fp] + fwd[7:]
    lib.moe_forward_biased.restype = i32
    lib.moe_forward_biased.argtypes = fwd_b
    lib.moe_forward_block.argtypes = [vp, fp, ctypes.c_float] + fwd_b[1:]
    lib.moe_rms_norm.restype = i32
    lib.moe_rms_norm.argtypes = [vp, fp, ctypes.c_float, i32, i32, vp, vp]
    lib.moe_forward_ex.restype = i32
    lib.moe_forward_ex.argtypes = fwd[:15] + [ctypes.POINTER(ForwardOpts), vp]
    lib.moe_forward_timed_ex.restype = i32
    lib.moe_forward_timed_ex.argtypes = fwd[:15] + [ctypes.POINTER(ForwardOpts), vp, ctypes.c_uint,
                                                    ctypes.POINTER(ctypes.c_float)]
    lib.moe_mx_quantize.restype = i32
    lib.moe_mx_quantize.argtypes = [vp, i32, i32, i32, u8p, u8p, vp]
    lib.moe_mx_split_e4m3.restype = i32
    lib.moe_mx_split_e4m3.argtypes = [vp, i32, i32, u8p, u8p, u8p, vp]
    lib.moe_sync_status.restype = i32
    lib.moe_sync_status.argtypes = [vp, sz, vp]
    lib.moe_selftest_wait_timeout.restype = i32
    lib.moe_selftest_wait_timeout.argtypes = [vp, vp]
    lib.moe_set_tile_policy.restype = i32
    lib.moe_set_tile_policy.argtypes = [i32]
    lib.moe_forward_launch_count.restype = i32
    lib.moe_forward_launch_count.argtypes = [i32] * 5
    _lib = lib
    return lib


_probe_lib = None


def load_probe(path: Optional[str] = None) -> ctypes.CDLL:
    """Load the tensor-core rate probe library (measurement tooling)."""
    global _probe_lib
    if _probe_lib is not None:
        return _probe_lib
    p = path or PROBE_LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m sparse_moe_layer_05_b200.build`")
    lib = ctypes.CDLL(p)
    lib.moe_probe_tensor_rate.restype = ctypes.c_int
    lib.moe_probe_tensor_rate.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.POINTER(ctypes.c_double), ctypes.c_void_p]
    lib.moe_probe_error_string.restype = ctypes.c_char_p
    lib.moe_probe_error_site.restype = ctypes.c_char_p
    _probe_lib = lib
    return lib


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise MoEError(fn, code)


def _ptr(t) -> int:
    if t is None:
        return 0
    return int(t.data_ptr())


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _require_cuda(*ts) -> None:
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("expected CUDA tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("expected contiguous tensors")


# ---------------------------------------------------------------- sizes ----

def moe_workspace_size(E: int, k: int, T: int, d: int, I: int) -> int:
    return int(load().moe_workspace_size(E, k, T, d, I))


def moe_workspace_size_hostio(E: int, k: int, T: int, d: int, I: int) -> int:
    return int(load().moe_workspace_size_hostio(E, k, T, d, I))


def moe_route_workspace_size(E: int, k: int, T: int, d: int) -> int:
    return int(load().moe_route_workspace_size(E, k, T, d))


def moe_workspace_layout(E: int, k: int, T: int, d: int, I: int) -> dict:
    L = WsLayout()
    _check("moe_workspace_layout", load().moe_workspace_layout(E, k, T, d, I, ctypes.byref(L)))
    return {n: getattr(L, n) for n, _ in WsLayout._fields_}


def moe_forward_launch_count(E: int, k: int, T: int, d: int, I: int) -> int:
    return int(load().moe_forward_launch_count(E, k, T, d, I))


# ---------------------------------------------------------------- calls ----

def moe_forward(x, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, E, k, T, d, I,
                out, workspace, stream=None) -> None:
    """Enqueue the forward pass (see include/moe_b200.h). x/out: uint16 or bf16 [T, d]."""
    _require_cuda(x, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, out, workspace)
    _check("moe_forward", load().moe_forward(
        _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(Wgu_codes), _ptr(Wgu_scales), _ptr(Wd_codes),
        _ptr(Wd_scales), E, k, T, d, I, _ptr(out), _ptr(workspace), workspace.numel(),
        _stream(stream)))


def moe_forward_biased(x, W_r, b_r, Wgu_codes, Wgu_scales, gu_bias, Wd_codes, Wd_scales, down_bias,
                       E, k, T, d, I, out, workspace, stream=None) -> None:
    """moe_forward with per-expert biases: gu_bias f32 [E, 2I] (gate then up),
    down_bias f32 [E, d]; either may be None."""
    _require_cuda(x, W_r, b_r, Wgu_codes, Wgu_scales, gu_bias, Wd_codes, Wd_scales, down_bias, out,
                  workspace)
    _check("moe_forward_biased", load().moe_forward_biased(
        _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(Wgu_codes), _ptr(Wgu_scales), _ptr(gu_bias),
        _ptr(Wd_codes), _ptr(Wd_scales), _ptr(down_bias), E, k, T, d, I, _ptr(out),
        _ptr(workspace), workspace.numel(), _stream(stream)))


def moe_forward_ex(x, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, E, k, T, d, I,
                   out, workspace, tile_policy: int = 0, act_quant=ACT_BF16, gu_bias=None,
                   down_bias=None, stream=None) -> None:
    """moe_forward with per-call options: tile_policy (-1 process default, 0 by
    shape, 1..4 forced), act_quant (ACT_BF16, ACT_MXFP8, ACT_MXFP4 or their
    names), optional expert biases."""
    _require_cuda(x, W_r, b_r, Wgu_codes, Wgu_scales, gu_bias, Wd_codes, Wd_scales, down_bias, out,
                  workspace)
    if isinstance(act_quant, str):
        act_quant = ACT_MODES[act_quant]
    o = ForwardOpts(tile_policy, act_quant, _ptr(gu_bias) or None, _ptr(down_bias) or None)
    _check("moe_forward_ex", load().moe_forward_ex(
        _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(Wgu_codes), _ptr(Wgu_scales), _ptr(Wd_codes),
        _ptr(Wd_scales), E, k, T, d, I, _ptr(out), _ptr(workspace), workspace.numel(),
        ctypes.byref(o), _stream(stream)))


def moe_forward_timed(x, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, E, k, T, d, I,
                      out, workspace, stream=None) -> list:
    """Forward pass with per-launch CUDA-event timing; returns len(STAGES)+1
    floats (ms): one per launch in the order of STAGES, then the whole span.
    Blocks."""
    _require_cuda(x, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, out, workspace)
    ms = (ctypes.c_float * (len(STAGES) + 1))()
    _check("moe_forward_timed", load().moe_forward_timed(
        _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(Wgu_codes), _ptr(Wgu_scales), _ptr(Wd_codes),
        _ptr(Wd_scales), E, k, T, d, I, _ptr(out), _ptr(workspace), workspace.numel(),
        _stream(stream), ms))
    return list(ms)


def moe_forward_timed_events(x, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, E, k, T, d,
                             I, out, workspace, event_mask: int, stream=None) -> list:
    """moe_forward_timed recording only the boundaries in event_mask (bit i:
    before launch i, bit len(STAGES): after the last); entries of unrecorded
    boundaries are 0, each recorded one spans to the next recorded. Blocks."""
    _require_cuda(x, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, out, workspace)
    ms = (ctypes.c_float * (len(STAGES) + 1))()
    _check("moe_forward_timed_events", load().moe_forward_timed_events(
        _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(Wgu_codes), _ptr(Wgu_scales), _ptr(Wd_codes),
        _ptr(Wd_scales), E, k, T, d, I, _ptr(out), _ptr(workspace), workspace.numel(),
        _stream(stream), event_mask, ms))
    return list(ms)


def moe_forward_hostio(x_host, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, E, k, T, d,
                       I, out_host, workspace, stream=None) -> None:
    """Forward pass with x and out in host memory (pinned for async copies); synchronises."""
    _require_cuda(W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales, workspace)
    if x_host.is_cuda or out_host.is_cuda:
        raise ValueError("x_host and out_host must be host tensors")
    _check("moe_forward_hostio", load().moe_forward_hostio(
        _ptr(x_host), _ptr(W_r), _ptr(b_r), _ptr(Wgu_codes), _ptr(Wgu_scales), _ptr(Wd_codes),
        _ptr(Wd_scales), E, k, T, d, I, _ptr(out_host), _ptr(workspace), workspace.numel(),
        _stream(stream)))


def moe_route(x, W_r, b_r, E, k, T, d, topk_idx, topk_w, counts=None, offsets=None, perm=None,
              workspace=None, stream=None) -> None:
    _require_cuda(x, W_r, b_r, topk_idx, topk_w, counts, offsets, perm, workspace)
    _check("moe_route", load().moe_route(
        _ptr(x), _ptr(W_r), _ptr(b_r), E, k, T, d, _ptr(topk_idx), _ptr(topk_w), _ptr(counts),
        _ptr(offsets), _ptr(perm), _ptr(workspace), workspace.numel(), _stream(stream)))


def moe_route_noalloc(x, W_r, b_r, E, k, T, d, topk_idx, topk_w, counts, offsets, perm,
                      stream=None) -> None:
    """moe_route with the library's own fixed device scratch (no workspace):
    for callers that cannot allocate; T * E <= 1,048,576."""
    _require_cuda(x, W_r, b_r, topk_idx, topk_w, counts, offsets, perm)
    _check("moe_route_noalloc", load().moe_route_noalloc(
        _ptr(x), _ptr(W_r), _ptr(b_r), E, k, T, d, _ptr(topk_idx), _ptr(topk_w), _ptr(counts),
        _ptr(offsets), _ptr(perm), _stream(stream)))


def moe_workspace_size_block(E: int, k: int, T: int, d: int, I: int) -> int:
    return int(load().moe_workspace_size_block(E, k, T, d, I))


def moe_rms_norm(h, g, eps: float, T: int, d: int, x, stream=None) -> None:
    _require_cuda(h, g, x)
    _check("moe_rms_norm", load().moe_rms_norm(_ptr(h), _ptr(g), eps, T, d, _ptr(x), _stream(stream)))


def moe_forward_block(h, g, eps: float, W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales,
                      E: int, k: int, T: int, d: int, I: int, out, workspace, stream=None,
                      gu_bias=None, down_bias=None) -> None:
    """out = h + MoE(RMSNorm(h)) (bf16 rows; g f32 gain; optional expert biases)."""
    _require_cuda(h, g, W_r, b_r, Wgu_codes, Wgu_scales, gu_bias, Wd_codes, Wd_scales, down_bias,
                  out, workspace)
    _check("moe_forward_block", load().moe_forward_block(
        _ptr(h), _ptr(g), eps, _ptr(W_r), _ptr(b_r), _ptr(Wgu_codes), _ptr(Wgu_scales),
        _ptr(gu_bias), _ptr(Wd_codes), _ptr(Wd_scales), _ptr(down_bias), E, k, T, d, I,
        _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)))


def moe_probe_tensor_rate(kind: int, N: int, per_commit: int, stream=None) -> float:
    """MACs per SM clock of back-to-back UMMAs (kind 0 bf16, 1 block-scaled
    E2M1 x E4M3, 2 block-scaled E2M1 x E2M1), from the probe library."""
    out = ctypes.c_double(0.0)
    lib = load_probe()
    code = lib.moe_probe_tensor_rate(kind, N, per_commit, ctypes.byref(out), _stream(stream))
    if code == 4:        # MOE_ERR_CUDA: say which call failed and how
        raise MoEError(f"moe_probe_tensor_rate ({lib.moe_probe_error_site().decode()}: "
                       f"{lib.moe_probe_error_string().decode()})", code)
    _check("moe_probe_tensor_rate", code)
    return out.value


def moe_mx_quantize(x, rows: int, K: int, act_quant, q, scales, stream=None) -> None:
    """The quantised modes' activation conversion on plain bf16 rows: q [rows, K]
    E4M3 (ACT_MXFP8) or [rows, K/2] packed E2M1 (ACT_MXFP4), scales [rows, K/32]."""
    _require_cuda(x, q, scales)
    if isinstance(act_quant, str):
        act_quant = ACT_MODES[act_quant]
    _check("moe_mx_quantize", load().moe_mx_quantize(
        _ptr(x), rows, K, act_quant, _ptr(q), _ptr(scales), _stream(stream)))


def moe_mx_split_e4m3(x, rows: int, K: int, hi, lo, scales, stream=None) -> None:
    _require_cuda(x, hi, lo, scales)
    _check("moe_mx_split_e4m3", load().moe_mx_split_e4m3(
        _ptr(x), rows, K, _ptr(hi), _ptr(lo), _ptr(scales), _stream(stream)))


def moe_mxfp4_to_bf16(codes, scales, rows: int, K: int, out, stream=None) -> None:
    _require_cuda(codes, scales, out)
    _check("moe_mxfp4_to_bf16", load().moe_mxfp4_to_bf16(
        _ptr(codes), _ptr(scales), rows, K, _ptr(out), _stream(stream)))


TILE_AUTO, TILE_SINGLE, TILE_PAIR, TILE_SWAP, TILE_MX, TILE_MX_PAIR = 0, 1, 2, 3, 4, 5


def moe_set_tile_policy(policy: int) -> None:
    """0 = by shape, 1 = single-CTA, 2 = CTA-pair, 3 = swapped-operand,
    4 = block-scaled tiles, 5 = block-scaled tiles on a CTA pair: the process
    default of the calls without options (moe_forward_ex takes one per call)."""
    _check("moe_set_tile_policy", load().moe_set_tile_policy(policy))


def moe_sync_status(workspace, stream=None) -> int:
    """Synchronise, then return (and clear) the device status code."""
    return int(load().moe_sync_status(_ptr(workspace), workspace.numel(), _stream(stream)))


def moe_selftest_wait_timeout(workspace, stream=None) -> None:
    _check("moe_selftest_wait_timeout",
           load().moe_selftest_wait_timeout(_ptr(workspace), _stream(stream)))


# ----------------------------------------------------------- convenience ----

class MoELayer:
    """Device-resident MoE layer: weights uploaded once, workspace owned here."""

    def __init__(self, inp, device="cuda", T_max: Optional[int] = None, hostio: bool = False):
        import torch
        self.d, self.I, self.E, self.k = inp.d, inp.I, inp.E, inp.k
        to = lambda a: torch.from_numpy(a).to(device)
        self.W_r = to(inp.W_r)
        self.b_r = to(inp.b_r)
        self.Wgu_codes = to(inp.Wgu_codes)
        self.Wgu_scales = to(inp.Wgu_scales)
        self.Wd_codes = to(inp.Wd_codes)
        self.Wd_scales = to(inp.Wd_scales)
        self.T_max = T_max if T_max is not None else inp.T
        size_fn = moe_workspace_size_hostio if hostio else moe_workspace_size
        nbytes = size_fn(self.E, self.k, self.T_max, self.d, self.I)
        if nbytes == 0:
            raise ValueError("unsupported shape")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def forward(self, x, out=None, stream=None):
        import torch
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError("more tokens than the workspace was sized for")
        if out is None:
            out = torch.empty((T, self.d), dtype=torch.uint16, device=x.device)
        moe_forward(x, self.W_r, self.b_r, self.Wgu_codes, self.Wgu_scales, self.Wd_codes,
                    self.Wd_scales, self.E, self.k, T, self.d, self.I, out, self.workspace, stream)
        return out

    def forward_timed(self, x, out, stream=None):
        T = x.shape[0]
        return moe_forward_timed(x, self.W_r, self.b_r, self.Wgu_codes, self.Wgu_scales,
                                 self.Wd_codes, self.Wd_scales, self.E, self.k, T, self.d,
                                 self.I, out, self.workspace, stream)

    def forward_timed_events(self, x, out, event_mask: int, stream=None, tile_policy=None,
                             act_quant=None):
        """moe_forward_timed_events; with tile_policy or act_quant given, the
        per-call options form (moe_forward_timed_ex)."""
        T = x.shape[0]
        if tile_policy is None and act_quant is None:
            return moe_forward_timed_events(x, self.W_r, self.b_r, self.Wgu_codes,
                                            self.Wgu_scales, self.Wd_codes, self.Wd_scales,
                                            self.E, self.k, T, self.d, self.I, out,
                                            self.workspace, event_mask, stream)
        if isinstance(act_quant, str):
            act_quant = ACT_MODES[act_quant]
        o = ForwardOpts(-1 if tile_policy is None else tile_policy,
                        ACT_BF16 if act_quant is None else act_quant, None, None)
        ms = (ctypes.c_float * (len(STAGES) + 1))()
        _check("moe_forward_timed_ex", load().moe_forward_timed_ex(
            _ptr(x), _ptr(self.W_r), _ptr(self.b_r), _ptr(self.Wgu_codes), _ptr(self.Wgu_scales),
            _ptr(self.Wd_codes), _ptr(self.Wd_scales), self.E, self.k, T, self.d, self.I, _ptr(out),
            _ptr(self.workspace), self.workspace.numel(), ctypes.byref(o), _stream(stream),
            event_mask, ms))
        return list(ms)

    def forward_hostio(self, x_host, out_host, stream=None):
        T = x_host.shape[0]
        moe_forward_hostio(x_host, self.W_r, self.b_r, self.Wgu_codes, self.Wgu_scales,
                           self.Wd_codes, self.Wd_scales, self.E, self.k, T, self.d, self.I,
                           out_host, self.workspace, stream)
        return out_host

    def layout(self, T: int) -> dict:
        return moe_workspace_layout(self.E, self.k, T, self.d, self.I)

    def intermediate(self, name: str, T: int):
        """View of an intermediate buffer inside the workspace after a forward."""
        import torch
        L = self.layout(T)
        P = T * self.k
        spec = {
            "logits": (torch.float32, (T, self.E)), "topk_idx": (torch.int32, (T, self.k)),
            "topk_w": (torch.float32, (T, self.k)), "counts": (torch.int32, (self.E,)),
            "offsets": (torch.int32, (self.E + 1,)), "perm": (torch.int32, (P,)),
            "xp": (torch.uint16, (P, self.d)), "h": (torch.uint16, (P, self.I)),
            "yw": (torch.float32, (P, self.d)),
        }[name]
        dt, shape = spec
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dt).element_size()
        raw = self.workspace[L[name]:L[name] + nbytes]
        return raw.view(dt).view(shape)
