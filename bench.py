"""Benchmark of the MoE layer forward pass (B200, sm_100a).

One step = one full forward pass of the layer (router, top-k, selected-set
softmax, permutation, gate/up GEMM + SwiGLU, down GEMM + weighted un-permute,
per-token sum) over one batch of synthetic tokens already resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 20b]
                    [--impl ours|reference]

N > 1 is launched with torch.distributed.run (one rank per GPU); every rank
runs its own batch through its own copy of the layer (weak scaling, no
collective on the data path) and rank 0 prints one JSON line. The reference
arm (--impl reference) times the CPU oracle on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sparse_moe_layer_05_b200 import workloads as W  # noqa: E402

METRIC = "MoE-layer tokens/s"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DOMINANT_STAGE = "gemm_gateup_swiglu"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = ["moe_grouped_gemm.cu", "moe_ptx.cuh", "moe_abi.cu"]


# ------------------------------------------------------------ host logic ----

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_token_order(T: int, rank: int) -> np.ndarray:
    """Rows of the workload batch that rank `rank` processes (a seeded
    permutation, so each rank has a batch of its own; rank 0 is the identity)."""
    if rank == 0:
        return np.arange(T)
    return np.random.Generator(np.random.PCG64(1000 + rank)).permutation(T)


def reduce_max(value: float, world: int) -> float:
    """Maximum of `value` over all ranks (timing plumbing, not data path)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def strip_c_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines (string and character
    literals kept intact), so that a comment edit leaves the hash unchanged."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            e = src.find("*/", i + 2)
            i = n if e < 0 else e + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).split("\n"))
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash(sources=None) -> str:
    """Hash of the code (comments stripped) of the kernel sources a recorded
    ncu figure depends on."""
    h = hashlib.sha256()
    for f in sources or KERNEL_SOURCES:
        with open(os.path.join(ROOT, "sparse_moe_layer_05_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(strip_c_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def quant_tiles(args, inp, T: int):
    """Tile family of a quantised-activation forward (w4a8, w4a4), as
    moe_forward_ex picks it: 16-token tiles under 64 rows per expert; the CTA
    pair when tile policy 5 forces it or, by shape, from 192 rows per expert;
    else 128-token tiles on one CTA."""
    P, E = T * inp.k, inp.E
    if P < 64 * E:
        return "small"
    if args.tile_policy == 5 or (args.tile_policy == 0 and P >= 192 * E):
        return "pair"
    return "large"


def quant_runs_mxf4(args, inp, T: int) -> bool:
    """w4a4 on the CTA pair runs kind::mxf4 where d and I are at least 256."""
    return (args.act_quant == "mxfp4" and quant_tiles(args, inp, T) == "pair"
            and min(inp.d, inp.I) >= 256)


def forward_launches(args, inp, T: int) -> int:
    """Kernel launches of one forward: the library's count for the bf16 path;
    for the quantised modes router (3), permutation (3; inside the router's
    top-k launch for at most 256 tokens), the converting gather, the two
    GEMMs and the combine, plus the down weights' atom pass on the CTA pair
    with 8-bit activations."""
    if args.act_quant == "bf16":
        from sparse_moe_layer_05_b200 import binding as B
        return B.moe_forward_launch_count(inp.E, inp.k, T, inp.d, inp.I)
    n = 10 - (3 if T <= 256 else 0)
    if quant_tiles(args, inp, T) == "pair" and not quant_runs_mxf4(args, inp, T):
        n += 1
    return n


def recorded_traffic(workload: str, T: int, tile_policy: int = 0, act_quant: str = "bf16"):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel source and in the same
    configuration (tile policy, activation mode); else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    ent = d.get(f"{workload}:T={T}")
    if not ent or ent.get("source_hash") != kernel_source_hash(ent.get("sources")):
        return None
    if ent.get("tile_policy", 0) != tile_policy or ent.get("act_quant", "bf16") != act_quant:
        return None
    return ent.get("bytes_per_launch")


def parse_cpulist(text: str) -> set:
    """CPU ids of a sysfs cpulist such as "0-3,8,10-11"."""
    cpus = set()
    for part in text.strip().split(","):
        if not part:
            continue
        lo, _, hi = part.partition("-")
        cpus.update(range(int(lo), int(hi or lo) + 1))
    return cpus


def gpu_local_cpus(dev_index: int):
    """The CPUs of the NUMA node the GPU hangs off (its PCI device's
    local_cpulist) that this process may run on, or None if unknown."""
    import torch
    try:
        p = torch.cuda.get_device_properties(dev_index)
        bdf = f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        with open(f"/sys/bus/pci/devices/{bdf}/local_cpulist") as f:
            cpus = parse_cpulist(f.read()) & os.sched_getaffinity(0)
    except (OSError, AttributeError, ValueError):
        return None
    return cpus or None


class NearGpuHostMemory:
    """Run the enclosed host allocations on the GPU's NUMA node, so that
    pinned buffers (placed where first touched) do not cross the socket link
    on every copy; the process's CPU affinity is restored on exit."""

    def __init__(self, dev_index: int):
        self.cpus = gpu_local_cpus(dev_index)
        self.saved = None

    def __enter__(self):
        if self.cpus:
            self.saved = os.sched_getaffinity(0)
            os.sched_setaffinity(0, self.cpus)
        return self

    def __exit__(self, *exc):
        if self.saved is not None:
            os.sched_setaffinity(0, self.saved)
        return False

    def describe(self) -> str:
        if not self.cpus:
            return "pinned (GPU's NUMA node unknown)"
        c = sorted(self.cpus)
        return f"pinned, first touched on the GPU's NUMA node ({len(c)} CPUs, {c[0]}..{c[-1]})"


def layer_flops(d, I, E, k, T) -> float:
    return 6.0 * d * I * T * k + 2.0 * d * E * T


def workload_config(inp, name: str) -> dict:
    return {
        "workload": f"{name} MoE layer forward: d={inp.d} I={inp.I} E={inp.E} k={inp.k} T={inp.T}",
        "d": inp.d, "I": inp.I, "E": inp.E, "k": inp.k, "tokens_per_gpu": inp.T,
        "weights": "MXFP4 (E2M1 codes, one E8M0 scale per 32 elements)",
        "l2": "flushed between timed steps (256 MiB write, outside the step events)",
        "parallelism": "token-parallel replicas (no collective on the data path)",
    }


# --------------------------------------------------------------- clocks ----

class ClockSampler:
    """Samples the SM clock and the active clock-event (throttle) reasons of
    one GPU every few milliseconds while the timed region runs. Read-only NVML
    queries; nothing about the GPU is changed."""

    REASONS = {  # NVML clocks-event reason bits
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40,
    }

    def __init__(self, gpu_index: int, path: str | None = None, period_s: float = 0.005):
        self.gpu_index, self.path, self.period = gpu_index, path, period_s
        self.samples = []
        self._stop = None
        self._thread = None
        self.sm_max = None

    def _sample(self, nv, h):
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        try:
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        try:
            pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        except Exception:
            pw = None
        self.samples.append((time.perf_counter(), sm, rs, pw))

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.sm_max = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._sample(nv, h)  # one sample before the region starts
        except Exception:
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self._sample(nv, h)
                except Exception:
                    break
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def _handle(self, nv):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if self.gpu_index < len(ids):
            tok = ids[self.gpu_index]
            if tok.isdigit():
                return nv.nvmlDeviceGetHandleByIndex(int(tok))
            return nv.nvmlDeviceGetHandleByUUID(tok)
        return nv.nvmlDeviceGetHandleByIndex(self.gpu_index)

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        if self.path and self.samples:
            with open(self.path, "w") as f:
                f.write("t_s,sm_mhz,reasons_mask,power_w\n")
                t0 = self.samples[0][0]
                for t, sm, rs, pw in self.samples:
                    f.write(f"{t - t0:.4f},{sm},{rs:#x},{pw}\n")

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": [], "samples": 0}
        reasons = set()
        for _, _, rs, _ in self.samples:
            for n, bit in self.REASONS.items():
                if rs & bit:
                    reasons.add(n)
        sm = [x[1] for x in self.samples]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.sm_max,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- CPU legs ----

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_tokens_per_s(inp, tokens: np.ndarray):
    from oracle import moe_oracle as O
    t0 = time.perf_counter()
    O.moe_forward(inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
                  inp.Wd_scales, k=inp.k, tokens=tokens)
    dt = time.perf_counter() - t0
    return len(tokens) / dt, dt


def routing_parity(inp, gpu_idx):
    """The GPU's top-k choice on every token of the batch against the oracle's
    (part of the oracle leg): tokens whose k-th and (k+1)-th oracle logits lie
    within 1e-5 are near-ties and are counted, the rest must match exactly."""
    from oracle import moe_oracle as O
    t0 = time.perf_counter()
    r = O.route(inp.x, inp.W_r, inp.b_r, inp.k)
    tie = r.near_tie(1e-5)
    same = np.all(gpu_idx == r.idx, axis=1)
    if inp.E >= 64 and inp.E % 32 == 0 and inp.k % 2 == 0:
        # silent-init copies tie exactly: compare index sets
        same = np.array([set(a.tolist()) == set(b.tolist()) for a, b in zip(gpu_idx, r.idx)])
    return {"tokens": int(inp.T), "near_ties": int(tie.sum()),
            "mismatched_outside_near_ties": int((~same & ~tie).sum()),
            "oracle_route_s": round(time.perf_counter() - t0, 2)}


def run_reference(args, inp, name):
    """The reference arm: the CPU oracle, as it stands, on bounded samples."""
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    per_step = args.ref_tokens
    times = []
    for s in range(args.warmup + args.steps):
        toks = (np.arange(per_step) + s * per_step) % inp.T
        _, dt = oracle_tokens_per_s(inp, toks)
        if s >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = per_step * len(times) / total
    cores = blas_threads()
    sample = (f"{per_step} tokens per step of the {inp.T}-token batch (the oracle decodes every "
              f"expert those tokens select, then runs fp64 numpy matmuls)")
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(inp, name),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------- GPU leg ----

def run_ours(args, inp, name):
    import torch
    from sparse_moe_layer_05_b200 import binding as B

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    T = inp.T
    order = rank_token_order(T, rank)
    near = NearGpuHostMemory(local)
    with near:
        x_host = torch.from_numpy(np.ascontiguousarray(inp.x[order])).pin_memory()
        out_host = torch.empty((T, inp.d), dtype=torch.uint16).pin_memory()
        out_host.zero_()
    x = x_host.to(dev)
    B.moe_set_tile_policy(args.tile_policy)
    layer = B.MoELayer(inp, device=dev, hostio=True)
    out = torch.empty((T, inp.d), dtype=torch.uint16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # launch boundaries recorded in the timed steps: the pass's start and end and
    # the two around the dominant kernel (each recorded event delays the next
    # launch by a few microseconds, so the per-stage breakdown is taken separately)
    dom = B.STAGES.index(DOMINANT_STAGE)
    nb = len(B.STAGES)
    timed_mask = (1 << 0) | (1 << dom) | (1 << (dom + 1)) | (1 << nb)
    # the per-call options (tile policy, activation mode) travel with every call
    act = None if args.act_quant == "bf16" else args.act_quant
    pol = args.tile_policy

    def timed_pass(mask):
        return layer.forward_timed_events(x, out, mask, tile_policy=pol, act_quant=act)

    for _ in range(args.warmup):
        flush.zero_()
        timed_pass(timed_mask)
    torch.cuda.synchronize()
    status = B.moe_sync_status(layer.workspace)
    if status != 0:
        raise RuntimeError(f"device status {B.STATUS.get(status, status)} after warm-up")

    clocks_path = args.clocks_csv
    step_ms = []
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local, clocks_path) as clk:
        for _ in range(args.steps):
            flush.zero_()
            step_ms.append(timed_pass(timed_mask))
        torch.cuda.synchronize()
    barrier(world)
    status = B.moe_sync_status(layer.workspace)
    if status != 0:
        raise RuntimeError(f"device status {B.STATUS.get(status, status)} in the timed region")
    step_s = sum(s[-1] for s in step_ms) / 1e3
    # per-launch breakdown, after the timed region: every boundary recorded
    stage_ms = []
    for _ in range(min(args.steps, 5)):
        flush.zero_()
        stage_ms.append(timed_pass((1 << (nb + 1)) - 1))
    if B.moe_sync_status(layer.workspace) != 0:
        raise RuntimeError("device status after the per-stage steps")
    # the device's routing of the batch (rank 0 runs the batch in its own order),
    # read before later calls reuse the workspace, for the oracle leg's record
    topk_idx = layer.intermediate("topk_idx", T).cpu().numpy() if rank == 0 else None
    block = None
    if args.block or args.bias:
        # the same steps through moe_forward_block (RMSNorm, the layer, the residual
        # add) and/or with per-expert biases (moe_forward_biased); the layer's stage
        # times above explain them
        rng = np.random.default_rng(7)
        gub = dnb = None
        if args.bias:
            gub = torch.from_numpy((rng.standard_normal((inp.E, 2 * inp.I)) * 0.1)
                                   .astype(np.float32)).to(dev)
            dnb = torch.from_numpy((rng.standard_normal((inp.E, inp.d)) * 0.1)
                                   .astype(np.float32)).to(dev)
        if args.block:
            g = torch.from_numpy(rng.uniform(0.5, 1.5, inp.d).astype(np.float32)).to(dev)
            bws = torch.empty(B.moe_workspace_size_block(inp.E, inp.k, T, inp.d, inp.I),
                              dtype=torch.uint8, device=dev)

            def variant_step():
                B.moe_forward_block(x, g, 1e-5, layer.W_r, layer.b_r, layer.Wgu_codes,
                                    layer.Wgu_scales, layer.Wd_codes, layer.Wd_scales, inp.E,
                                    inp.k, T, inp.d, inp.I, out, bws, gu_bias=gub, down_bias=dnb)
        else:
            bws = layer.workspace

            def variant_step():
                B.moe_forward_biased(x, layer.W_r, layer.b_r, layer.Wgu_codes, layer.Wgu_scales,
                                     gub, layer.Wd_codes, layer.Wd_scales, dnb, inp.E, inp.k, T,
                                     inp.d, inp.I, out, bws)
        def plain_step():
            layer.forward(x, out)

        def timed(fn) -> float:
            flush.zero_()
            ev0 = torch.cuda.Event(enable_timing=True)
            ev1 = torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            fn()
            ev1.record(stream)
            ev1.synchronize()
            return ev0.elapsed_time(ev1) / 1e3

        for _ in range(args.warmup):
            timed(variant_step)
            timed(plain_step)
        barrier(world)
        torch.cuda.synchronize()
        # the plain layer timed the same way (two events, no per-stage events),
        # alternating with the variant so that both see the same conditions
        bsum = psum = 0.0
        for _ in range(args.steps):
            bsum += timed(variant_step)
            psum += timed(plain_step)
        if B.moe_sync_status(bws) != 0 or B.moe_sync_status(layer.workspace) != 0:
            raise RuntimeError("device status after the block / biased steps")
        extra = ("norm_and_residual" if args.block else "bias") + (
            "_and_bias" if args.block and args.bias else "")
        block = {"layer_ms_per_step": 1e3 * psum / args.steps,
                 f"{extra}_ms_per_step": 1e3 * (bsum - psum) / args.steps}
        step_s = bsum
    step_s_max = reduce_max(step_s, world)
    tokens_all = T * args.steps * world
    value = tokens_all / step_s_max
    ms_per_step = 1e3 * step_s_max / args.steps

    # dominant kernel: live CUDA-event durations of the gate/up GEMM launches
    # in the timed steps
    dom_ms = sum(s[dom] for s in step_ms) / len(step_ms)
    dom_flops = 4.0 * inp.d * inp.I * T * inp.k
    peaks, kind = load_peaks()
    stage_avg = {n: sum(s[i] for s in stage_ms) / len(stage_ms) for i, n in enumerate(B.STAGES)}
    counts = layer.intermediate("counts", T).cpu().numpy()
    touched = int((counts > 0).sum())
    # the load the routing puts on the experts (the skewed 128a4 workload
    # concentrates it): routed rows per touched expert, and the 256-row tiles
    # they make against the 74 CTA pairs of the prefill kernels
    nz = counts[counts > 0]
    tiles256 = int(np.sum((nz + 255) // 256))
    routing_load = {"rows_per_touched_expert": {"min": int(nz.min()), "median": float(np.median(nz)),
                                                "max": int(nz.max())},
                    "touched_experts": touched, "row_tiles_256": tiles256}
    # algorithmic bytes of one gate/up launch: the touched experts' MXFP4
    # gate/up weights (codes + scales), the permuted activations read, H written
    dom_bytes = (touched * (2 * inp.I * inp.d // 2 + 2 * inp.I * inp.d // 32)
                 + T * inp.k * inp.d * 2 + T * inp.k * inp.I * 2)
    decode = T * inp.k < 16 * inp.E       # few rows per expert: weight streaming
    if decode:
        peak = float(peaks["hbm_gbs"])
        achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "unit": "GB/s", "peak_source": f"hbm_gbs ({kind})",
                "algorithmic_bytes_per_launch": dom_bytes}
    else:
        # the peak of the MMA kind the kernel runs: bf16 precision runs at the
        # bf16 rate (kind::f16, or two E4M3 terms on the FP8-rate kind); w4a8
        # and w4a4 on one CTA at the FP8 rate (kind::mxf8f6f4); w4a4 on a CTA
        # pair at the FP4 rate (kind::mxf4): the measured bf16 peak times the
        # nominal dense ratios 2 and 4
        ratio, kname = 1.0, "bf16 rate"
        if args.act_quant != "bf16" and not quant_runs_mxf4(args, inp, T):
            ratio, kname = 2.0, "kind::mxf8f6f4, x2 (nominal FP8:BF16)"
        elif args.act_quant == "mxfp4":
            ratio, kname = 4.0, "kind::mxf4, x4 (nominal FP4:BF16)"
        peak = ratio * float(peaks["bf16_tflops"])
        achieved = dom_flops / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "unit": "TFLOP/s",
                "peak_source": f"bf16_tflops ({kind}, burst); {kname}",
                "algorithmic_flops_per_launch": dom_flops}
        # the pages' MXFP4 target: the same achieved rate against the dense FP4
        # peak, taken as the measured bf16 peak times the nominal dense ratio
        # (9 : 2.25 PFLOP/s); bf16-precision activations cannot use the FP4 kind
        fp4_peak = 4.0 * float(peaks["bf16_tflops"])
        roof["vs_mxfp4_peak"] = {
            "peak": fp4_peak, "frac": achieved / fp4_peak,
            "peak_source": f"bf16_tflops ({kind}, burst) x 4, the nominal dense FP4:BF16 ratio"}
    # the whole step against HBM: the touched experts' weights, x, out and the
    # router weights over the step time (decode steps are weight streaming)
    step_bytes = (touched * 13219200 * (inp.d * inp.I) / (2880 * 2880)
                  + 2 * T * inp.d * 2 + inp.E * inp.d * 4)
    roof["step_hbm"] = {"algorithmic_bytes": step_bytes,
                        "achieved_gbs": step_bytes / (ms_per_step * 1e-3) / 1e9,
                        "frac": step_bytes / (ms_per_step * 1e-3) / 1e9 / float(peaks["hbm_gbs"])}

    # end to end through the C ABI with host buffers: H2D + forward + D2H
    # (the quantised modes: pinned copies around moe_forward_ex, the calls a
    # user makes, since the host-buffer entry has no options)
    e2e_s = 0.0
    barrier(world)
    torch.cuda.synchronize()
    for _ in range(args.steps):
        flush.zero_()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        if act is None and pol == 0:
            layer.forward_hostio(x_host, out_host)
        else:
            x.copy_(x_host, non_blocking=True)
            B.moe_forward_ex(x, layer.W_r, layer.b_r, layer.Wgu_codes, layer.Wgu_scales,
                             layer.Wd_codes, layer.Wd_scales, inp.E, inp.k, T, inp.d, inp.I, out,
                             layer.workspace, tile_policy=pol, act_quant=act or "bf16")
            out_host.copy_(out, non_blocking=True)
        ev1.record(stream)
        ev1.synchronize()
        e2e_s += ev0.elapsed_time(ev1) / 1e3
    barrier(world)
    e2e_s_max = reduce_max(e2e_s, world)
    e2e_value = tokens_all / e2e_s_max

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {"bf16": "bf16", "mxfp8": "e4m3", "mxfp4": "e2m1"}[args.act_quant],
        "data": "synthetic",
        "config": dict(workload_config(inp, name), tile_policy=args.tile_policy,
                       activations={"bf16": "bf16 (the pages' layer)",
                                    "mxfp8": "MXFP8 E4M3 (the w4a8 layer)",
                                    "mxfp4": "MXFP4 E2M1 (the w4a4 layer)"}[args.act_quant],
                       **({"block": "out = h + MoE(RMSNorm(h)), eps 1e-5"} if args.block else {}),
                       **({"expert_biases": "gate/up [E, 2I] and down [E, d], f32"}
                          if args.bias else {})),
        "layer_tflops": layer_flops(inp.d, inp.I, inp.E, inp.k, T) * args.steps * world
        / step_s_max / 1e12,
        "roofline": dict(roof, kernel=DOMINANT_STAGE, achieved=achieved, peak=peak,
                         frac=achieved / peak,
                         traffic=recorded_traffic(name, T, args.tile_policy, args.act_quant),
                         avg_launch_ms=dom_ms, touched_experts=touched),
        "stage_ms": stage_avg,
        "routing_load": routing_load,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(T * inp.d * 2),
                "d2h_bytes_per_step": int(T * inp.d * 2), "host_buffers": near.describe()},
        "gpu_launches": (forward_launches(args, inp, T) + (1 if args.block else 0)) * args.steps,
        "clocks": clk.summary(),
    }
    line["_topk_idx"] = topk_idx
    if block:
        line["block" if args.block else "bias"] = block
    return line


def probe_tensor():
    """Measured UMMA rates on this device (the separate probe library): MACs per
    SM clock for bf16 (kind::f16, K = 16), the block-scaled E2M1 x E4M3 kind
    (kind::mxf8f6f4, K = 32) and the block-scaled E2M1 x E2M1 kind (kind::mxf4,
    K = 64), M = 128, several N and UMMAs per commit; TFLOP/s at the SM count and
    the maximum SM clock."""
    import torch
    from sparse_moe_layer_05_b200 import binding as B
    torch.cuda.init()
    props = torch.cuda.get_device_properties(0)
    peaks, _ = load_peaks()
    mhz = float(peaks.get("sm_max_mhz", 1965.0))
    rows = []
    for kind, kname in ((0, "bf16"), (1, "e2m1_x_e4m3_block_scaled"),
                        (2, "e2m1_x_e2m1_block_scaled")):
        for n in (32, 64, 128, 240, 256):
            for per_commit in (4, 16):
                r = B.moe_probe_tensor_rate(kind, n, per_commit)
                rows.append({"kind": kname, "N": n, "umma_per_commit": per_commit,
                             "mac_per_clk_sm": round(r, 1),
                             "tflops_at_max_clock": round(2 * r * props.multi_processor_count
                                                          * mhz * 1e6 / 1e12, 1)})
    print(json.dumps({"probe": "tensor_rate", "sms": props.multi_processor_count,
                      "sm_max_mhz": mhz, "M": 128, "rows": rows}))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="20b", choices=list(W.SHAPES))
    ap.add_argument("--T", type=int, default=None, help="tokens per GPU (default: prefill T)")
    ap.add_argument("--ref-tokens", type=int, default=2, help="oracle tokens per reference step")
    ap.add_argument("--block", action="store_true",
                    help="time the MoE sublayer with its pre-norm and residual add "
                         "(moe_forward_block: out = h + MoE(RMSNorm(h)))")
    ap.add_argument("--clocks-csv", default=None,
                    help="also write every clock sample of the timed region to this CSV file")
    ap.add_argument("--bias", action="store_true",
                    help="time the layer with per-expert gate/up and down biases "
                         "(moe_forward_biased; with --block, the sublayer with biases)")
    ap.add_argument("--probe-tensor", action="store_true",
                    help="print the measured UMMA rates (MAC per SM clock) and exit")
    ap.add_argument("--tile-policy", type=int, default=0, choices=[0, 1, 2, 3, 4, 5],
                    help="grouped-GEMM tiles: 0 by shape, 1 single, 2 pair, 3 swap, "
                         "4 block-scaled, 5 block-scaled CTA pair")
    ap.add_argument("--act-quant", default="bf16", choices=["bf16", "mxfp8", "mxfp4"],
                    help="activation precision of the expert GEMMs: bf16 (the pages' layer), "
                         "or the w4a8 / w4a4 layers (moe_forward_ex act_quant)")
    ap.add_argument("--cpu-sample", type=int, default=256,
                    help="tokens of the batch the oracle runs for cpu_baseline (0 = skip)")
    args = ap.parse_args(argv)
    if args.probe_tensor:
        probe_tensor()
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 must be launched with torch.distributed.run")
    name = args.workload
    inp = W.make_inputs(name, T=args.T)

    if world > 1:
        import torch.distributed as dist
        backend = "gloo" if args.impl == "reference" else "nccl"
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))

    try:
        if args.impl == "reference":
            line = run_reference(args, inp, name)
        else:
            line = run_ours(args, inp, name)
            gpu_idx = line.pop("_topk_idx", None) if line is not None else None
            if line is not None and rank == 0 and world == 1 and args.cpu_sample > 0:
                if gpu_idx is not None and not args.block:
                    line["parity"] = routing_parity(inp, gpu_idx)
                n = min(args.cpu_sample, inp.T)
                v, dt = oracle_tokens_per_s(inp, np.arange(n))
                line["cpu_baseline"] = {
                    "value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                    "sample": f"first {n} tokens of the {inp.T}-token batch, {dt:.1f} s of "
                              f"fp64 oracle work on the host"}
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
