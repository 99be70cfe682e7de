"""Seeded synthetic inputs for the sparse-MoE layer.

This module is shared by the CPU oracle's tests and by the GPU path's tests
and benchmark. It only *draws* inputs: it holds no step of the layer's
arithmetic (no MXFP4 decode, no routing, no expert math). Every array is
produced on the CPU from numpy's PCG64 generator so that the oracle and the
CUDA path see identical bits.

Workloads follow the shapes the pages give:

* ``fixture``  -- the shrunken gpt-oss fixture (hidden 64, intermediate 128,
  4 experts, top-2), "shrink/gpt_oss-mic", "Config changes" table.
* ``20b``      -- gpt-oss-20b MoE shape (width 2,880, intermediate 2,880,
  32 experts, top-4), field guide "gpt-oss 20B", "03 Sparse Mixture of Experts".
* ``64a8``     -- silent-init x2 expansion of ``20b`` (64 experts, top-8),
  "llm-surgery-dark-arts-gpt-oss-40b-64a8-init", section 2 "Silent Init".
* ``96a12``    -- silent-init x3 expansion of ``20b`` (96 experts, top-12),
  the same page's 96a12 variant (copies at e+32 and e+64).
* ``64a4``, ``96a4`` -- the same two layers with the active count reduced to
  4 (the page's "64a8 to 64a4, 96a12 to 96a4"); the page reaches it by router
  bias adjustment after training, which is not specified, so at silent init
  these are the expanded layers run at k = 4.
* ``128a4``    -- gpt-oss-120b routing (128 experts, top-4), "gpt-oss-20b and
  gpt-oss-120b" overview; with 8 router biases raised by 2.0 (skewed load).
* ``248a20``   -- "gpt-oss-220a20b" model card: 128 base + 120 added expert
  rows, top-20.

Layouts (all C-contiguous, row-major):

* ``x``          [T, d]          uint16 (bf16 bit patterns)
* ``W_r``        [E, d]          float32
* ``b_r``        [E]             float32
* ``Wgu_codes``  [E, 2I, d/2]    uint8, rows 0..I-1 gate, I..2I-1 up;
                                 byte b holds element 2b (low nibble) and
                                 element 2b+1 (high nibble)
* ``Wgu_scales`` [E, 2I, d/32]   uint8 E8M0 (one per 32 consecutive elements
                                 along the contraction dimension)
* ``Wd_codes``   [E, d, I/2]     uint8
* ``Wd_scales``  [E, d, I/32]    uint8

Distribution notation N(mu, v) is read with v as the variance.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = [
    "Shape",
    "SHAPES",
    "MoEInputs",
    "make_inputs",
    "make_custom",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
]


@dataclasses.dataclass(frozen=True)
class Shape:
    name: str
    d: int
    I: int
    E: int
    k: int
    T_prefill: int
    T_decode: Optional[int]
    scale_lo: int  # inclusive E8M0 byte range of the expert scales
    scale_hi: int
    doc: str


SHAPES: Dict[str, Shape] = {
    "fixture": Shape("fixture", 64, 128, 4, 2, 256, None, 121, 124,
                     "d=64 I=128 E=4 k=2, x~N(0,1) fp32 rounded to bf16, "
                     "scale exponent uniform in [-6,-3]"),
    "20b": Shape("20b", 2880, 2880, 32, 4, 8192, None, 119, 123,
                 "gpt-oss-20b MoE layer, unbiased routing, scale exponent "
                 "uniform in [-8,-4]"),
    "64a8": Shape("64a8", 2880, 2880, 64, 8, 8192, 64, 119, 123,
                  "silent-init x2 expansion of 20b (copies at e+32)"),
    "96a12": Shape("96a12", 2880, 2880, 96, 12, 8192, 64, 119, 123,
                   "silent-init x3 expansion of 20b (copies at e+32, e+64)"),
    "64a4": Shape("64a4", 2880, 2880, 64, 4, 8192, 64, 119, 123,
                  "64a8 layer run with the active count reduced to 4"),
    "96a4": Shape("96a4", 2880, 2880, 96, 4, 8192, 64, 119, 123,
                  "96a12 layer run with the active count reduced to 4"),
    "128a4": Shape("128a4", 2880, 2880, 128, 4, 16384, 32, 119, 123,
                   "gpt-oss-120b routing with +2.0 bias on experts 0..7"),
    "248a20": Shape("248a20", 2880, 2880, 248, 20, 4096, 16, 119, 123,
                    "128 base + 120 added experts (copies with N(0,0.01)-"
                    "perturbed scales), top-20"),
}


@dataclasses.dataclass
class MoEInputs:
    d: int
    I: int
    E: int
    k: int
    T: int
    x: np.ndarray
    W_r: np.ndarray
    b_r: np.ndarray
    Wgu_codes: np.ndarray
    Wgu_scales: np.ndarray
    Wd_codes: np.ndarray
    Wd_scales: np.ndarray
    name: str = "custom"
    notes: str = ""

    def take_tokens(self, T: int) -> "MoEInputs":
        """Same layer, first ``T`` tokens of the activation batch."""
        return dataclasses.replace(self, T=T, x=np.ascontiguousarray(self.x[:T]))

    @property
    def weight_bytes_per_expert(self) -> int:
        return (self.Wgu_codes[0].nbytes + self.Wgu_scales[0].nbytes
                + self.Wd_codes[0].nbytes + self.Wd_scales[0].nbytes)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest even), returned as uint16 bits.

    Input generation only: the fixture draws fp32 activations and rounds them
    once so that every consumer sees the same bf16 values.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def _codes(rng: np.random.Generator, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return np.frombuffer(rng.bytes(n), dtype=np.uint8).reshape(shape).copy()


def _scales(rng: np.random.Generator, shape, lo: int, hi: int) -> np.ndarray:
    return rng.integers(lo, hi + 1, size=shape, dtype=np.uint8)


def make_custom(d: int, I: int, E: int, k: int, T: int, seed: int = 0,
                scale_lo: int = 119, scale_hi: int = 123,
                bias_var: float = 0.1, name: str = "custom",
                T_draw: Optional[int] = None) -> MoEInputs:
    """Layer of arbitrary shape drawn like the 20b recipe.

    Order of draws from one PCG64 stream: x (``T_draw`` rows, default T),
    W_r, b_r, Wgu_codes, Wgu_scales, Wd_codes, Wd_scales. The first ``T``
    rows of x are kept, so every T <= T_draw sees the same weights.
    """
    if d % 32 or I % 32:
        raise ValueError("d and I must be multiples of the 32-element MX group")
    T_draw = T if T_draw is None else max(T_draw, T)
    rng = np.random.Generator(np.random.PCG64(seed))
    x = np.ascontiguousarray(_normal_bf16(rng, (T_draw, d))[:T])
    W_r = (rng.standard_normal((E, d), dtype=np.float64) / np.sqrt(d)).astype(np.float32)
    b_r = (rng.standard_normal(E, dtype=np.float64) * np.sqrt(bias_var)).astype(np.float32)
    Wgu_codes = _codes(rng, (E, 2 * I, d // 2))
    Wgu_scales = _scales(rng, (E, 2 * I, d // 32), scale_lo, scale_hi)
    Wd_codes = _codes(rng, (E, d, I // 2))
    Wd_scales = _scales(rng, (E, d, I // 32), scale_lo, scale_hi)
    return MoEInputs(d, I, E, k, T, x, W_r, b_r, Wgu_codes, Wgu_scales,
                     Wd_codes, Wd_scales, name=name)


def _expand_silent(base: MoEInputs, M: int) -> MoEInputs:
    """Duplicate every expert and router row M times (copies at e + m*E)."""
    rep = lambda a: np.ascontiguousarray(np.concatenate([a] * M, axis=0))
    return MoEInputs(base.d, base.I, base.E * M, base.k * M, base.T, base.x,
                     rep(base.W_r), rep(base.b_r), rep(base.Wgu_codes),
                     rep(base.Wgu_scales), rep(base.Wd_codes), rep(base.Wd_scales),
                     name=f"{base.E * M}a{base.k * M}",
                     notes=f"silent-init x{M} of {base.name}")


def expand_silent(base: MoEInputs, M: int) -> MoEInputs:
    """Public wrapper: the x-M silent-init expansion of a layer."""
    return _expand_silent(base, M)


def make_inputs(name: str, T: Optional[int] = None, seed: int = 0) -> MoEInputs:
    """Seeded inputs for one named workload.

    ``T`` defaults to the workload's prefill token count. Token counts below
    the prefill count take the first T rows of the same activation draw, so a
    decode step is a prefix of the prefill batch.
    """
    s = SHAPES[name]
    T_full = s.T_prefill
    T = T_full if T is None else T
    if name in ("fixture", "20b"):
        return make_custom(s.d, s.I, s.E, s.k, T, seed=seed,
                           scale_lo=s.scale_lo, scale_hi=s.scale_hi,
                           name=name, T_draw=T_full)
    if name in ("64a8", "96a12", "64a4", "96a4"):
        base = make_inputs("20b", T=T, seed=seed)
        out = _expand_silent(base, 2 if name.startswith("64") else 3)
        out.k = s.k
        out.name = name
        return out
    if name == "128a4":
        inp = make_custom(s.d, s.I, s.E, s.k, T, seed=seed + 1,
                          scale_lo=s.scale_lo, scale_hi=s.scale_hi, name=name,
                          T_draw=T_full)
        inp.b_r[:8] += np.float32(2.0)
        inp.notes = "router bias of experts 0..7 raised by +2.0"
        return inp
    if name == "248a20":
        return _make_248(T, seed)
    raise KeyError(name)


def _make_248(T: int, seed: int) -> MoEInputs:
    s = SHAPES["248a20"]
    base = make_custom(s.d, s.I, 128, s.k, T, seed=seed + 2,
                       scale_lo=s.scale_lo, scale_hi=s.scale_hi, name="248a20-base",
                       T_draw=s.T_prefill)
    rng = np.random.Generator(np.random.PCG64(seed + 3))
    # fresh router over all 248 rows: W_r ~ N(0, 1/d), b_r ~ N(0, 0.1)
    W_r = (rng.standard_normal((248, s.d), dtype=np.float64) / np.sqrt(s.d)).astype(np.float32)
    b_r = (rng.standard_normal(248, dtype=np.float64) * np.sqrt(0.1)).astype(np.float32)
    src = rng.integers(0, 128, size=120)

    def perturb(sc: np.ndarray) -> np.ndarray:
        # log2(scale) + N(0, 0.01), rounded back to the integer E8M0 grid
        eps = rng.standard_normal(sc.shape) * 0.1
        return np.clip(np.rint(sc.astype(np.float64) + eps), 0, 254).astype(np.uint8)

    add_gu_sc = np.stack([perturb(base.Wgu_scales[j]) for j in src])
    add_d_sc = np.stack([perturb(base.Wd_scales[j]) for j in src])
    cat = lambda a, b: np.ascontiguousarray(np.concatenate([a, b], axis=0))
    changed = int((add_gu_sc != base.Wgu_scales[src]).sum()
                  + (add_d_sc != base.Wd_scales[src]).sum())
    return MoEInputs(
        s.d, s.I, 248, s.k, T, base.x, W_r, b_r,
        cat(base.Wgu_codes, base.Wgu_codes[src]), cat(base.Wgu_scales, add_gu_sc),
        cat(base.Wd_codes, base.Wd_codes[src]), cat(base.Wd_scales, add_d_sc),
        name="248a20",
        notes=f"added experts copy base rows {src[:4].tolist()}...; "
              f"{changed} scale bytes changed by the perturbation")
