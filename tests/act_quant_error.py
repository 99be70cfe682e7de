"""Simulated cost of quantising the expert inputs (the oracle's ``act_quant``).

Runs the fp64 oracle on the first tokens of a seeded workload three times --
exact, with MXFP8 (E4M3) blocks and with MXFP4 (E2M1) blocks on every expert's
input rows and hidden rows -- and prints, per mode, the largest and the RMS
deviation from the exact output relative to the exact output's RMS, next to
the layer's output tolerance (2e-2 x RMS). CPU only; uses only the oracle and
the seeded input generators.

    python -m tests.act_quant_error [--workload 20b] [--tokens 64]
"""
import argparse
import json

import numpy as np

from oracle import moe_oracle as O
from sparse_moe_layer_05_b200 import workloads as W

TOL = 2e-2


def simulate(name: str, tokens: int) -> dict:
    inp = W.make_inputs(name, T=tokens)
    args = (inp.x, inp.W_r, inp.b_r, inp.Wgu_codes, inp.Wgu_scales, inp.Wd_codes,
            inp.Wd_scales)
    exact = O.moe_forward(*args, k=inp.k)
    rms = float(np.sqrt(np.mean(exact ** 2)))
    res = {"workload": name, "tokens": tokens, "tolerance_x_rms": TOL}
    for mode, fmt in (("w4a8 (E4M3 blocks)", "e4m3"), ("w4a4 (E2M1 blocks)", "e2m1")):
        err = O.moe_forward(*args, k=inp.k, act_quant=fmt) - exact
        res[mode] = {"max_err_x_rms": float(np.max(np.abs(err)) / rms),
                     "rms_err_x_rms": float(np.sqrt(np.mean(err ** 2)) / rms),
                     "elements_over_tolerance": float(np.mean(np.abs(err) > TOL * rms))}
    return res


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="20b", choices=list(W.SHAPES))
    ap.add_argument("--tokens", type=int, default=64)
    a = ap.parse_args(argv)
    print(json.dumps(simulate(a.workload, a.tokens), indent=1))


if __name__ == "__main__":
    main()
