"""Writes tests/golden/oracle_tiny_fp32_T256.json and
tests/golden/oracle_gdelta_fp32_T130.json from the fp64 oracle alone.

The pages print no worked numerical example for the method, so the only stored
expected values here are the oracle's own, on the tiny fp32 workload (B=1,
Hq=Hkv=2, T=256, planted keys, seed 0), kept to catch unintended drift of the
oracle's arithmetic.  Every value comes from ``oracle.polar_fwd``; nothing is
taken from the CUDA library.  The memory-channel fixture holds the gated-delta
oracle's outputs and final state on a small fp32 case (B=1, T=130, H=2: two
full chunks and a ragged tail, seed 5).  Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from polar_attention_b200 import workloads as W  # noqa: E402

SAMPLE_ROWS = list(range(0, 512, 37)) + [255, 256, 511]


def compute():
    w = W.TINY
    x = W.prefill_inputs(w, "cpu")
    h = {k: W.to_host_bits(x[k]) for k in ("q", "k", "v")}
    p = oracle.Params(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta)
    res = oracle.polar_fwd(h["q"], h["k"], h["v"], x["u"].numpy(), p)
    return {
        "workload": w.describe() + f", seed {w.seed}, planted keys ({w.plant})",
        "params": {"s": w.s, "alpha": w.alpha, "L": w.L, "beta": w.beta},
        "row_index": "flat (b*Hq + h)*T + i",
        "neff": [float(x) for x in res.neff],
        "sample_rows": SAMPLE_ROWS,
        "out_sample": [[float(x) for x in res.out[r]] for r in SAMPLE_ROWS],
        "stats_sample": [[float(x) for x in res.stats[r]] for r in SAMPLE_ROWS],
    }


GD_WORKLOAD = dict(B=1, T=130, H=2, dtype="fp32", seed=5)
GD_ROWS = [0, 1, 63, 64, 65, 127, 128, 129]


def compute_gdelta():
    w = W.small_gdelta(**GD_WORKLOAD)
    x = W.gdelta_inputs(w, "cpu")
    o, S = oracle.gdelta(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(),
                         x["alpha"].numpy().astype("float64"), x["beta"].numpy().astype("float64"))
    return {
        "workload": w.describe() + f", seed {w.seed}",
        "sample_tokens": GD_ROWS,
        "out_sample": [[[float(v) for v in o[0, t, h]] for h in range(w.H)] for t in GD_ROWS],
        "state_row0": [[float(v) for v in S[0, h, 0]] for h in range(w.H)],
        "state_fro": [float((S[0, h] ** 2).sum() ** 0.5) for h in range(w.H)],
    }


if __name__ == "__main__":
    here = os.path.dirname(os.path.abspath(__file__))
    for name, fn in (("oracle_tiny_fp32_T256.json", compute),
                     ("oracle_gdelta_fp32_T130.json", compute_gdelta)):
        path = os.path.join(here, name)
        with open(path, "w") as f:
            json.dump(fn(), f, indent=0)
        print("wrote", path)
