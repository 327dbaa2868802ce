"""Writes tests/golden/oracle_tiny_fp32_T256.json from the fp64 oracle alone.

The pages print no worked numerical example for the method, so the only stored
expected values here are the oracle's own, on the tiny fp32 workload (B=1,
Hq=Hkv=2, T=256, planted keys, seed 0), kept to catch unintended drift of the
oracle's arithmetic.  Every value comes from ``oracle.polar_fwd``; nothing is
taken from the CUDA library.  Run from the repository root:

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


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_fp32_T256.json")
    with open(path, "w") as f:
        json.dump(compute(), f, indent=0)
    print("wrote", path)
