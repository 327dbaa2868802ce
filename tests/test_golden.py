"""The oracle still reproduces its committed golden fixture (CPU)."""
import json
import os

import numpy as np

import oracle
from polar_attention_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_golden_fixture():
    with open(os.path.join(HERE, "golden", "oracle_tiny_fp32_T256.json")) as f:
        g = json.load(f)
    w = W.TINY
    x = W.prefill_inputs(w, "cpu")
    h = {k: W.to_host_bits(x[k]) for k in ("q", "k", "v")}
    res = oracle.polar_fwd(h["q"], h["k"], h["v"], x["u"].numpy(),
                           oracle.Params(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta))
    np.testing.assert_allclose(res.neff, g["neff"], rtol=1e-13)
    np.testing.assert_allclose(res.out[g["sample_rows"]], g["out_sample"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(res.stats[g["sample_rows"]], g["stats_sample"], rtol=1e-13,
                               atol=1e-15)


def test_tiny_workload_has_planted_signal():
    """The planted keys make some rows concentrate (small n_eff) while the
    unplanted rows spread over many keys: the workload exercises both ends."""
    with open(os.path.join(HERE, "golden", "oracle_tiny_fp32_T256.json")) as f:
        g = json.load(f)
    neff = np.array(g["neff"])
    assert neff.min() >= 1.0
    assert (neff[np.r_[64:256, 320:512]] < 3).any()
    assert (neff > 20).any()


def test_memory_oracle_matches_golden_fixture():
    with open(os.path.join(HERE, "golden", "oracle_gdelta_fp32_T130.json")) as f:
        g = json.load(f)
    w = W.small_gdelta(B=1, T=130, H=2, dtype="fp32", seed=5)
    x = W.gdelta_inputs(w, "cpu")
    o, S = oracle.gdelta(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(),
                         x["alpha"].numpy().astype(np.float64), x["beta"].numpy().astype(np.float64))
    np.testing.assert_allclose(o[0, g["sample_tokens"]], g["out_sample"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S[0, :, 0], g["state_row0"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(np.sqrt((S[0] ** 2).sum(axis=(1, 2))), g["state_fro"], rtol=1e-12)
