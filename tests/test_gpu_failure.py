"""Failure detection on the GPU without a fault: a bounded wait that can never
complete gives up, reports POLAR_ERR_TIMEOUT through the status word, and
leaves the context usable."""
import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import native
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives(cuda_ok):
    assert pa.get_status() == 0
    native.selftest_timeout()
    assert pa.get_status() == 5    # POLAR_ERR_TIMEOUT
    assert pa.get_status() == 0    # read and cleared
    # the next call computes normally
    w = W.small_prefill(B=1, T=200, Hq=4, Hkv=2, dtype="bf16", seed=3, plant="frac",
                        plant_frac=0.02)
    x = W.prefill_inputs(w, "cpu")
    xd = PT.to_device(x)
    out, neff = pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], s=w.s, alpha=w.alpha, L=w.L,
                       beta=w.beta)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    rows = np.arange(w.B * w.Hq * w.T)
    ref = PT.oracle_prefill(w, x, rows)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what="after a timeout")
