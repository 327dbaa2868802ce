"""GPU parity of the CUDA-core prefill kernel against the fp64 oracle."""
import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _run(w, impl="simt"):
    x = W.prefill_inputs(w, "cpu")
    xd = PT.to_device(x)
    out, neff = pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], s=w.s, alpha=w.alpha, L=w.L,
                       beta=w.beta, impl=impl)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    return x, out, neff


def test_tiny_fp32_all_rows(cuda_ok):
    """The tiny fp32 workload, every row: fp32 FFMA on the exact inputs."""
    w = W.TINY
    x, out, neff = _run(w)
    ref = PT.oracle_prefill(w, x)
    rows = np.arange(w.B * w.Hq * w.T)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_FP32, 1e-4, what="tiny fp32")


@pytest.mark.parametrize("T", [1, 2, 63, 129, 300])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_ragged_small(cuda_ok, T, dtype):
    w = W.small_prefill(B=2, T=T, Hq=8, Hkv=2, dtype=dtype, seed=T, plant="frac", plant_frac=0.05,
                        L=64)
    x, out, neff = _run(w)
    ref = PT.oracle_prefill(w, x)
    rows = np.arange(w.B * w.Hq * w.T)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    tol = PT.OUT_TOL_FP32 if dtype == "fp32" else PT.OUT_TOL_BF16
    PT.compare(o, n, ref, grp, tol, what=f"simt {dtype} T={T}")


def test_causality_on_gpu(cuda_ok):
    """Changing keys/values after row i leaves rows <= i bit-identical."""
    w = W.small_prefill(B=1, T=256, Hq=4, Hkv=1, dtype="bf16", seed=3)
    x = PT.to_device(W.prefill_inputs(w, "cpu"))
    a, na = pa.fwd(x["q"], x["k"], x["v"], x["u"], impl="simt", L=64)
    k2, v2 = x["k"].clone(), x["v"].clone()
    k2[:, 200:] = k2[:, 200:].flip(1)
    v2[:, 200:] = -v2[:, 200:]
    b, nb = pa.fwd(x["q"], k2, v2, x["u"], impl="simt", L=64)
    assert torch.equal(a[:, :200], b[:, :200]) and torch.equal(na[..., :200], nb[..., :200])
    assert not torch.equal(a[:, 200:], b[:, 200:])
