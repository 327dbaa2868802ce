"""GPU parity of the prefill backward (polar_attn_bwd) against the fp64 oracle
gradients, which are themselves pinned by finite differences of the oracle
forward."""
import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

# normwise max|gpu - oracle| / max|oracle| per slice: fp32 inputs run fp32
# arithmetic; bf16 inputs run the gradient products on the tensor cores with
# dA, dS and the weights rounded to bf16 (the forward's bf16 output tolerance).
GRAD_TOL = {"fp32": 2e-3, "bf16": 2e-2}
# Where the exact gradient vanishes (one visible key: the direction, gate and
# magnitude do not depend on q), what is left is rounding residue: about 1e-7
# in fp32, and about 1e-2 when the products run on bf16 operands.  The slice
# scale therefore has a floor, in the gradients' natural units (dq, dk, dv are
# of order 1-10 here: c = 8 times unit vectors).
GRAD_FLOOR = {"fp32": 1e-3, "bf16": 1.0}


def _gout(w, seed):
    g = torch.Generator().manual_seed(seed)
    t = torch.randn((w.B, w.T, w.Hq, w.D), generator=g)
    return t.to(torch.bfloat16 if w.dtype == "bf16" else torch.float32)


def _run(w, x, gout):
    xd = PT.to_device(x)
    dq, dk, dv, du = pa.bwd(xd["q"], xd["k"], xd["v"], xd["u"], gout.cuda().contiguous(),
                            s=w.s, alpha=w.alpha, L=w.L, beta=w.beta, window=w.window)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    return dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy(), du.cpu().numpy()


def _slices(a, axis_heads):
    """Per-(batch, head) slices of a [B, T, H, D] gradient."""
    B, H = a.shape[0], a.shape[axis_heads]
    return [a[b, :, h] for b in range(B) for h in range(H)]


def _check(name, got, ref, tol, floor):
    assert np.all(np.isfinite(got)), f"{name}: non-finite gradient"
    worst = 0.0
    pairs = [(got, ref)] if got.ndim == 2 else list(zip(_slices(got, 2), _slices(ref, 2)))
    for g, r in pairs:
        scale = max(np.max(np.abs(r)), floor)
        worst = max(worst, np.max(np.abs(g - r)) / scale)
    print(f"{name}: normwise error {worst:.3e} (tol {tol})")
    assert worst <= tol, f"{name}: normwise error {worst:.3e} > {tol}"
    return worst


def _compare(w, x, seed=0):
    gout = _gout(w, seed)
    got = _run(w, x, gout)
    ref = PT.oracle_bwd(w, x, gout)
    for name, g, r in zip(("dq", "dk", "dv", "du"), got, ref):
        _check(f"{name} T={w.T} window={w.window}", g, r, GRAD_TOL[w.dtype], GRAD_FLOOR[w.dtype])


CASES = [(1, 2, 0, "bf16"), (77, 2, 0, "bf16"), (300, 4, 0, "bf16"), (300, 2, 64, "bf16"),
         (500, 8, 0, "bf16"), (200, 2, 0, "fp32")]


@pytest.mark.parametrize("T,G,Wn,dt", CASES)
def test_small_vs_oracle(cuda_ok, T, G, Wn, dt):
    """One key (n = 1: gate 1/2, n_eff 1), ragged lengths, GQA groups 2/4/8, a
    window, fp32 inputs; the count vector is large enough that the magnitude
    channel's gradient matters."""
    w = W.small_prefill(B=2, T=T, Hq=2 * G, Hkv=2, dtype=dt, seed=T + G, plant="frac",
                        plant_frac=0.02, L=32, window=Wn)
    x = W.prefill_inputs(w, "cpu")
    x["u"] = x["u"] * 25.0  # |u| ~ 1: comparable to the unit direction
    _compare(w, x, seed=T)


def test_medium_temperature_active(cuda_ok):
    w = W.small_prefill(B=1, T=1024, Hq=8, Hkv=2, dtype="bf16", seed=3, plant="frac",
                        plant_frac=0.01, L=256)
    x = W.prefill_inputs(w, "cpu")
    x["u"] = x["u"] * 25.0
    _compare(w, x, seed=5)


def test_multi_tile_gqa4_ragged(cuda_ok):
    """Twelve query and key tiles with a ragged last one (T = 1500), four query
    heads per kv head: every (key tile, query tile) pair of the tensor-core
    passes, the diagonal tiles and the padded rows past the end."""
    w = W.small_prefill(B=2, T=1500, Hq=8, Hkv=2, dtype="bf16", seed=15, plant="frac",
                        plant_frac=0.01, L=512)
    x = W.prefill_inputs(w, "cpu")
    x["u"] = x["u"] * 25.0
    _compare(w, x, seed=7)


def test_window_multi_tile(cuda_ok):
    """A sliding window of 200 keys over 900 rows: key tiles whose rows reach
    past the window's edge, and query tiles that start after it."""
    w = W.small_prefill(B=1, T=900, Hq=4, Hkv=2, dtype="bf16", seed=16, plant="frac",
                        plant_frac=0.01, L=64, window=200)
    x = W.prefill_inputs(w, "cpu")
    x["u"] = x["u"] * 25.0
    _compare(w, x, seed=8)


def test_tied_max_takes_the_first_key(cuda_ok):
    """Every key appears twice in a row (positions 2m and 2m+1, equal bits),
    so each row's max raw dot is attained by two keys; the max's subgradient
    goes to the first of them, as in the oracle.  A kernel that split it, or
    gave it to the later copy, would move dk between the twins."""
    w = W.small_prefill(B=1, T=600, Hq=4, Hkv=2, dtype="bf16", seed=17, plant="frac",
                        plant_frac=0.02, L=128)
    x = W.prefill_inputs(w, "cpu")
    x["k"][:, 1::2] = x["k"][:, 0::2]
    x["v"][:, 1::2] = x["v"][:, 0::2]
    x["u"] = x["u"] * 25.0
    _compare(w, x, seed=9)


def test_train_length_full_size_batch0(cuda_ok):
    """The bench's backward launch (B=8, T=2048, Hq=16, Hkv=4, bf16, 1% planted
    keys): the whole call runs on the GPU, and batch 0's gradients (every row,
    key and dimension of it; batches are independent) are checked against the
    oracle run on batch 0 alone.  du sums over every batch, so it is left to
    the smaller tests, which compare it with the oracle directly."""
    w = W.TRAIN
    x = W.prefill_inputs(w, "cpu")
    gout = _gout(w, seed=21)
    dq, dk, dv, _ = _run(w, x, gout)
    x0 = {k: (v[:1] if k in ("q", "k", "v") else v) for k, v in x.items()}
    import dataclasses
    w0 = dataclasses.replace(w, B=1)
    ref = PT.oracle_bwd(w0, x0, gout[:1])
    for name, g, r in zip(("dq", "dk", "dv"), (dq[:1], dk[:1], dv[:1]), ref[:3]):
        _check(f"{name} full-size batch 0", g, r, GRAD_TOL["bf16"], GRAD_FLOOR["bf16"])


def test_deterministic(cuda_ok):
    w = W.small_prefill(B=1, T=700, Hq=4, Hkv=2, dtype="bf16", seed=4, plant="frac",
                        plant_frac=0.02)
    x = W.prefill_inputs(w, "cpu")
    gout = _gout(w, 1)
    a = _run(w, x, gout)
    b = _run(w, x, gout)
    for ga, gb in zip(a, b):
        assert np.array_equal(ga, gb)


def test_empty_sequence_zeroes_du(cuda_ok):
    w = W.small_prefill(B=1, T=0, Hq=4, Hkv=2, dtype="bf16", seed=1)
    u = torch.ones((4, 64), device="cuda")
    e = torch.empty((1, 0, 4, 64), device="cuda", dtype=torch.bfloat16)
    ek = torch.empty((1, 0, 2, 64), device="cuda", dtype=torch.bfloat16)
    du = torch.full((4, 64), 3.0, device="cuda")
    pa.bwd(e, ek, ek, u, e, du=du)
    torch.cuda.synchronize()
    assert torch.all(du == 0)
