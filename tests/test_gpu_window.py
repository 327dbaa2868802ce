"""GPU parity of the sliding-window option (polar_params_t.window) against the
oracle: tensor-core and CUDA-core prefill, single-token and multi-token decode."""
import dataclasses

import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _prefill(w, x, impl="tc", **kw):
    xd = PT.to_device(x)
    out, neff = pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], s=w.s, alpha=w.alpha, L=w.L,
                       beta=w.beta, impl=impl, window=w.window, **kw)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    return out, neff


def _check_prefill(w, x, out, neff, rows=None, tol=PT.OUT_TOL_BF16):
    rows = np.arange(w.B * w.Hq * w.T) if rows is None else rows
    ref = PT.oracle_prefill(w, x, rows)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, tol, what=f"window {w.window} T={w.T}")


# (T, G, W): one key, less than a tile, exactly a tile, not a tile multiple
# (several lower-masked tiles per query tile), the temperature active past
# L=256 within the window, and a window longer than the sequence.
CASES = [(300, 2, 1), (300, 2, 64), (500, 4, 128), (777, 8, 200), (1000, 2, 333), (700, 2, 1000)]


@pytest.mark.parametrize("T,G,Wn", CASES)
def test_tc_prefill_window_all_rows(cuda_ok, T, G, Wn):
    w = W.small_prefill(B=2, T=T, Hq=2 * G, Hkv=2, dtype="bf16", seed=T + Wn, plant="frac",
                        plant_frac=0.02, L=256, window=Wn)
    x = W.prefill_inputs(w, "cpu")
    out, neff = _prefill(w, x)
    _check_prefill(w, x, out, neff)


@pytest.mark.parametrize("T,Wn", [(6000, 4200), (4700, 4096)])
def test_tc_window_key_moments_all_rows(cuda_ok, T, Wn):
    """A window of at least 4096 keys with a workspace: the raw sums of the key
    tiles every row of a query tile sees in full come from differences of
    key-moment prefixes (the tiles before the window and the diagonal tile
    score by score).  Every row against the oracle; the no-workspace call
    forms the same sums score by score and agrees to rounding."""
    w = W.small_prefill(B=1, T=T, Hq=4, Hkv=2, dtype="bf16", seed=T, plant="frac",
                        plant_frac=0.01, L=1024, window=Wn)
    x = W.prefill_inputs(w, "cpu")
    out, neff = _prefill(w, x)
    _check_prefill(w, x, out, neff)
    out0, neff0 = _prefill(w, x, moments=False)
    assert ((neff - neff0).abs() / neff0).max().item() < 1e-4
    assert (out.float() - out0.float()).abs().max().item() <= 2.0 ** -6


def test_tc_window_running_max_path(cuda_ok):
    """A logit scale too large for the fixed reference takes the running-max
    kernel; its masked tiles honour the window too."""
    w = W.small_prefill(B=1, T=700, Hq=4, Hkv=2, dtype="bf16", seed=3, plant="frac",
                        plant_frac=0.02, s=24.0, L=256, window=200)
    x = W.prefill_inputs(w, "cpu")
    out, neff = _prefill(w, x)
    _check_prefill(w, x, out, neff)


def test_simt_prefill_window_fp32(cuda_ok):
    w = W.small_prefill(B=1, T=300, Hq=4, Hkv=2, dtype="fp32", seed=4, plant="frac",
                        plant_frac=0.02, L=64, window=50)
    x = W.prefill_inputs(w, "cpu")
    out, neff = _prefill(w, x, impl="simt")
    _check_prefill(w, x, out, neff, tol=PT.OUT_TOL_FP32)


def test_window_as_long_as_the_sequence_changes_nothing(cuda_ok):
    w = W.small_prefill(B=1, T=300, Hq=4, Hkv=2, dtype="bf16", seed=5)
    x = W.prefill_inputs(w, "cpu")
    a, na = _prefill(w, x, moments=False)
    for Wn in (300, 5000):
        b, nb = _prefill(dataclasses.replace(w, window=Wn), x, moments=False)
        assert torch.equal(a, b) and torch.equal(na, nb)


def test_extrapolation_T16384_window4096_sampled(cuda_ok):
    """The T=16384 workload with a 4096-key window (32 key tiles per row), the
    configuration the bench's windowed leg times; sampled rows."""
    w = dataclasses.replace(W.EXTRAP, window=4096)
    x = W.prefill_inputs(w, "cuda")
    out, neff = pa.fwd(x["q"], x["k"], x["v"], x["u"], s=w.s, alpha=w.alpha, L=w.L, beta=w.beta,
                       window=w.window)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    rows = PT.sample_rows(w.B, w.Hq, w.T, 400, seed=9)
    ref = PT.oracle_prefill(w, x, rows)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what="window 4096 T=16384")


@pytest.mark.parametrize("Wn", [1, 100, 640, 5000])
@pytest.mark.parametrize("C", [1, 4])
def test_decode_window(cuda_ok, Wn, C):
    """Single- and multi-token decode with a window: each token sees the last W
    positions below its own; splits start at the first visible page."""
    lens = [max(C, 16), 65, 130, 700, 3000, 9000]
    w = W.small_decode(num_seqs=len(lens), min_len=1, max_len=9000, Hq=8, Hkv=2, seed=Wn + C,
                       L=128, plant=2, window=Wn)
    x = PT.to_device(W.decode_inputs(w, "cpu", seqlens=lens))
    q = W.decode_chunk_queries(w, x, C)
    out, neff = pa.decode_paged_chunk(q, x["kv_pages"], x["page_table"], x["seqlens"], x["u"],
                                      s=w.s, alpha=w.alpha, L=w.L, beta=w.beta, window=Wn)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    ref = PT.oracle_decode_chunk(w, x, q)
    D = out.shape[-1]
    rows = np.arange(out.numel() // D)
    o = out.float().cpu().numpy().reshape(-1, D).astype(np.float64)
    n = neff.cpu().numpy().reshape(-1).astype(np.float64)
    PT.compare(o, n, ref, rows, PT.OUT_TOL_BF16, what=f"decode window {Wn} chunk {C}")


def test_decode_window_equals_prefill_last_row(cuda_ok):
    """Windowed decode over a paged copy of a sequence matches the windowed
    prefill's last row."""
    T, Wn = 1000, 300
    wp = W.small_prefill(B=1, T=T, Hq=8, Hkv=2, dtype="bf16", seed=6, plant="frac",
                         plant_frac=0.01, window=Wn)
    x = PT.to_device(W.prefill_inputs(wp, "cpu"))
    out_p, neff_p = pa.fwd(x["q"], x["k"], x["v"], x["u"], window=Wn)
    npg = (T + 63) // 64
    pool = torch.zeros((npg, 2, 2, 64, 64), device="cuda", dtype=torch.bfloat16)
    kk = torch.zeros((npg * 64, 2, 64), device="cuda", dtype=torch.bfloat16)
    vv = torch.zeros_like(kk)
    kk[:T], vv[:T] = x["k"][0], x["v"][0]
    pool[:, 0] = kk.view(npg, 64, 2, 64).transpose(1, 2)
    pool[:, 1] = vv.view(npg, 64, 2, 64).transpose(1, 2)
    pt = torch.arange(npg, device="cuda", dtype=torch.int32)[None].contiguous()
    sl = torch.tensor([T], device="cuda", dtype=torch.int32)
    out_d, neff_d = pa.decode_paged(x["q"][:, T - 1].contiguous(), pool.contiguous(), pt, sl,
                                    x["u"], window=Wn)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    ref = out_p[0, T - 1].float()
    err = (out_d[0].float() - ref).abs().amax() / ref.abs().amax()
    assert err < 2e-2, float(err)
    assert ((neff_d[0] - neff_p[0, :, T - 1]).abs() / neff_p[0, :, T - 1]).amax() < 1e-3


def test_negative_window_is_refused(cuda_ok):
    w = W.small_prefill(B=1, T=100, Hq=4, Hkv=2, dtype="bf16", seed=1)
    xd = PT.to_device(W.prefill_inputs(w, "cpu"))
    with pytest.raises(pa.PolarError) as e:
        pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], window=-1)
    assert e.value.code == 1  # POLAR_ERR_INVALID_ARG
