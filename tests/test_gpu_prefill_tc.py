"""GPU parity of the tcgen05/TMEM tensor-core prefill against the fp64 oracle."""
import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _run(w, x=None, impl="tc", moments=True):
    x = W.prefill_inputs(w, "cpu") if x is None else x
    xd = PT.to_device(x)
    out, neff = pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], s=w.s, alpha=w.alpha, L=w.L,
                       beta=w.beta, impl=impl, moments=moments)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    return x, out, neff


@pytest.mark.parametrize("T", [1, 77, 128, 129, 300, 1000])
@pytest.mark.parametrize("G", [2, 4, 8])
def test_small_all_rows(cuda_ok, T, G):
    """Every row, ragged T (one partial tile, exact tiles, a tile plus one row),
    GQA groups 2/4/8, temperature active past L=256."""
    w = W.small_prefill(B=2, T=T, Hq=2 * G, Hkv=2, dtype="bf16", seed=T + G, plant="frac",
                        plant_frac=0.02, L=256)
    x, out, neff = _run(w)
    ref = PT.oracle_prefill(w, x)
    rows = np.arange(w.B * w.Hq * w.T)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what=f"tc T={T} G={G}")


@pytest.mark.parametrize("T,G", [(4097, 2), (4500, 4), (4200, 8)])
def test_moment_chunks_all_rows(cuda_ok, T, G):
    """From 32 query tiles on, the null-floor sums over the full key tiles come
    from the key moments, whose records run in chunks of 8 tiles: query tiles
    1-8 read one running record, later ones add the records closing up to
    four chunks; T=4097 ends on a one-row tile, T=4500 on a ragged chunk.
    Every row against the oracle, GQA groups 2/4/8."""
    w = W.small_prefill(B=1, T=T, Hq=2 * G, Hkv=2, dtype="bf16", seed=T + G, plant="frac",
                        plant_frac=0.02, L=512)
    x, out, neff = _run(w)
    ref = PT.oracle_prefill(w, x)
    rows = np.arange(w.B * w.Hq * w.T)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what=f"moment chunks T={T}")


def test_moments_agree_with_in_loop_sums(cuda_ok):
    """The two ways of forming the null-floor sums give the same rows: n_eff
    does not depend on them, and out moves only by their rounding."""
    w = W.small_prefill(B=2, T=4500, Hq=4, Hkv=2, dtype="bf16", seed=5, plant="frac",
                        plant_frac=0.01, L=512)
    x = W.prefill_inputs(w, "cpu")
    _, oa, na = _run(w, x, moments=True)
    _, ob, nb = _run(w, x, moments=False)
    assert ((na - nb).abs() / nb).amax() < 1e-6
    err = (oa.float() - ob.float()).abs().amax() / ob.float().abs().amax()
    assert err < 2e-3


def test_moment_records_are_key_moments(cuda_ok):
    """After a call the workspace holds, per (batch, kv head, full key tile t),
    the Gram sum k k^T and the sum of k over the keys from the start of t's
    chunk of 8 tiles through tile t (fp32, checked against fp64 sums of the
    same bf16 keys)."""
    w = W.small_prefill(B=2, T=4500, Hq=4, Hkv=2, dtype="bf16", seed=8)
    x = W.prefill_inputs(w, "cpu")
    xd = PT.to_device(x)
    nbytes = pa.fwd_workspace_size(w.B, w.T, w.Hq, w.Hkv)
    nrec = (w.T + 127) // 128 - 1
    assert nbytes == w.B * w.Hkv * nrec * 4160 * 4
    ws = torch.empty(nbytes, device="cuda", dtype=torch.uint8)
    pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], workspace=ws, impl="tc")
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    rec = ws.view(torch.float32).view(w.B, w.Hkv, nrec, 4160).double().cpu().numpy()
    k = x["k"].float().double().numpy()  # [B, T, Hkv, 64]
    for b in range(w.B):
        for g in range(w.Hkv):
            for t in range(nrec):
                lo = (t // 8) * 8 * 128
                kk = k[b, lo:(t + 1) * 128, g, :]
                gram = kk.T @ kk
                scale = np.abs(gram).max()
                assert np.abs(rec[b, g, t, :4096].reshape(64, 64) - gram).max() < 1e-5 * scale
                ks = kk.sum(0)
                assert np.abs(rec[b, g, t, 4096:] - ks).max() < 1e-5 * max(1.0, np.abs(ks).max())


def test_workspace_unused_below_32_tiles(cuda_ok):
    """Below 32 query tiles the moments do not pay off: a call with a workspace
    gives bit-identical rows to one without."""
    w = W.small_prefill(B=1, T=3000, Hq=4, Hkv=2, dtype="bf16", seed=6, plant="frac",
                        plant_frac=0.01, L=512)
    x = W.prefill_inputs(w, "cpu")
    _, oa, na = _run(w, x, moments=True)
    _, ob, nb = _run(w, x, moments=False)
    assert torch.equal(oa, ob) and torch.equal(na, nb)


def test_small_workspace_is_rejected(cuda_ok):
    w = W.small_prefill(B=1, T=300, Hq=4, Hkv=2, dtype="bf16", seed=1)
    xd = PT.to_device(W.prefill_inputs(w, "cpu"))
    need = pa.fwd_workspace_size(w.B, w.T, w.Hq, w.Hkv)
    ws = torch.empty(need - 16, device="cuda", dtype=torch.uint8)
    with pytest.raises(pa.PolarError) as e:
        pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], workspace=ws, impl="tc")
    assert e.value.code == 3  # POLAR_ERR_WORKSPACE


def test_matches_cuda_core_kernel(cuda_ok):
    """Tensor-core and CUDA-core kernels agree on the same bf16 inputs."""
    w = W.small_prefill(B=1, T=777, Hq=8, Hkv=2, dtype="bf16", seed=9, plant="frac",
                        plant_frac=0.01, L=128)
    x = W.prefill_inputs(w, "cpu")
    _, o_tc, n_tc = _run(w, x, "tc")
    _, o_si, n_si = _run(w, x, "simt")
    err = (o_tc.float() - o_si.float()).abs().amax() / o_si.float().abs().amax()
    assert err < 2e-2
    assert ((n_tc - n_si).abs() / n_si).amax() < 1e-3


def test_auto_uses_tensor_cores_for_bf16(cuda_ok):
    w = W.small_prefill(B=1, T=300, Hq=4, Hkv=2, dtype="bf16", seed=1)
    x = W.prefill_inputs(w, "cpu")
    _, a, na = _run(w, x, "auto")
    _, b, nb = _run(w, x, "tc")
    assert torch.equal(a, b) and torch.equal(na, nb)


def test_train_length_all_rows(cuda_ok):
    """Training-length workload (B=8, Hq=16, Hkv=4, T=2048, 1% planted keys):
    all 262,144 rows against the oracle."""
    w = W.TRAIN
    x, out, neff = _run(w)
    rows = np.arange(w.B * w.Hq * w.T, dtype=np.int64)
    ref = PT.oracle_prefill(w, x)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what="train_len, all rows")


def test_extrapolation_T16384_all_rows(cuda_ok):
    """Full-size T=16384 workload (temperature active up to tau=1.62), in the
    launch configuration the bench times: all 524,288 rows against the oracle
    (about 40 s of oracle time on 16 host threads)."""
    w = W.EXTRAP
    x, out, neff = _run(w)
    rows = np.arange(w.B * w.Hq * w.T, dtype=np.int64)
    ref = PT.oracle_prefill(w, x)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what="extrapolation_T16384, all rows")


def test_extrapolation_T16384_eight_argument_call(cuda_ok):
    """The same full-size workload through polar_attn_fwd(q, k, v, u, params,
    out, neff_out, stream), which takes no workspace, and through
    polar_attn_fwd_ws: both against the oracle on the same sampled rows.  The
    two calls form the null floor's raw sums in different fp32 orders (score
    by score, or from key moments), so out may differ by that rounding; n_eff
    does not depend on those sums and must agree."""
    w = W.EXTRAP
    x, out, neff = _run(w, moments=False)
    rows = PT.sample_rows(w.B, w.Hq, w.T, 600, seed=12)
    ref = PT.oracle_prefill(w, x, rows)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what="extrapolation_T16384, 8-argument call")
    _, out_ws, neff_ws = _run(w, x, moments=True)
    o, n, grp = PT.gpu_rows_prefill(out_ws, neff_ws, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what="extrapolation_T16384, workspace call")
    assert ((neff - neff_ws).abs() / neff_ws).amax() < 1e-6


def test_long_T65536_sampled(cuda_ok):
    """T=65536 with a 16-key needle per kv head matched by the last 64 queries:
    the needle rows and random rows against the oracle, and the needle rows
    concentrate (n_eff well below the unplanted rows')."""
    w = W.LONG
    x, out, neff = _run(w)
    T, Hq = w.T, w.Hq
    needle = [h * T + i for h in (0, 5, 10, 15) for i in range(T - 64, T, 8)]
    rows = PT.sample_rows(w.B, Hq, T, 200, seed=3, include=needle)
    ref = PT.oracle_prefill(w, x, rows)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, T, Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what="long_T65536")
    nn = neff[0, :, T - 64:].float()
    assert nn.median() < 0.01 * neff[0, :, T // 2:T - 64].float().median()


@pytest.mark.parametrize("T", [300, 1000])
def test_large_logit_scale_uses_running_max(cuda_ok, T):
    """A logit scale whose weights could underflow against the fixed reference
    (s * log2e > 28) takes the running-max kernel; it must match too."""
    w = W.small_prefill(B=1, T=T, Hq=8, Hkv=2, dtype="bf16", seed=T, plant="frac",
                        plant_frac=0.02, s=24.0, L=256)
    x, out, neff = _run(w)
    ref = PT.oracle_prefill(w, x)
    rows = np.arange(w.B * w.Hq * w.T)
    o, n, grp = PT.gpu_rows_prefill(out, neff, rows, w.B, w.T, w.Hq)
    PT.compare(o, n, ref, grp, PT.OUT_TOL_BF16, what=f"running max T={T}")


def test_unnormalised_inputs_are_reported(cuda_ok):
    """q scaled by 3 breaks the L2-normalisation precondition: the fixed-
    reference kernel sees logits past the unit-vector bound and reports
    POLAR_ERR_INVALID_ARG through the status word (no fault, finite output)."""
    w = W.small_prefill(B=1, T=256, Hq=4, Hkv=2, dtype="bf16", seed=2, plant="frac",
                        plant_frac=0.05)
    x = PT.to_device(W.prefill_inputs(w, "cpu"))
    assert pa.get_status() == 0
    out, neff = pa.fwd((x["q"].float() * 3).bfloat16(), x["k"], x["v"], x["u"], impl="tc")
    torch.cuda.synchronize()
    assert pa.get_status() == 1  # POLAR_ERR_INVALID_ARG
    assert pa.get_status() == 0


@pytest.mark.parametrize("T,Wn", [(300, 0), (4500, 0), (4500, 700), (8192, 0), (8192, 1500),
                                   (8192, 4200)])
def test_host_buffers_match_device_buffers(cuda_ok, T, Wn):
    """polar_attn_fwd_host runs the prefill batch by batch: a batch's keys and
    values first (and its key moments), then its queries in row segments from
    the last rows to the first, on two compute streams (T=4500: rows 3456-4499,
    2304-3455, 1152-2303, 512-1151, 0-511; T=8192: 6144-8191, 4096-6143,
    2048-4095, 1024-2047, 0-1023; T=300: one segment).  With three batches, on
    the key-moment path (T=4500, 8192), below it, with a window and with a
    window long enough for key moments (W=4200), its rows equal the
    device-buffer call's bit for bit: a row depends on neither the other
    batches nor the split."""
    w = W.small_prefill(B=3, T=T, Hq=8, Hkv=2, dtype="bf16", seed=T, plant="frac",
                        plant_frac=0.01, L=512, window=Wn)
    x = W.prefill_inputs(w, "cpu")
    xd = PT.to_device(x)
    p = dict(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta, window=w.window)
    ref, nref = pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], **p)
    pin = lambda t: t.contiguous().pin_memory()  # noqa: E731
    ho = torch.empty_like(x["q"]).pin_memory()
    hn = torch.empty((w.B, w.Hq, w.T)).pin_memory()
    stg = torch.empty(pa.fwd_staging_size(w.B, w.T, w.Hq, w.Hkv), device="cuda", dtype=torch.uint8)
    pa.fwd_host(pin(x["q"]), pin(x["k"]), pin(x["v"]), pin(x["u"]), ho, hn, stg, **p)
    assert pa.get_status() == 0
    assert torch.equal(ho, ref.cpu()) and torch.equal(hn, nref.cpu())
