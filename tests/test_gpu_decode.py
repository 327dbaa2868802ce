"""GPU parity of the GQA paged decode (split + merge kernels) against the oracle."""
import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _decode(w, x, **kw):
    out, neff = pa.decode_paged(x["q"], x["kv_pages"], x["page_table"], x["seqlens"], x["u"],
                                s=w.s, alpha=w.alpha, L=w.L, beta=w.beta, **kw)
    torch.cuda.synchronize()
    return out, neff


def _check(w, x, out, neff, rows=None):
    ref = PT.oracle_decode(w, x, rows=rows)
    N, Hq = out.shape[0], out.shape[1]
    rows = np.arange(N * Hq) if rows is None else np.asarray(rows)
    o = out.float().cpu().numpy().reshape(N * Hq, -1)[rows].astype(np.float64)
    n = neff.cpu().numpy().reshape(-1)[rows].astype(np.float64)
    return PT.compare(o, n, ref, rows, PT.OUT_TOL_BF16, what=w.name)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_small_ragged(cuda_ok, G):
    """Sequence lengths from 1 to a few pages (ragged last page), GQA groups 1-8."""
    w = W.small_decode(num_seqs=5, min_len=1, max_len=700, Hq=2 * G, Hkv=2, seed=G, L=128, plant=2)
    x = PT.to_device(W.decode_inputs(w, "cpu", seqlens=[1, 63, 64, 65, 700]))
    out, neff = _decode(w, x)
    assert pa.get_status() == 0
    _check(w, x, out, neff)


def test_many_splits(cuda_ok):
    """Lengths that span many splits (merge across splits) with the temperature active."""
    w = W.small_decode(num_seqs=3, min_len=5000, max_len=40000, Hq=16, Hkv=4, seed=7, plant=3)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    out, neff = _decode(w, x)
    assert pa.get_status() == 0
    _check(w, x, out, neff)


def test_page_permutation_is_bitwise_invariant(cuda_ok):
    w = W.small_decode(num_seqs=2, min_len=3000, max_len=9000, Hq=8, Hkv=2, seed=11)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    a, na = _decode(w, x)
    P = x["kv_pages"].shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(0)).to("cuda")
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(P, device="cuda")
    kv2 = x["kv_pages"][perm].contiguous()          # physical page p moves to inv[p]
    pt2 = torch.where(x["page_table"] >= 0, inv[x["page_table"].clamp(min=0).long()].int(),
                      x["page_table"])
    x2 = dict(x, kv_pages=kv2, page_table=pt2.contiguous())
    b, nb = _decode(w, x2)
    assert torch.equal(a, b) and torch.equal(na, nb)


def test_decode_equals_prefill_last_row(cuda_ok):
    """Decode over a paged copy of a sequence matches the CUDA-core prefill's
    last row (both within tolerance of the oracle, and of each other)."""
    T = 1000
    wp = W.small_prefill(B=1, T=T, Hq=8, Hkv=2, dtype="bf16", seed=5, plant="frac", plant_frac=0.01)
    x = PT.to_device(W.prefill_inputs(wp, "cpu"))
    out_p, neff_p = pa.fwd(x["q"], x["k"], x["v"], x["u"], impl="simt")
    npg = (T + 63) // 64
    pool = torch.zeros((npg, 2, 2, 64, 64), device="cuda", dtype=torch.bfloat16)
    kk = torch.zeros((npg * 64, 2, 64), device="cuda", dtype=torch.bfloat16)
    vv = torch.zeros_like(kk)
    kk[:T], vv[:T] = x["k"][0], x["v"][0]
    pool[:, 0] = kk.view(npg, 64, 2, 64).transpose(1, 2)
    pool[:, 1] = vv.view(npg, 64, 2, 64).transpose(1, 2)
    perm = torch.randperm(npg, generator=torch.Generator().manual_seed(1))
    pool_s = torch.empty_like(pool)
    pool_s[perm.to("cuda")] = pool
    pt = perm.int().view(1, npg).to("cuda")
    sl = torch.tensor([T], dtype=torch.int32, device="cuda")
    q = x["q"][0, T - 1].unsqueeze(0).contiguous()
    out_d, neff_d = pa.decode_paged(q, pool_s, pt, sl, x["u"])
    torch.cuda.synchronize()
    o_p = out_p[0, T - 1].float()
    o_d = out_d[0].float()
    assert (o_p - o_d).abs().max() / o_p.abs().max() < 2e-2
    assert ((neff_p[0, :, T - 1] - neff_d[0]).abs() / neff_p[0, :, T - 1]).max() < 1e-3


def test_bad_page_is_reported_not_trapped(cuda_ok):
    """A page id outside the pool is caught by the kernel's range check: the
    status word reports it, the page is skipped, and the context stays usable."""
    w = W.small_decode(num_seqs=2, min_len=500, max_len=600, Hq=8, Hkv=2, seed=3)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    assert pa.get_status() == 0
    pt = x["page_table"].clone()
    pt[1, 2] = x["kv_pages"].shape[0] + 5
    _decode(w, dict(x, page_table=pt))
    assert pa.get_status() == 4  # POLAR_ERR_BAD_PAGE
    assert pa.get_status() == 0  # cleared
    out, neff = _decode(w, x)    # still usable
    assert pa.get_status() == 0
    _check(w, x, out, neff)


def test_bad_seqlen_is_reported(cuda_ok):
    w = W.small_decode(num_seqs=2, min_len=100, max_len=200, Hq=8, Hkv=2, seed=4)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    sl = x["seqlens"].clone()
    sl[0] = x["page_table"].shape[1] * 64 + 1
    _decode(w, dict(x, seqlens=sl))
    assert pa.get_status() == 7  # POLAR_ERR_BAD_SEQLEN


def test_host_buffers_match_device_buffers(cuda_ok):
    w = W.small_decode(num_seqs=4, min_len=100, max_len=3000, Hq=16, Hkv=4, seed=8)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    a, na = _decode(w, x)
    N, Hq = a.shape[0], a.shape[1]
    st = torch.empty(pa.decode_staging_size(N, x["page_table"].shape[1], Hq, 4), device="cuda",
                     dtype=torch.uint8)
    oh = torch.empty((N, Hq, 64), dtype=torch.bfloat16).pin_memory()
    nh = torch.empty((N, Hq), dtype=torch.float32).pin_memory()
    pa.decode_paged_host(x["q"].cpu().pin_memory(), x["kv_pages"], x["page_table"].cpu().pin_memory(),
                         x["seqlens"].cpu().pin_memory(), x["u"].cpu().pin_memory(), oh, nh, st)
    assert torch.equal(oh, a.cpu()) and torch.equal(nh, na.cpu())


def test_full_workload_every_sequence(cuda_ok):
    """The 32-sequence, 128K-256K-context pool (6.6 GB, shuffled pages) in the
    launch configuration the bench times: every head of every sequence against
    the oracle, eight sequences at a time, each group's oracle reading a host
    copy of just that group's pages."""
    w = W.DECODE
    x = W.decode_inputs(w, "cuda")
    out, neff = _decode(w, x)
    assert pa.get_status() == 0
    assert torch.isfinite(out.float()).all() and (neff >= 1).all()
    for g0 in range(0, w.num_seqs, 8):
        seqs = list(range(g0, min(g0 + 8, w.num_seqs)))
        pt = x["page_table"][seqs].cpu()
        sl = x["seqlens"][seqs].cpu()
        used = [int(pt[i, p]) for i in range(len(seqs)) for p in range((int(sl[i]) + 63) // 64)]
        remap = {pg: k for k, pg in enumerate(used)}
        sub = x["kv_pages"][torch.tensor(used, device="cuda")]
        pt2 = torch.full_like(pt, -1)
        for i in range(len(seqs)):
            for p in range((int(sl[i]) + 63) // 64):
                pt2[i, p] = remap[int(pt[i, p])]
        xs = {"q": x["q"][seqs], "kv_pages": sub, "page_table": pt2, "seqlens": sl, "u": x["u"]}
        ref = PT.oracle_decode(w, xs)
        o = out[seqs].float().cpu().numpy().reshape(len(seqs) * w.Hq, -1).astype(np.float64)
        n = neff[seqs].cpu().numpy().reshape(-1).astype(np.float64)
        PT.compare(o, n, ref, np.arange(len(seqs) * w.Hq), PT.OUT_TOL_BF16,
                   what=f"decode full, sequences {seqs[0]}-{seqs[-1]}")
        del sub, xs, ref


def test_per_head_variant_reads_the_same_pages(cuda_ok):
    """The test-only per-head decode (one query head per CTA, each page read
    once per query head) gives the grouped decode's rows bit for bit: the mma
    rows of a group are independent, and the merge is the same."""
    from polar_attention_b200 import native
    w = W.small_decode(num_seqs=5, min_len=1, max_len=40000, Hq=16, Hkv=4, seed=33, plant=2)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    p = dict(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta)
    a, na = pa.decode_paged(x["q"], x["kv_pages"], x["page_table"], x["seqlens"], x["u"], **p)
    b, nb = native.selftest_decode_per_head(x["q"], x["kv_pages"], x["page_table"],
                                            x["seqlens"], x["u"], **p)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    assert torch.equal(a, b) and torch.equal(na, nb)
