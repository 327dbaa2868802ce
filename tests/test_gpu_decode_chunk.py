"""GPU parity of the multi-token paged decode (polar_attn_decode_paged_chunk):
each chunk token against the oracle's single-token decode with its own
visible length, plus the structural properties of the chunked call."""
import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _chunk(w, x, q, **kw):
    out, neff = pa.decode_paged_chunk(q, x["kv_pages"], x["page_table"], x["seqlens"], x["u"],
                                      s=w.s, alpha=w.alpha, L=w.L, beta=w.beta, **kw)
    torch.cuda.synchronize()
    return out, neff


def _check(w, x, q, out, neff, rows=None, what=""):
    ref = PT.oracle_decode_chunk(w, x, q, rows=rows)
    D = out.shape[-1]
    nrows = out.numel() // D
    rows = np.arange(nrows) if rows is None else np.asarray(rows)
    o = out.float().cpu().numpy().reshape(nrows, D)[rows].astype(np.float64)
    n = neff.cpu().numpy().reshape(-1)[rows].astype(np.float64)
    return PT.compare(o, n, ref, rows, PT.OUT_TOL_BF16, what=what or w.name)


# (G, chunk): one row set (G * chunk <= 8) and both halves of the mma tile
# (G * chunk up to 16).
CASES = [(1, 1), (1, 3), (1, 16), (2, 2), (2, 5), (2, 8), (4, 2), (4, 3), (4, 4), (8, 1), (8, 2)]


@pytest.mark.parametrize("G,C", CASES)
def test_small_ragged(cuda_ok, G, C):
    """Ragged lengths whose chunk straddles a page boundary (65, 130), sits at
    the start of a page (64 + C), fills the cache exactly (C) or runs long
    (700); the temperature is active past L=128."""
    lens = [max(C, 16), 65, 130, 64 + C, 700, C]
    w = W.small_decode(num_seqs=len(lens), min_len=1, max_len=700, Hq=2 * G, Hkv=2, seed=G + C,
                       L=128, plant=2)
    x = PT.to_device(W.decode_inputs(w, "cpu", seqlens=lens))
    q = W.decode_chunk_queries(w, x, C)
    out, neff = _chunk(w, x, q)
    assert pa.get_status() == 0
    _check(w, x, q, out, neff, what=f"chunk G={G} C={C}")


def test_many_splits(cuda_ok):
    """Chunks over lengths that span many splits, so that early chunk tokens
    can see nothing of the last split."""
    w = W.small_decode(num_seqs=3, min_len=5000, max_len=40000, Hq=16, Hkv=4, seed=17, plant=3)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    q = W.decode_chunk_queries(w, x, 4)
    out, neff = _chunk(w, x, q)
    assert pa.get_status() == 0
    _check(w, x, q, out, neff, what="chunk many splits")


def test_chunk_of_one_is_decode(cuda_ok):
    """chunk = 1 is the plain decode, bit for bit."""
    w = W.small_decode(num_seqs=4, min_len=100, max_len=5000, Hq=8, Hkv=2, seed=3, plant=2)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    a, na = pa.decode_paged(x["q"], x["kv_pages"], x["page_table"], x["seqlens"], x["u"])
    b, nb = pa.decode_paged_chunk(x["q"][:, None].contiguous(), x["kv_pages"], x["page_table"],
                                  x["seqlens"], x["u"])
    torch.cuda.synchronize()
    assert torch.equal(a, b[:, 0]) and torch.equal(na, nb[:, 0])


def test_each_token_is_a_shorter_decode(cuda_ok):
    """Token t of a chunk equals a single-token decode of the same query with
    seqlen - C + t + 1 over the same cache (within rounding: the split of the
    keys into pages per CTA is the same, so the results agree closely)."""
    C = 4
    w = W.small_decode(num_seqs=3, min_len=200, max_len=3000, Hq=16, Hkv=4, seed=21, plant=2)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    q = W.decode_chunk_queries(w, x, C)
    out, neff = _chunk(w, x, q)
    for t in range(C):
        lens_t = (x["seqlens"] - C + t + 1).int().contiguous()
        o1, n1 = pa.decode_paged(q[:, t].contiguous(), x["kv_pages"], x["page_table"], lens_t,
                                 x["u"], s=w.s, alpha=w.alpha, L=w.L, beta=w.beta)
        torch.cuda.synchronize()
        err = (out[:, t].float() - o1.float()).abs().amax() / o1.float().abs().amax()
        assert err < 1e-2, (t, float(err))
        assert ((neff[:, t] - n1).abs() / n1).amax() < 1e-4


def test_chunk_equals_prefill_tail(cuda_ok):
    """A chunk of the last C tokens over a paged copy of a sequence matches the
    prefill's last C rows (causal within the chunk)."""
    T, C = 1000, 4
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
    pt = torch.arange(npg, device="cuda", dtype=torch.int32)[None].contiguous()
    sl = torch.tensor([T], device="cuda", dtype=torch.int32)
    q = x["q"][:, T - C:].contiguous()  # [1, C, Hq, 64]
    out_d, neff_d = pa.decode_paged_chunk(q, pool.contiguous(), pt, sl, x["u"])
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    ref = out_p[:, T - C:].float()
    err = (out_d.float() - ref).abs().amax() / ref.abs().amax()
    assert err < 2e-2, float(err)
    ne_ref = neff_p[0, :, T - C:].transpose(0, 1)  # [C, Hq]
    assert ((neff_d[0] - ne_ref).abs() / ne_ref).amax() < 1e-3


def test_seqlen_below_chunk_is_reported(cuda_ok):
    """A sequence shorter than the chunk has no room for its queries: the
    device reports POLAR_ERR_BAD_SEQLEN and skips it (its outputs stay as they
    were); the other sequences are computed."""
    C = 4
    w = W.small_decode(num_seqs=3, min_len=1, max_len=300, Hq=8, Hkv=2, seed=4)
    x = PT.to_device(W.decode_inputs(w, "cpu", seqlens=[300, 3, 200]))
    q = W.decode_chunk_queries(w, x, C)
    out = torch.full_like(q, 7.0)
    out, neff = _chunk(w, x, q, out=out)
    assert pa.get_status() == 7  # POLAR_ERR_BAD_SEQLEN
    assert torch.all(out[1] == 7.0)
    good = [0, 2]
    xs = {"kv_pages": x["kv_pages"], "page_table": x["page_table"][good].contiguous(),
          "seqlens": x["seqlens"][good].contiguous(), "u": x["u"]}
    _check(w, xs, q[good], out[good], neff[good], what="chunk with a bad sequence")


def test_oversized_chunk_is_refused(cuda_ok):
    """G * chunk must fit the 16 rows of one mma tile: G=4 with chunk=5 is
    refused on the host with POLAR_ERR_UNSUPPORTED and nothing is launched."""
    w = W.small_decode(num_seqs=2, min_len=100, max_len=200, Hq=8, Hkv=2, seed=1)
    x = PT.to_device(W.decode_inputs(w, "cpu"))
    q = W.decode_chunk_queries(w, x, 5)
    n0 = pa.launch_count()
    with pytest.raises(pa.PolarError) as e:
        pa.decode_paged_chunk(q, x["kv_pages"], x["page_table"], x["seqlens"], x["u"])
    assert e.value.code == 2  # POLAR_ERR_UNSUPPORTED
    assert pa.launch_count() == n0


def test_full_workload_chunk4_sampled(cuda_ok):
    """The 32-sequence 128K-256K workload with 4-token chunks (G=4: all 16 mma
    rows in use), in the launch configuration the bench times: every token and
    head of three sequences against the oracle, which reads a host copy of just
    those sequences' pages."""
    C = 4
    w = W.DECODE
    x = W.decode_inputs(w, "cuda")
    q = W.decode_chunk_queries(w, x, C)
    out, neff = _chunk(w, x, q)
    assert pa.get_status() == 0
    assert torch.isfinite(out.float()).all() and (neff >= 1).all()
    seqs = [0, 13, 31]
    pt = x["page_table"][seqs].cpu()
    sl = x["seqlens"][seqs].cpu()
    used = [int(pt[i, p]) for i in range(len(seqs)) for p in range((int(sl[i]) + 63) // 64)]
    remap = {pg: k for k, pg in enumerate(used)}
    pt2 = torch.full_like(pt, -1)
    for i in range(len(seqs)):
        for p in range((int(sl[i]) + 63) // 64):
            pt2[i, p] = remap[int(pt[i, p])]
    xs = {"kv_pages": x["kv_pages"][torch.tensor(used, device="cuda")], "page_table": pt2,
          "seqlens": sl, "u": x["u"]}
    _check(w, xs, q[seqs], out[seqs], neff[seqs], what="chunk4 full workload")
