"""polar_attn_decode_paged_noalloc: the paged decode for callers that cannot
allocate device memory (for example a serving process whose free device memory
all went to its KV-cache pool at start-up, or a plug-in with no device
allocator of its own), so they cannot pass a workspace.

The entry point runs the same decode with its split scratch in a fixed 16 MiB
device array the library keeps per device.  Its split plan depends only on the
shape, so each call must give the same bits as polar_attn_decode_paged with a
workspace of its own, on calls in a row that leave each other's partial states
behind in the array.  After one set-up call, a call takes no device memory
(checked in a fresh process).  This file is collected last.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import native
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _inputs(seed, seqlens, width=None):
    """Decode inputs; `width` pads the page table to that many columns (never
    read past each sequence's pages), which fixes the partial-state layout."""
    w = W.small_decode(num_seqs=len(seqlens), min_len=1, max_len=max(seqlens), Hq=16, Hkv=4,
                       seed=seed, plant=2)
    x = W.decode_inputs(w, "cpu", seqlens=seqlens)
    if width is not None:
        pt = x["page_table"]
        x["page_table"] = torch.cat(
            [pt, torch.full((pt.shape[0], width - pt.shape[1]), -1, dtype=pt.dtype)], 1).contiguous()
    return w, {k: (v.to("cuda") if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _both(w, x):
    """(noalloc out, neff), (workspace-decode out, neff) on the same inputs."""
    p = dict(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta)
    ref, nref = pa.decode_paged(x["q"], x["kv_pages"], x["page_table"], x["seqlens"], x["u"], **p)
    out = torch.empty_like(x["q"])
    neff = torch.empty((x["q"].shape[0], 16), device="cuda")
    native.decode_paged_noalloc(x["q"], x["kv_pages"], x["page_table"], x["seqlens"], x["u"],
                                out, neff, **p)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    return (out, neff), (ref, nref)


def test_noalloc_matches_workspace_decode_twice(cuda_ok):
    """Two calls in a row on different inputs: each is bit-identical to the
    workspace decode (same kernels, same split plan).  The first case is also
    held to the oracle on every row."""
    cases = [(21, [70000, 1, 4097, 33000, 64, 12345]), (22, [129, 90000, 2, 50000])]
    for n, (seed, lens) in enumerate(cases):
        w, x = _inputs(seed, lens)
        (out, neff), (ref, nref) = _both(w, x)
        assert torch.equal(out, ref) and torch.equal(neff, nref), f"case {n}"
        if n == 0:
            o = PT.oracle_decode(w, x)
            PT.compare(out.float().cpu().numpy().reshape(-1, 64).astype(np.float64),
                       neff.cpu().numpy().reshape(-1).astype(np.float64), o,
                       np.arange(len(lens) * 16), PT.OUT_TOL_BF16, what="noalloc")


def test_noalloc_second_call_reads_only_its_own_partials(cuda_ok):
    """Same number of sequences and page-table width, so both calls lay their
    partial states out in the same slots of the array; the second call's
    sequences are shorter, so each of its merges covers slots that the first
    call also wrote.  Its rows must still be the workspace decode's, bit for
    bit: a merge that read a stale partial would differ."""
    lens_a = [60000, 40000, 65000, 30000]
    lens_b = [3000, 129, 64000, 700]
    for seed, lens in ((31, lens_a), (32, lens_b)):
        w, x = _inputs(seed, lens, width=1024)
        (out, neff), (ref, nref) = _both(w, x)
        assert torch.equal(out, ref) and torch.equal(neff, nref), lens


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_ok):
    """A shape whose scratch would exceed the fixed array is refused up front."""
    N, max_pages = 512, 4096
    need = pa.decode_workspace_size(N, max_pages, 16, 4)
    assert need > native.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((N, 16, 64), device="cuda", dtype=torch.bfloat16)
    kv = torch.zeros((4, 2, 4, 64, 64), device="cuda", dtype=torch.bfloat16)
    pt = torch.zeros((N, max_pages), device="cuda", dtype=torch.int32)
    sl = torch.ones((N,), device="cuda", dtype=torch.int32)
    u = torch.zeros((16, 64), device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(pa.PolarError) as e:
        native.decode_paged_noalloc(q, kv, pt, sl, u, out)
    assert e.value.code == 3  # POLAR_ERR_WORKSPACE


_FRESH = textwrap.dedent("""
    import json, sys, torch
    sys.path.insert(0, sys.argv[1])
    from polar_attention_b200 import native, workloads as W
    w = W.small_decode(num_seqs=6, min_len=1, max_len=70000, Hq=16, Hkv=4, seed=41, plant=2)
    x = {k: (v.cuda() if isinstance(v, torch.Tensor) else v)
         for k, v in W.decode_inputs(w, "cpu").items()}
    out = torch.empty_like(x["q"]); neff = torch.empty((6, 16), device="cuda")
    p = dict(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta)
    torch.cuda.synchronize()
    free = [torch.cuda.mem_get_info()[0]]
    # set-up call: no sequences, same pool and page-table width
    native.decode_paged_noalloc(x["q"][:0], x["kv_pages"], x["page_table"][:0],
                                x["seqlens"][:0], x["u"], out[:0], neff[:0], **p)
    torch.cuda.synchronize(); free.append(torch.cuda.mem_get_info()[0])
    for _ in range(2):
        native.decode_paged_noalloc(x["q"], x["kv_pages"], x["page_table"], x["seqlens"],
                                    x["u"], out, neff, **p)
        torch.cuda.synchronize(); free.append(torch.cuda.mem_get_info()[0])
    print(json.dumps({"free": free, "status": native.get_status(),
                      "finite": bool(torch.isfinite(out.float()).all())}))
""")


def test_noalloc_takes_no_device_memory_after_setup(cuda_ok):
    """In a fresh process: after the set-up call (num_seqs = 0), two full calls
    leave the device's free memory unchanged."""
    r = subprocess.run([sys.executable, "-c", _FRESH, ROOT], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    import json
    res = json.loads(r.stdout.strip().splitlines()[-1])
    free = res["free"]
    assert res["status"] == 0 and res["finite"], res
    assert free[2] == free[1] and free[3] == free[1], free
