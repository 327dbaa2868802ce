"""polar_attn_decode_paged_noalloc: the paged decode for callers that cannot
allocate device memory (for example a serving process whose free device memory
all went to its KV-cache pool at start-up, or a plug-in with no device
allocator of its own), so they cannot pass a workspace.

The entry point runs the same decode with its split scratch in a fixed 16 MiB
device array the library keeps per device.  Two calls in a row, on different
inputs (so the second call finds the first call's leftovers in the array), must
each agree with polar_attn_decode_paged given a workspace of its own, within
the tolerance of the other parity tests.  This file is collected last.
"""
import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import native
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _inputs(seed, seqlens):
    w = W.small_decode(num_seqs=len(seqlens), min_len=1, max_len=max(seqlens), Hq=16, Hkv=4,
                       seed=seed, plant=2)
    x = W.decode_inputs(w, "cpu", seqlens=seqlens)
    return w, {k: (v.to("cuda") if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _close(a, na, b, nb):
    a, b = a.float().cpu().numpy(), b.float().cpu().numpy()
    err = np.abs(a - b).max() / np.abs(b).max()
    nrel = (np.abs(na.cpu().numpy() - nb.cpu().numpy()) / nb.cpu().numpy()).max()
    assert err <= PT.OUT_TOL_BF16 and nrel <= PT.NEFF_TOL, (err, nrel)


def test_noalloc_matches_workspace_decode_twice(cuda_ok):
    cases = [(21, [70000, 1, 4097, 33000, 64, 12345]), (22, [129, 90000, 2, 50000])]
    for seed, lens in cases:
        w, x = _inputs(seed, lens)
        p = dict(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta)
        ref, nref = pa.decode_paged(x["q"], x["kv_pages"], x["page_table"], x["seqlens"], x["u"], **p)
        out = torch.empty_like(x["q"])
        neff = torch.empty((len(lens), 16), device="cuda")
        native.decode_paged_noalloc(x["q"], x["kv_pages"], x["page_table"], x["seqlens"], x["u"],
                                    out, neff, **p)
        torch.cuda.synchronize()
        assert pa.get_status() == 0
        _close(out, neff, ref, nref)


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
