"""Shared helpers of the GPU parity tests: oracle runs on the exact input bits
and the comparison rules.

Tolerances, as the method's specification fixes them:
  * out: normwise relative error max|gpu - ref| / max|ref| <= 2e-2 per
    (batch, head) slice for bf16 outputs (element-relative error is
    meaningless for content entries near zero); fp32 outputs from the fp32
    path are held to 1e-4.
  * n_eff: elementwise relative error <= 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from polar_attention_b200 import workloads as W

OUT_TOL_BF16 = 2e-2
OUT_TOL_FP32 = 1e-4
NEFF_TOL = 1e-3


def oracle_params(w) -> oracle.Params:
    return oracle.Params(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta, window=getattr(w, "window", 0))


def oracle_prefill(w, x, rows=None):
    h = {k: W.to_host_bits(x[k]) for k in ("q", "k", "v")}
    return oracle.polar_fwd(h["q"], h["k"], h["v"], x["u"].detach().cpu().numpy(), oracle_params(w),
                            rows=rows)


def oracle_decode(w, x, rows=None):
    return oracle.polar_decode(W.to_host_bits(x["q"]), W.to_host_bits(x["kv_pages"]),
                               x["page_table"].cpu().numpy(), x["seqlens"].cpu().numpy(),
                               x["u"].detach().cpu().numpy(), oracle_params(w), rows=rows)


def oracle_decode_chunk(w, x, q, rows=None):
    """Oracle of a multi-token decode: token t of sequence n is a single-token
    decode of its own query with seqlen n_t = seqlens[n] - C + t + 1 over the
    same page table (one virtual sequence per token).  Rows are flat
    ((n*C + t)*Hq + h), matching out.reshape(-1, D)."""
    N, C = q.shape[0], q.shape[1]
    lens = x["seqlens"].cpu().numpy().astype(np.int64)
    vlens = (lens[:, None] - C + np.arange(C)[None, :] + 1).reshape(-1).astype(np.int32)
    vpt = np.repeat(x["page_table"].cpu().numpy(), C, axis=0)
    qv = W.to_host_bits(q.reshape(N * C, q.shape[2], q.shape[3]))
    return oracle.polar_decode(qv, W.to_host_bits(x["kv_pages"]), vpt, vlens,
                               x["u"].detach().cpu().numpy(), oracle_params(w), rows=rows)


def oracle_bwd(w, x, gout):
    """Oracle gradients (dq, dk, dv, du) in fp64 for the upstream gradient gout
    (a CUDA or host tensor shaped like q, any float dtype; widened exactly)."""
    h = {k: W.to_host_bits(x[k]) for k in ("q", "k", "v")}
    g = gout.detach().float().cpu().numpy().astype(np.float64)
    return oracle.polar_bwd(h["q"], h["k"], h["v"], x["u"].detach().cpu().numpy(), g,
                            oracle_params(w))


def gpu_rows_prefill(out, neff, rows, B, T, Hq):
    """Gather flat oracle rows ((b*Hq + h)*T + i) from GPU out [B,T,Hq,D] and
    neff [B,Hq,T]."""
    rows = np.asarray(rows, np.int64)
    i = rows % T
    bh = rows // T
    h = bh % Hq
    b = bh // Hq
    o = out.float().cpu().numpy()[b, i, h].astype(np.float64)
    n = neff.cpu().numpy()[b, h, i].astype(np.float64)
    return o, n, b * Hq + h


def compare(o_gpu, n_gpu, ref, groups, out_tol, neff_tol=NEFF_TOL, what=""):
    """Normwise out error per group (slice) and elementwise n_eff error."""
    o_ref, n_ref = ref.out, ref.neff
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    worst = 0.0
    for gid in np.unique(groups):
        m = groups == gid
        err = np.max(np.abs(o_gpu[m] - o_ref[m])) / np.max(np.abs(o_ref[m]))
        worst = max(worst, err)
    nrel = np.max(np.abs(n_gpu - n_ref) / n_ref)
    cos = np.sum(o_gpu * o_ref, 1) / (np.linalg.norm(o_gpu, axis=1) * np.linalg.norm(o_ref, axis=1))
    msg = f"{what}: out normwise {worst:.3e} (tol {out_tol}), neff rel {nrel:.3e} " \
          f"(tol {neff_tol}), min cos {cos.min():.6f}"
    assert worst <= out_tol, msg
    assert nrel <= neff_tol, msg
    return worst, nrel


def sample_rows(B, Hq, T, n, seed=0, include=()):
    """n seeded flat row indices spread over every (b, h), plus the first and
    last rows and the ragged tail, plus `include`."""
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in include)
    for b in range(B):
        for h in range(Hq):
            base = (b * Hq + h) * T
            rows.update([base, base + T - 1, base + max(0, T - 2)])
    rows.update(int(r) for r in rng.integers(0, B * Hq * T, size=n))
    return np.array(sorted(rows), np.int64)


def to_device(x, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
