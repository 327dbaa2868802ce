"""GPU parity of the training pair: polar_attn_fwd_train (the forward that also
saves each row's streaming state) and polar_attn_bwd_from_state (the backward
that starts from that state), against the fp64 oracle's gradients, plus the
saved state itself against quantities that fix it: n_eff = l^2/l2, the max
raw dot and its first key, and the plain forward's output."""
import dataclasses

import numpy as np
import pytest
import torch

import parity as PT
import polar_attention_b200 as pa
from polar_attention_b200 import workloads as W
from test_gpu_backward import GRAD_FLOOR, GRAD_TOL, _check, _gout

pytestmark = pytest.mark.gpu


def _kw(w):
    return dict(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta, window=w.window)


def _train_pair(w, x, gout, state_fill=None):
    xd = PT.to_device(x)
    state = None
    if state_fill is not None:
        state = torch.full((w.B, w.Hq, w.T, 8), state_fill, device="cuda", dtype=torch.float32)
    out, neff, state = pa.fwd_train(xd["q"], xd["k"], xd["v"], xd["u"], state=state, **_kw(w))
    grads = pa.bwd_from_state(xd["q"], xd["k"], xd["v"], xd["u"], out, state,
                              gout.cuda().contiguous(), **_kw(w))
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    return xd, out, neff, state, tuple(g.cpu().numpy() for g in grads)


def _compare_grads(w, got, x, gout, what=""):
    ref = PT.oracle_bwd(w, x, gout)
    for name, g, r in zip(("dq", "dk", "dv", "du"), got, ref):
        _check(f"{name} {what} T={w.T} window={w.window}", g, r, GRAD_TOL[w.dtype],
               GRAD_FLOOR[w.dtype])


def _check_state(w, xd, out, neff, state):
    """The saved state against what fixes it on its own."""
    st = state.cpu()
    l, l2, mx, s1, s2, an = (st[..., i] for i in range(6))
    arg = st[..., 6].contiguous().view(torch.int32)
    assert torch.all(torch.isfinite(st[..., :6])), "non-finite saved state"
    assert torch.all(st[..., 7] == 0)
    # n_eff = l^2 / l2, clamped to [1, n]: the same fp32 arithmetic as the epilogue.
    n = torch.arange(1, w.T + 1, dtype=torch.float32)
    if w.window > 0:
        n = torch.clamp(n, max=float(w.window))
    ne = torch.minimum(torch.clamp(l * l / l2, min=1.0), n)
    assert torch.equal(ne, neff.cpu()), "saved l, l2 do not give the output n_eff"
    # The max raw dot and its first key, from fp64 dots of the same bf16 inputs.
    G = w.Hq // w.Hkv
    q = xd["q"].double().cpu()
    k = xd["k"].double().cpu()
    rows = torch.arange(w.T)
    for b in range(w.B):
        for h in range(w.Hq):
            dots = q[b, :, h] @ k[b, :, h // G].T  # [T, T]
            lo = (rows - w.window + 1).clamp(min=0) if w.window > 0 else torch.zeros_like(rows)
            cols = torch.arange(w.T)[None, :]
            vis = (cols <= rows[:, None]) & (cols >= lo[:, None])
            dots = dots.masked_fill(~vis, -np.inf)
            m_ref = dots.max(dim=1).values
            # fp32 sums of exact bf16 products on the tensor cores.
            assert torch.allclose(mx[b, h].double(), m_ref, atol=1e-5), "max raw dot"
            a = arg[b, h].long()
            assert torch.all((a >= lo) & (a <= rows)), "argmax key outside the visible range"
            at = dots[rows, a]
            assert torch.allclose(at, m_ref, atol=1e-5), "saved argmax key does not hold the max"
            # |acc| is a norm of a weighted sum of unit-ish vectors: positive and finite.
            assert torch.all(an[b, h] > 0)


CASES = [(1, 2, 0), (77, 2, 0), (300, 4, 0), (300, 2, 64), (500, 8, 0)]


@pytest.mark.parametrize("T,G,Wn", CASES)
def test_small_vs_oracle(cuda_ok, T, G, Wn):
    """One key, ragged lengths, GQA groups 2/4/8 and a window; the count vector
    is large enough that the magnitude channel's gradient matters."""
    w = W.small_prefill(B=2, T=T, Hq=2 * G, Hkv=2, dtype="bf16", seed=T + G, plant="frac",
                        plant_frac=0.02, L=32, window=Wn)
    x = W.prefill_inputs(w, "cpu")
    x["u"] = x["u"] * 25.0
    gout = _gout(w, T)
    xd, out, neff, state, got = _train_pair(w, x, gout)
    _check_state(w, xd, out, neff, state)
    _compare_grads(w, got, x, gout, "from state")


def test_forward_output_equals_plain_forward(cuda_ok):
    """Below the key-moment threshold the training forward runs the plain
    forward's sweep (plus the argmax search), so out and n_eff are the same
    bits."""
    for wn in (0, 300):
        w = W.small_prefill(B=2, T=1500, Hq=8, Hkv=2, dtype="bf16", seed=31, plant="frac",
                            plant_frac=0.01, L=512, window=wn)
        xd = PT.to_device(W.prefill_inputs(w, "cpu"))
        o1, n1 = pa.fwd(xd["q"], xd["k"], xd["v"], xd["u"], **_kw(w))
        o2, n2, _ = pa.fwd_train(xd["q"], xd["k"], xd["v"], xd["u"], **_kw(w))
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(n1, n2), f"window {wn}"


def test_multi_tile_gqa4_ragged(cuda_ok):
    w = W.small_prefill(B=2, T=1500, Hq=8, Hkv=2, dtype="bf16", seed=15, plant="frac",
                        plant_frac=0.01, L=512)
    x = W.prefill_inputs(w, "cpu")
    x["u"] = x["u"] * 25.0
    gout = _gout(w, 7)
    xd, out, neff, state, got = _train_pair(w, x, gout)
    _check_state(w, xd, out, neff, state)
    _compare_grads(w, got, x, gout, "from state")


def test_window_multi_tile(cuda_ok):
    w = W.small_prefill(B=1, T=900, Hq=4, Hkv=2, dtype="bf16", seed=16, plant="frac",
                        plant_frac=0.01, L=64, window=200)
    x = W.prefill_inputs(w, "cpu")
    x["u"] = x["u"] * 25.0
    gout = _gout(w, 8)
    xd, out, neff, state, got = _train_pair(w, x, gout)
    _check_state(w, xd, out, neff, state)
    _compare_grads(w, got, x, gout, "from state")


def test_tied_max_takes_the_first_key(cuda_ok):
    """Every key appears twice (positions 2m and 2m+1): the saved argmax must be
    the even one of each tied pair, and dk must match the oracle's split."""
    w = W.small_prefill(B=1, T=600, Hq=4, Hkv=2, dtype="bf16", seed=17, plant="frac",
                        plant_frac=0.02, L=128)
    x = W.prefill_inputs(w, "cpu")
    x["k"][:, 1::2] = x["k"][:, 0::2]
    x["v"][:, 1::2] = x["v"][:, 0::2]
    x["u"] = x["u"] * 25.0
    gout = _gout(w, 9)
    xd, out, neff, state, got = _train_pair(w, x, gout)
    _check_state(w, xd, out, neff, state)
    arg = state.cpu()[..., 6].contiguous().view(torch.int32)
    # Key 2m is visible wherever its twin 2m + 1 is, so the first key holding
    # a row's max is always the even copy.
    assert torch.all(arg % 2 == 0), "tie resolved to the later copy"
    _compare_grads(w, got, x, gout, "from state")


@pytest.mark.parametrize("what", ["odd_group", "fp32", "large_scale"])
def test_no_state_path_recomputes(cuda_ok, what):
    """Where the state path does not apply (odd group size, fp32 inputs, a logit
    scale past the fixed reference), the training forward saves nothing -- the
    state keeps its sentinel -- and the backward recomputes the rows."""
    if what == "odd_group":
        w = W.small_prefill(B=1, T=400, Hq=3, Hkv=1, dtype="bf16", seed=41, plant="frac",
                            plant_frac=0.02, L=64)
    elif what == "fp32":
        w = W.small_prefill(B=1, T=200, Hq=4, Hkv=2, dtype="fp32", seed=42, plant="frac",
                            plant_frac=0.02, L=64)
    else:
        w = W.small_prefill(B=1, T=400, Hq=4, Hkv=2, dtype="bf16", seed=43, plant="frac",
                            plant_frac=0.02, L=64)
        w = dataclasses.replace(w, s=25.0)
    x = W.prefill_inputs(w, "cpu")
    x["u"] = x["u"] * 25.0
    gout = _gout(w, 11)
    xd, out, neff, state, got = _train_pair(w, x, gout, state_fill=-7.0)
    assert torch.all(state == -7.0), "state written where the state path does not apply"
    _compare_grads(w, got, x, gout, f"no state ({what})")


def test_train_length_full_size_batch0(cuda_ok):
    """The bench's training launch (B=8, T=2048, Hq=16, Hkv=4, bf16): the whole
    pair runs on the GPU; batch 0's gradients are checked against the oracle
    on batch 0 alone, and every gradient against the recomputing backward."""
    w = W.TRAIN
    x = W.prefill_inputs(w, "cpu")
    gout = _gout(w, 21)
    xd, out, neff, state, got = _train_pair(w, x, gout)
    x0 = {k: (v[:1] if k in ("q", "k", "v") else v) for k, v in x.items()}
    w0 = dataclasses.replace(w, B=1)
    ref = PT.oracle_bwd(w0, x0, gout[:1])
    for name, g, r in zip(("dq", "dk", "dv"), (got[0][:1], got[1][:1], got[2][:1]), ref[:3]):
        _check(f"{name} from state, full-size batch 0", g, r, GRAD_TOL["bf16"], GRAD_FLOOR["bf16"])
    rec = pa.bwd(xd["q"], xd["k"], xd["v"], xd["u"], gout.cuda().contiguous(), **_kw(w))
    torch.cuda.synchronize()
    for name, g, r in zip(("dq", "dk", "dv", "du"), got, rec):
        _check(f"{name} from state vs recomputed", g, r.cpu().numpy(), GRAD_TOL["bf16"],
               GRAD_FLOOR["bf16"])


def test_deterministic(cuda_ok):
    w = W.small_prefill(B=1, T=700, Hq=4, Hkv=2, dtype="bf16", seed=4, plant="frac",
                        plant_frac=0.02)
    x = W.prefill_inputs(w, "cpu")
    gout = _gout(w, 1)
    a = _train_pair(w, x, gout)[4]
    b = _train_pair(w, x, gout)[4]
    for ga, gb in zip(a, b):
        assert np.array_equal(ga, gb)


def test_empty_sequence_zeroes_du(cuda_ok):
    u = torch.ones((4, 64), device="cuda")
    e = torch.empty((1, 0, 4, 64), device="cuda", dtype=torch.bfloat16)
    ek = torch.empty((1, 0, 2, 64), device="cuda", dtype=torch.bfloat16)
    st = torch.empty((1, 4, 0, 8), device="cuda")
    pa.fwd_train(e, ek, ek, u, out=e, state=st)
    du = torch.full((4, 64), 3.0, device="cuda")
    pa.bwd_from_state(e, ek, ek, u, e, st, e, du=du)
    torch.cuda.synchronize()
    assert torch.all(du == 0)
