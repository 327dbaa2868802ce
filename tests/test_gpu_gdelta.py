"""GPU parity of the memory channel (polar_gdelta_prefill, polar_gdelta_step)
against the fp64 oracle's token-by-token gated-delta recurrence."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import polar_attention_b200 as pa
from polar_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

# Normwise max|gpu - oracle| / max|oracle| per (sequence, head).  The kernels
# compute in fp32 (chunked form: a 64 x 64 triangular solve per chunk and
# state products accumulated over the chunks), so fp32 outputs and the fp32
# state land within ~1e-5; bf16 outputs add their own rounding, 2^-9 of each
# element.
OUT_TOL = {"fp32": 1e-4, "bf16": 6e-3}
STATE_TOL = 1e-4


def _host(x):
    return W.to_host_bits(x)


def _oracle(x, S0=None):
    return oracle.gdelta(_host(x["q"]), _host(x["k"]), _host(x["v"]),
                         x["alpha"].cpu().numpy().astype(np.float64),
                         x["beta"].cpu().numpy().astype(np.float64), S0)


def _normwise(got, ref, axes):
    """max over slices of max|got - ref| / max|ref| (slices: all but `axes`)."""
    err = np.max(np.abs(got - ref), axis=axes)
    scale = np.maximum(np.max(np.abs(ref), axis=axes), 1e-30)
    return float(np.max(err / scale))


def _dev(x):
    return {k: v.cuda().contiguous() for k, v in x.items()}


def _run_prefill(x, state=None, out=None, accumulate=False):
    out, state = pa.gdelta_prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], state=state,
                                   out=out, accumulate=accumulate)
    torch.cuda.synchronize()
    assert pa.get_status() == 0
    return out, state


def _check(out, state, o_ref, S_ref, dtype, what=""):
    o = out.float().cpu().numpy().astype(np.float64)
    e_o = _normwise(o, o_ref, axes=(1, 3))           # per (b, h): over t and d
    e_s = _normwise(state.cpu().numpy().astype(np.float64), S_ref, axes=(2, 3))
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    assert e_o <= OUT_TOL[dtype], f"{what}: output error {e_o:.3e}"
    assert e_s <= STATE_TOL, f"{what}: state error {e_s:.3e}"
    return e_o, e_s


# T: one token, less than a chunk, exactly one, one plus one, several with a
# ragged tail.
@pytest.mark.parametrize("T", [1, 63, 64, 65, 300, 777])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_prefill_all_rows(cuda_ok, T, dtype):
    w = W.small_gdelta(B=2, T=T, H=3, dtype=dtype, seed=T)
    x = W.gdelta_inputs(w)
    out, state = _run_prefill(_dev(x))
    o_ref, S_ref = _oracle(x)
    _check(out, state, o_ref, S_ref, dtype, what=f"T={T} {dtype}")


def test_prefill_from_a_given_state_and_continuation(cuda_ok):
    """S_0 given (not zero): prefill of T1 tokens, then of the next T2 from the
    returned state, equals one prefill of T1 + T2 and the oracle."""
    w = W.small_gdelta(B=2, T=400, H=2, seed=11)
    x = W.gdelta_inputs(w)
    g = torch.Generator().manual_seed(3)
    S0 = 0.2 * torch.randn((2, 2, 64, 64), generator=g)
    o_ref, S_ref = _oracle(x, S0.numpy().astype(np.float64))
    xd = _dev(x)
    out, state = _run_prefill(xd, state=S0.cuda().clone())
    _check(out, state, o_ref, S_ref, "bf16", what="given S_0")
    T1 = 130
    first = {k: v[:, :T1].contiguous() for k, v in xd.items()}
    second = {k: v[:, T1:].contiguous() for k, v in xd.items()}
    oa, sa = _run_prefill(first, state=S0.cuda().clone())
    ob, sb = _run_prefill(second, state=sa)
    _check(torch.cat([oa, ob], dim=1), sb, o_ref, S_ref, "bf16", what="continued")


def test_prefill_accumulates_into_attention_output(cuda_ok):
    """accumulate = 1 adds the memory read to what `out` holds: the attention
    output (content + count) becomes content + count + memory."""
    B, T, H = 1, 300, 4
    wa = W.small_prefill(B=B, T=T, Hq=H, Hkv=2, dtype="bf16", seed=2, plant="frac",
                         plant_frac=0.02)
    xa = W.prefill_inputs(wa, "cuda")
    att, _ = pa.fwd(xa["q"], xa["k"], xa["v"], xa["u"])
    base = att.clone()
    wm = W.small_gdelta(B=B, T=T, H=H, seed=4)
    xm = W.gdelta_inputs(wm)
    out, _ = _run_prefill(_dev(xm), out=att, accumulate=True)
    o_ref, _ = _oracle(xm)
    want = base.double().cpu().numpy() + o_ref
    got = out.double().cpu().numpy()
    err = np.max(np.abs(got - want)) / np.max(np.abs(want))
    assert err < 1e-2, err


def test_prefill_gate_extremes(cuda_ok):
    """alpha = 0 (the memory forgets everything before the write), beta = 0
    (nothing is written), and all-zero query and key rows (normalised to zero)."""
    w = W.small_gdelta(B=1, T=200, H=2, seed=7)
    x = W.gdelta_inputs(w)
    x["alpha"][0, [5, 64, 65, 130], 0] = 0.0
    x["alpha"][0, 100:, 1] = 1.0
    x["beta"][0, [0, 1, 63, 64, 199], :] = 0.0
    x["q"][0, [3, 70], 1] = 0
    x["k"][0, [4, 64], 0] = 0
    out, state = _run_prefill(_dev(x))
    o_ref, S_ref = _oracle(x)
    _check(out, state, o_ref, S_ref, "bf16", what="gate extremes")


def test_prefill_full_size(cuda_ok):
    """B=8, T=2048, H=16 (the configuration the bench times), every output and
    the final states against the oracle."""
    w = W.GD_TRAIN
    x = W.gdelta_inputs(w, "cuda")
    out, state = _run_prefill(x)
    o_ref, S_ref = _oracle(x)
    _check(out, state, o_ref, S_ref, "bf16", what="full size")


def test_prefill_long_sequence_error_stays_bounded(cuda_ok):
    """T = 16384 with long memories (alpha up to 0.9999): the fp32 state error
    does not grow with the number of chunks beyond the tolerance."""
    w = dataclasses.replace(W.small_gdelta(B=1, T=16384, H=2, seed=8), lg_lo=-4.0, lg_hi=-2.0)
    x = W.gdelta_inputs(w, "cuda")
    out, state = _run_prefill(x)
    o_ref, S_ref = _oracle(x)
    _check(out, state, o_ref, S_ref, "bf16", what="T=16384")


@pytest.mark.parametrize("T,given_state", [(3000, True), (2100, False)])
def test_prefill_two_level_scan(cuda_ok, T, given_state):
    """Few (sequence x head) slices and many chunks take the two-level scan:
    each group of chunks gets its map S -> S M + E, the groups' initial states
    follow in sequence, then every group runs with its outputs.  Here 47 and 33
    chunks of one sequence and two heads (5 and 4 groups), a given initial state,
    a ragged last chunk, and the decay gate closed (alpha = 0) at the first
    token of a group and in its middle."""
    w = W.small_gdelta(B=1, T=T, H=2, seed=T)
    x = W.gdelta_inputs(w)
    x["alpha"][0, [640, 650, 1280], 0] = 0.0
    x["beta"][0, 641, 1] = 0.0
    S0 = None
    if given_state:
        g = torch.Generator().manual_seed(5)
        S0 = 0.2 * torch.randn((1, 2, 64, 64), generator=g)
    o_ref, S_ref = _oracle(x, None if S0 is None else S0.numpy().astype(np.float64))
    out, state = _run_prefill(_dev(x), state=None if S0 is None else S0.cuda().clone())
    e = _check(out, state, o_ref, S_ref, "bf16", what=f"two-level T={T}")
    print(f"two-level T={T}: output {e[0]:.2e}, state {e[1]:.2e}")


def _step(x, out=None, accumulate=False):
    o = pa.gdelta_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["state_pool"], x["slots"],
                       out=out, accumulate=accumulate)
    torch.cuda.synchronize()
    return o


def _step_oracle(x, pool0):
    """The oracle on T = 1 from the states in the used slots."""
    slots = x["slots"].cpu().numpy()
    used = slots >= 0
    sl = slots[used]
    sel = torch.from_numpy(used)
    one = {k: x[k].cpu()[sel][:, None].contiguous() for k in ("q", "k", "v", "alpha", "beta")}
    o, S = _oracle(one, pool0[sl].astype(np.float64))
    return used, sl, o[:, 0], S


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_step_in_place(cuda_ok, dtype):
    w = W.GdeltaStepWorkload("t", num_seqs=37, num_slots=50, H=4, dtype=dtype, seed=5)
    x = _dev(W.gdelta_step_inputs(w))
    x["slots"][[3, 20]] = -1  # skipped sequences
    pool0 = x["state_pool"].cpu().numpy().copy()
    out = torch.full_like(x["q"], 7.0)
    out = _step(x, out=out)
    assert pa.get_status() == 0
    used, sl, o_ref, S_ref = _step_oracle(x, pool0)
    o = out.float().cpu().numpy().astype(np.float64)
    assert np.all(o[~used] == 7.0), "a skipped sequence's output was written"
    e_o = _normwise(o[used], o_ref, axes=(2,))
    assert e_o <= OUT_TOL[dtype], e_o
    pool = x["state_pool"].cpu().numpy()
    e_s = _normwise(pool[sl].astype(np.float64), S_ref, axes=(2, 3))
    assert e_s <= 1e-5, e_s
    untouched = np.setdiff1d(np.arange(w.num_slots), sl)
    assert np.array_equal(pool[untouched], pool0[untouched]), "a slot outside the batch changed"


def test_step_accumulate_and_bad_slot(cuda_ok):
    w = W.GdeltaStepWorkload("t", num_seqs=8, num_slots=8, H=2, seed=6)
    x = _dev(W.gdelta_step_inputs(w))
    pool0 = x["state_pool"].cpu().numpy().copy()
    base = torch.randn(x["q"].shape, generator=torch.Generator().manual_seed(1)).to(
        x["q"].dtype).cuda()
    out = _step(x, out=base.clone(), accumulate=True)
    assert pa.get_status() == 0
    used, sl, o_ref, _ = _step_oracle(x, pool0)
    want = base.double().cpu().numpy() + o_ref
    err = np.max(np.abs(out.double().cpu().numpy() - want)) / np.max(np.abs(want))
    assert err < 1e-2, err
    x["slots"][2] = 8  # == num_slots: out of range
    out2 = torch.full_like(x["q"], 3.0)
    _step(x, out=out2)
    assert pa.get_status() == 8  # POLAR_ERR_BAD_SLOT
    assert torch.all(out2[2] == 3.0)


def test_step_continues_prefill(cuda_ok):
    """A prefill of T tokens, then one step with the next token from its final
    state (placed in a pool slot), equals the prefill of T + 1 tokens."""
    T, H = 321, 4
    w = W.small_gdelta(B=1, T=T + 1, H=H, seed=9)
    x = _dev(W.gdelta_inputs(w))
    full, S_full = _run_prefill(x)
    head = {k: v[:, :T].contiguous() for k, v in x.items()}
    _, S = _run_prefill(head)
    pool = torch.zeros((3, H, 64, 64), device="cuda")
    pool[1] = S[0]
    step = {"q": x["q"][:, T].contiguous(), "k": x["k"][:, T].contiguous(),
            "v": x["v"][:, T].contiguous(), "alpha": x["alpha"][:, T].contiguous(),
            "beta": x["beta"][:, T].contiguous(), "state_pool": pool,
            "slots": torch.tensor([1], dtype=torch.int32, device="cuda")}
    o = _step(step)
    assert pa.get_status() == 0
    ref = full[:, T].float()
    err = (o.float() - ref).abs().amax() / ref.abs().amax()
    assert err < 1e-2, float(err)
    e_s = ((pool[1] - S_full[0]).abs().amax() / S_full[0].abs().amax()).item()
    assert e_s < 1e-4, e_s


def test_step_full_size(cuda_ok):
    """1024 sequences x 16 heads over a 1024-slot pool (the bench's step)."""
    w = W.GD_STEP
    x = W.gdelta_step_inputs(w, "cuda")
    pool0 = x["state_pool"].cpu().numpy().copy()
    out = _step(x)
    assert pa.get_status() == 0
    used, sl, o_ref, S_ref = _step_oracle(x, pool0)
    e_o = _normwise(out.float().cpu().numpy().astype(np.float64), o_ref, axes=(2,))
    assert e_o <= OUT_TOL["bf16"], e_o
    e_s = _normwise(x["state_pool"].cpu().numpy()[sl].astype(np.float64), S_ref, axes=(2, 3))
    assert e_s <= 1e-5, e_s


def test_bad_arguments_are_refused(cuda_ok):
    w = W.small_gdelta(B=1, T=64, H=2)
    x = _dev(W.gdelta_inputs(w))
    n0 = pa.launch_count()
    with pytest.raises(pa.PolarError) as e:
        pa.gdelta_prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                          workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == 3  # POLAR_ERR_WORKSPACE
    with pytest.raises(pa.PolarError) as e:
        pa.gdelta_prefill(x["q"][..., 1:].contiguous(), x["k"][..., 1:].contiguous(),
                          x["v"][..., 1:].contiguous(), x["alpha"], x["beta"])
    assert e.value.code == 2  # POLAR_ERR_UNSUPPORTED: head_dim 63
    assert pa.launch_count() == n0
