"""Host-side argument checks of the C ABI (no GPU needed).

Every entry point refuses a bad shape, parameter, flag, pointer alignment or
workspace size on the host, with the documented status code, before it
touches the CUDA runtime; these calls therefore run on a machine without a
GPU.  The pointers passed are never dereferenced (the checks fail first)."""
import ctypes

import pytest

from polar_attention_b200 import native as N

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
A16 = ctypes.c_void_p(0x100000)        # 16-byte aligned, never dereferenced
MIS = ctypes.c_void_p(0x100008)        # 8 mod 16
MIS4 = ctypes.c_void_p(0x100002)       # 2 mod 4


@pytest.fixture(scope="module")
def lib():
    import os
    if not os.path.exists(N.LIB_PATH):
        from polar_attention_b200 import build
        build.build()
    return N.lib()


def _params(**kw):
    p = N.make_params(B=kw.pop("B", 1), T=kw.pop("T", 128), Hq=kw.pop("Hq", 4), Hkv=kw.pop("Hkv", 2))
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def _fwd(lib, p, q=A16, out=A16, ws=None, ws_bytes=0):
    """polar_attn_fwd_ws; without a workspace also polar_attn_fwd, which must
    refuse exactly the same arguments."""
    code = lib.polar_attn_fwd_ws(q, A16, A16, A16, ctypes.byref(p), out, None, ws, ws_bytes, None)
    if ws is None:
        assert lib.polar_attn_fwd(q, A16, A16, A16, ctypes.byref(p), out, None, None) == code
    return code


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 63, UNSUPPORTED),
    ("Hkv", 3, INVALID),               # Hq % Hkv != 0
    ("dtype", 7, INVALID),
    ("logit_scale", 0.0, INVALID),
    ("logit_scale", float("inf"), INVALID),
    ("alpha", -0.1, INVALID),
    ("beta", float("nan"), INVALID),
    ("L_train", 1, INVALID),
    ("window", -1, INVALID),
    ("causal", 0, UNSUPPORTED),
    ("impl", 9, INVALID),
    ("B", -1, INVALID),
    ("T", (1 << 30) // 64 + 1, UNSUPPORTED),
])
def test_prefill_refuses_bad_params(lib, field, value, code):
    p = _params(**{field: value})
    assert _fwd(lib, p) == code
    assert lib.polar_attn_fwd_train(A16, A16, A16, A16, ctypes.byref(p), A16, None, A16, None) == code
    assert _bwd_state(lib, p) == code
    assert lib.polar_attn_fwd_workspace_size(ctypes.byref(p)) == 0
    assert lib.polar_attn_bwd_workspace_size(ctypes.byref(p)) == 0
    assert lib.polar_attn_fwd_state_size(ctypes.byref(p)) == 0


def _bwd_state(lib, p, out=A16, state=A16, ws_bytes=1 << 30):
    return lib.polar_attn_bwd_from_state(A16, A16, A16, A16, out, state, A16, ctypes.byref(p), A16,
                                         A16, A16, A16, A16, ws_bytes, None)


def test_training_pair_checks(lib):
    """polar_attn_fwd_train needs an aligned state buffer; polar_attn_bwd_from_state
    needs out, the state and the backward's workspace; the state is B*Hq*T rows
    of 8 fp32 words."""
    p = _params(B=2, T=300, Hq=4, Hkv=2)
    assert lib.polar_attn_fwd_state_size(ctypes.byref(p)) == 2 * 4 * 300 * 8 * 4
    assert lib.polar_attn_fwd_train(A16, A16, A16, A16, ctypes.byref(p), A16, None, None, None) == INVALID
    assert lib.polar_attn_fwd_train(A16, A16, A16, A16, ctypes.byref(p), A16, None, MIS, None) == INVALID
    assert _bwd_state(lib, p, out=None) == INVALID
    assert _bwd_state(lib, p, out=MIS) == INVALID
    assert _bwd_state(lib, p, state=None) == INVALID
    assert _bwd_state(lib, p, state=MIS) == INVALID
    need = lib.polar_attn_bwd_workspace_size(ctypes.byref(p))
    assert _bwd_state(lib, p, ws_bytes=need - 1) == WORKSPACE
    for shape in ({"B": 0}, {"T": 0}):
        e = _params(**shape)
        assert lib.polar_attn_fwd_train(None, None, None, None, ctypes.byref(e), None, None, None,
                                        None) == OK


def test_prefill_pointer_and_workspace_checks(lib):
    p = _params()
    assert _fwd(lib, p, q=None) == INVALID
    assert _fwd(lib, p, q=MIS) == INVALID
    assert _fwd(lib, p, out=MIS) == INVALID
    assert _fwd(lib, p, ws=MIS, ws_bytes=1 << 30) == INVALID
    big = _params(T=4096)   # needs key-moment records
    need = lib.polar_attn_fwd_workspace_size(ctypes.byref(big))
    assert need > 0
    assert _fwd(lib, big, ws=A16, ws_bytes=need - 1) == WORKSPACE


def test_empty_prefill_is_a_no_op(lib):
    for shape in ({"B": 0}, {"T": 0}):
        assert _fwd(lib, _params(**shape), q=None, out=None) == OK


def _decode(lib, p, num_seqs=2, max_pages=4, chunk=1, ws_bytes=1 << 20, q=A16):
    return lib.polar_attn_decode_paged_chunk(q, A16, 8, A16, max_pages, A16, num_seqs, chunk, A16,
                                             ctypes.byref(p), A16, None, A16, ws_bytes, None)


def test_decode_refuses_bad_shapes(lib):
    assert _decode(lib, _params(dtype=N.POLAR_FP32)) == UNSUPPORTED
    assert _decode(lib, _params(Hq=6, Hkv=2)) == UNSUPPORTED        # group of 3
    assert _decode(lib, _params(Hq=32, Hkv=2)) == UNSUPPORTED       # group of 16
    assert _decode(lib, _params(), max_pages=0) == INVALID
    assert _decode(lib, _params(), num_seqs=-1) == INVALID
    assert _decode(lib, _params(), chunk=0) == INVALID
    assert _decode(lib, _params(Hq=8, Hkv=2), chunk=5) == UNSUPPORTED  # 4 x 5 rows > 16
    assert _decode(lib, _params(), q=MIS) == INVALID
    assert _decode(lib, _params(), ws_bytes=0) == WORKSPACE
    assert _decode(lib, _params(), num_seqs=0) == OK                # nothing to do


def _gd(B=1, T=64, H=2, head_dim=64, dtype=N.POLAR_BF16, zero_init=1, accumulate=0):
    p = N.GdeltaParams(B, T, H, head_dim, dtype, zero_init, accumulate)
    return p


def _gd_prefill(lib, p, q=A16, alpha=A16, state=A16, ws=A16, ws_bytes=1 << 30):
    return lib.polar_gdelta_prefill(q, A16, A16, alpha, A16, state, ctypes.byref(p), A16, ws,
                                    ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    ({"head_dim": 32}, UNSUPPORTED),
    ({"dtype": 3}, INVALID),
    ({"H": 0}, INVALID),
    ({"B": -1}, INVALID),
    ({"T": -5}, INVALID),
    ({"zero_init": 2}, INVALID),
    ({"accumulate": -1}, INVALID),
    ({"B": 4096, "H": 16}, UNSUPPORTED),   # B * H > 65535 (the scan grid's second dimension)
])
def test_memory_prefill_refuses_bad_params(lib, kw, code):
    p = _gd(**kw)
    assert _gd_prefill(lib, p) == code
    assert lib.polar_gdelta_prefill_workspace_size(ctypes.byref(p)) == 0


def test_memory_prefill_pointer_and_workspace_checks(lib):
    p = _gd(B=2, T=300, H=4)
    need = lib.polar_gdelta_prefill_workspace_size(ctypes.byref(p))
    assert need == 2 * 4 * 5 * 49920       # 5 chunks of 64 tokens per (sequence, head)
    assert _gd_prefill(lib, p, q=None) == INVALID
    assert _gd_prefill(lib, p, q=MIS) == INVALID
    assert _gd_prefill(lib, p, state=MIS) == INVALID
    assert _gd_prefill(lib, p, alpha=MIS4) == INVALID
    assert _gd_prefill(lib, p, ws=None) == INVALID
    assert _gd_prefill(lib, p, ws_bytes=need - 1) == WORKSPACE
    assert _gd_prefill(lib, _gd(B=0), q=None, state=None, ws=None) == OK
    assert _gd_prefill(lib, _gd(T=0), q=None, state=None, ws=None) == OK


def _gd_step(lib, p, num_seqs=3, num_slots=8, slots=A16, pool=A16):
    return lib.polar_gdelta_step(A16, A16, A16, A16, A16, pool, num_slots, slots, num_seqs,
                                 ctypes.byref(p), A16, None)


def test_memory_step_checks(lib):
    p = _gd()
    p.B, p.T = -7, -7                      # ignored by the step
    assert _gd_step(lib, p, num_seqs=-1) == INVALID
    assert _gd_step(lib, p, num_slots=-1) == INVALID
    assert _gd_step(lib, p, slots=None) == INVALID
    assert _gd_step(lib, p, slots=MIS4) == INVALID
    assert _gd_step(lib, p, pool=MIS) == INVALID
    assert _gd_step(lib, p, num_seqs=0) == OK
    big = _gd(H=64)
    assert _gd_step(lib, big, num_seqs=(1 << 31) // 64 + 1) == UNSUPPORTED
    assert _gd_step(lib, _gd(head_dim=128)) == UNSUPPORTED


def test_status_strings(lib):
    for code in range(9):
        assert lib.polar_attn_status_string(code).decode() != "unknown status"
    assert "slot" in lib.polar_attn_status_string(8).decode()
    assert lib.polar_attn_status_string(99).decode() == "unknown status"
