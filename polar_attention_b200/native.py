"""ctypes binding of libpolar_attn.so, the C ABI of include/polar_attn.h and
include/polar_gdelta.h.

Argument marshalling only: torch tensors supply device memory and streams, and
every step of the computation runs in the library's CUDA kernels.  There is no
CPU or PyTorch fallback; a missing or unloadable library raises at once.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpolar_attn.so")

POLAR_BF16, POLAR_FP32 = 0, 1
IMPLS = {"auto": 0, "simt": 1, "tc": 2}
STATUS = {0: "POLAR_OK", 1: "POLAR_ERR_INVALID_ARG", 2: "POLAR_ERR_UNSUPPORTED",
          3: "POLAR_ERR_WORKSPACE", 4: "POLAR_ERR_BAD_PAGE", 5: "POLAR_ERR_TIMEOUT",
          6: "POLAR_ERR_CUDA", 7: "POLAR_ERR_BAD_SEQLEN", 8: "POLAR_ERR_BAD_SLOT"}

# Every entry point include/polar_attn.h and include/polar_gdelta.h declare.
EXPORTS = ["polar_attn_default_params", "polar_attn_fwd_workspace_size", "polar_attn_fwd",
           "polar_attn_fwd_ws",
           "polar_attn_fwd_staging_size",
           "polar_attn_fwd_host", "polar_attn_decode_workspace_size", "polar_attn_decode_paged",
           "polar_attn_decode_staging_size", "polar_attn_decode_paged_host",
           "polar_attn_get_status", "polar_attn_status_string", "polar_attn_launch_count",
           "polar_attn_decode_paged_noalloc", "polar_attn_selftest_exp2",
           "polar_attn_decode_chunk_workspace_size", "polar_attn_decode_paged_chunk",
           "polar_attn_bwd_workspace_size", "polar_attn_bwd",
           "polar_gdelta_prefill_workspace_size", "polar_gdelta_prefill", "polar_gdelta_step",
           "polar_attn_selftest_timeout", "polar_attn_selftest_decode_per_head",
           "polar_attn_fwd_state_size", "polar_attn_fwd_train", "polar_attn_bwd_from_state",
           "polar_attn_selftest_fwd_host_segments"]


class PolarError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({status_string(code)})")


class Params(ctypes.Structure):
    """polar_params_t."""
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int),
                ("Hkv", ctypes.c_int), ("head_dim", ctypes.c_int), ("dtype", ctypes.c_int),
                ("logit_scale", ctypes.c_float), ("alpha", ctypes.c_float),
                ("L_train", ctypes.c_int), ("beta", ctypes.c_float), ("causal", ctypes.c_int),
                ("impl", ctypes.c_int), ("window", ctypes.c_int)]


class GdeltaParams(ctypes.Structure):
    """polar_gdelta_params_t."""
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("dtype", ctypes.c_int), ("zero_init", ctypes.c_int),
                ("accumulate", ctypes.c_int)]


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Loads libpolar_attn.so (build it with ``python -m polar_attention_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build the CUDA library with "
                                   "`python -m polar_attention_b200.build` (no fallback exists)")
            L = ctypes.CDLL(LIB_PATH)
            P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            PP = ctypes.POINTER(Params)
            L.polar_attn_default_params.argtypes = [PP, I, I, I, I, I]
            L.polar_attn_default_params.restype = None
            L.polar_attn_fwd_workspace_size.argtypes = [PP]
            L.polar_attn_fwd_workspace_size.restype = Z
            L.polar_attn_fwd.argtypes = [P, P, P, P, PP, P, P, P]
            L.polar_attn_fwd_ws.argtypes = [P, P, P, P, PP, P, P, P, Z, P]
            L.polar_attn_bwd_workspace_size.argtypes = [PP]
            L.polar_attn_bwd_workspace_size.restype = Z
            L.polar_attn_bwd.argtypes = [P, P, P, P, P, PP, P, P, P, P, P, Z, P]
            L.polar_attn_fwd_state_size.argtypes = [PP]
            L.polar_attn_fwd_state_size.restype = Z
            L.polar_attn_fwd_train.argtypes = [P, P, P, P, PP, P, P, P, P]
            L.polar_attn_bwd_from_state.argtypes = [P, P, P, P, P, P, P, PP, P, P, P, P, P, Z, P]
            L.polar_attn_fwd_staging_size.argtypes = [PP]
            L.polar_attn_fwd_staging_size.restype = Z
            L.polar_attn_fwd_host.argtypes = [P, P, P, P, PP, P, P, P, Z, P]
            L.polar_attn_decode_workspace_size.argtypes = [I, I, PP]
            L.polar_attn_decode_workspace_size.restype = Z
            L.polar_attn_decode_paged.argtypes = [P, P, I, P, I, P, I, P, PP, P, P, P, Z, P]
            L.polar_attn_decode_chunk_workspace_size.argtypes = [I, I, I, PP]
            L.polar_attn_decode_chunk_workspace_size.restype = Z
            L.polar_attn_decode_paged_chunk.argtypes = [P, P, I, P, I, P, I, I, P, PP, P, P, P, Z, P]
            L.polar_attn_decode_staging_size.argtypes = [I, I, PP]
            L.polar_attn_decode_staging_size.restype = Z
            L.polar_attn_decode_paged_host.argtypes = [P, P, I, P, I, P, I, P, PP, P, P, P, Z, P]
            L.polar_attn_decode_paged_noalloc.argtypes = [P, P, I, P, I, P, I, P, PP, P, P, P]
            L.polar_attn_selftest_exp2.argtypes = [P, P, P, I, P]
            L.polar_attn_selftest_timeout.argtypes = [P]
            L.polar_attn_selftest_decode_per_head.argtypes = [P, P, I, P, I, P, I, P, PP, P, P, P,
                                                              Z, P]
            IP = ctypes.POINTER(ctypes.c_int)
            L.polar_attn_selftest_fwd_host_segments.argtypes = [I, IP, IP, I]
            L.polar_attn_selftest_fwd_host_segments.restype = I
            GP = ctypes.POINTER(GdeltaParams)
            L.polar_gdelta_prefill_workspace_size.argtypes = [GP]
            L.polar_gdelta_prefill_workspace_size.restype = Z
            L.polar_gdelta_prefill.argtypes = [P, P, P, P, P, P, GP, P, P, Z, P]
            L.polar_gdelta_step.argtypes = [P, P, P, P, P, P, I, P, I, GP, P, P]
            L.polar_attn_get_status.argtypes = [P]
            L.polar_attn_status_string.argtypes = [I]
            L.polar_attn_status_string.restype = ctypes.c_char_p
            L.polar_attn_launch_count.restype = ctypes.c_uint64
            for name in ("polar_attn_fwd", "polar_attn_fwd_ws", "polar_attn_fwd_host", "polar_attn_decode_paged",
                         "polar_attn_decode_paged_host", "polar_attn_get_status",
                         "polar_attn_decode_paged_noalloc", "polar_attn_selftest_exp2",
                         "polar_attn_decode_paged_chunk", "polar_attn_bwd",
                         "polar_gdelta_prefill", "polar_gdelta_step",
                         "polar_attn_selftest_timeout", "polar_attn_selftest_decode_per_head",
                         "polar_attn_fwd_train", "polar_attn_bwd_from_state"):
                getattr(L, name).restype = I
            _lib = L
    return _lib


def fwd_host_segments(T: int, cap: int = 64):
    """The row segments polar_attn_fwd_host sends for a tensor-core prefill of
    T rows, in order: a list of (lo, hi) (host logic; no device work)."""
    lo = (ctypes.c_int * max(cap, 1))()
    hi = (ctypes.c_int * max(cap, 1))()
    n = lib().polar_attn_selftest_fwd_host_segments(int(T), lo, hi, int(cap))
    if n < 0:
        raise ValueError(f"polar_attn_selftest_fwd_host_segments: bad arguments (T={T}, cap={cap})")
    return [(lo[i], hi[i]) for i in range(n)]


def status_string(code: int) -> str:
    try:
        return lib().polar_attn_status_string(int(code)).decode()
    except Exception:  # the library may be what failed
        return "?"


def make_params(B=0, T=0, Hq=16, Hkv=4, dtype=POLAR_BF16, s=8.0, alpha=0.3, L=2048, beta=1.0,
                impl="auto", window=0) -> Params:
    p = Params()
    lib().polar_attn_default_params(ctypes.byref(p), B, T, Hq, Hkv, dtype)
    p.logit_scale, p.alpha, p.L_train, p.beta = s, alpha, L, beta
    p.window = int(window)
    p.impl = IMPLS[impl] if isinstance(impl, str) else int(impl)
    return p


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return POLAR_BF16
    if t.dtype == torch.float32:
        return POLAR_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        raise PolarError(code, where)


def fwd_workspace_size(B: int, T: int, Hq: int, Hkv: int) -> int:
    p = make_params(B, T, Hq, Hkv, POLAR_BF16)
    return int(lib().polar_attn_fwd_workspace_size(ctypes.byref(p)))


def fwd(q, k, v, u, out=None, neff=None, workspace=None, *, s=8.0, alpha=0.3, L=2048, beta=1.0,
        impl="auto", stream=None, want_neff=True, moments=True, window=0):
    """Causal prefill.  q [B,T,Hq,64], k/v [B,T,Hkv,64] (bf16 or fp32, CUDA,
    contiguous), u [Hq,64] fp32.  Returns (out [B,T,Hq,64], neff [B,Hq,T]).
    moments=True calls polar_attn_fwd_ws with a workspace for the key-moment
    pre-pass (allocated here when `workspace` is None); moments=False calls
    polar_attn_fwd, which takes none."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    for t in (q, k, v, u):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if u.dtype != torch.float32:
        raise TypeError("u must be float32")
    if out is None:
        out = torch.empty_like(q)
    if neff is None and want_neff:
        neff = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    p = make_params(B, T, Hq, Hkv, _dt(q), s, alpha, L, beta, impl, window)
    p.head_dim = D
    if not moments:
        _check(lib().polar_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(u), ctypes.byref(p),
                                    _ptr(out), _ptr(neff), _stream(stream)), "polar_attn_fwd")
        return out, neff
    ws_bytes = int(lib().polar_attn_fwd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), device=q.device, dtype=torch.uint8)
    else:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().polar_attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(u), ctypes.byref(p),
                                   _ptr(out), _ptr(neff), _ptr(workspace), ws_bytes,
                                   _stream(stream)), "polar_attn_fwd_ws")
    return out, neff


def bwd_workspace_size(B: int, T: int, Hq: int, Hkv: int) -> int:
    p = make_params(B, T, Hq, Hkv, POLAR_BF16)
    return int(lib().polar_attn_bwd_workspace_size(ctypes.byref(p)))


def bwd(q, k, v, u, dout, dq=None, dk=None, dv=None, du=None, workspace=None, *, s=8.0,
        alpha=0.3, L=2048, beta=1.0, window=0, stream=None):
    """Backward of the causal prefill.  q, dout [B,T,Hq,64] and k, v [B,T,Hkv,64]
    (bf16 or fp32, CUDA, contiguous), u [Hq,64] fp32.  Returns fp32
    (dq, dk, dv, du) shaped like q, k, v, u."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    for t in (q, k, v, u, dout):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if dout.dtype != q.dtype:
        raise TypeError("dout must have the dtype of q")
    p = make_params(B, T, Hq, Hkv, _dt(q), s, alpha, L, beta, "auto", window)
    p.head_dim = D
    f32 = torch.float32
    dq = torch.empty(q.shape, device=q.device, dtype=f32) if dq is None else dq
    dk = torch.empty(k.shape, device=q.device, dtype=f32) if dk is None else dk
    dv = torch.empty(v.shape, device=q.device, dtype=f32) if dv is None else dv
    du = torch.empty(u.shape, device=q.device, dtype=f32) if du is None else du
    need = int(lib().polar_attn_bwd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    _check(lib().polar_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(dout), ctypes.byref(p),
                                _ptr(dq), _ptr(dk), _ptr(dv), _ptr(du), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "polar_attn_bwd")
    return dq, dk, dv, du


def fwd_state_size(B: int, T: int, Hq: int, Hkv: int) -> int:
    p = make_params(B, T, Hq, Hkv, POLAR_BF16)
    return int(lib().polar_attn_fwd_state_size(ctypes.byref(p)))


def fwd_train(q, k, v, u, out=None, neff=None, state=None, *, s=8.0, alpha=0.3, L=2048, beta=1.0,
              impl="auto", window=0, stream=None, want_neff=True):
    """Training forward: as fwd, plus each row's saved state for
    bwd_from_state.  Returns (out, neff, state); state is a float32
    [B, Hq, T, 8] tensor (left untouched where the state path does not
    apply)."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    for t in (q, k, v, u):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if u.dtype != torch.float32:
        raise TypeError("u must be float32")
    if out is None:
        out = torch.empty_like(q)
    if neff is None and want_neff:
        neff = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    if state is None:
        state = torch.empty((B, Hq, T, 8), device=q.device, dtype=torch.float32)
    p = make_params(B, T, Hq, Hkv, _dt(q), s, alpha, L, beta, impl, window)
    p.head_dim = D
    _check(lib().polar_attn_fwd_train(_ptr(q), _ptr(k), _ptr(v), _ptr(u), ctypes.byref(p),
                                      _ptr(out), _ptr(neff), _ptr(state), _stream(stream)),
           "polar_attn_fwd_train")
    return out, neff, state


def bwd_from_state(q, k, v, u, out, state, dout, dq=None, dk=None, dv=None, du=None,
                   workspace=None, *, s=8.0, alpha=0.3, L=2048, beta=1.0, impl="auto", window=0,
                   stream=None):
    """Backward from a training forward's out and saved state (fwd_train with
    the same arguments).  Returns fp32 (dq, dk, dv, du) as bwd."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    for t in (q, k, v, u, out, state, dout):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if dout.dtype != q.dtype or out.dtype != q.dtype:
        raise TypeError("out and dout must have the dtype of q")
    p = make_params(B, T, Hq, Hkv, _dt(q), s, alpha, L, beta, impl, window)
    p.head_dim = D
    f32 = torch.float32
    dq = torch.empty(q.shape, device=q.device, dtype=f32) if dq is None else dq
    dk = torch.empty(k.shape, device=q.device, dtype=f32) if dk is None else dk
    dv = torch.empty(v.shape, device=q.device, dtype=f32) if dv is None else dv
    du = torch.empty(u.shape, device=q.device, dtype=f32) if du is None else du
    need = int(lib().polar_attn_bwd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    _check(lib().polar_attn_bwd_from_state(_ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(out),
                                           _ptr(state), _ptr(dout), ctypes.byref(p), _ptr(dq),
                                           _ptr(dk), _ptr(dv), _ptr(du), _ptr(workspace),
                                           workspace.numel(), _stream(stream)),
           "polar_attn_bwd_from_state")
    return dq, dk, dv, du


def decode_workspace_size(num_seqs: int, max_pages: int, Hq: int, Hkv: int) -> int:
    p = make_params(0, 0, Hq, Hkv, POLAR_BF16)
    return int(lib().polar_attn_decode_workspace_size(num_seqs, max_pages, ctypes.byref(p)))


def decode_paged(q, kv_pages, page_table, seqlens, u, out=None, neff=None, workspace=None, *,
                 s=8.0, alpha=0.3, L=2048, beta=1.0, stream=None, want_neff=True, window=0):
    """Paged GQA decode.  q [N,Hq,64] bf16; kv_pages [P,2,Hkv,64,64] bf16;
    page_table [N,max_pages] int32; seqlens [N] int32; u [Hq,64] fp32.
    Returns (out [N,Hq,64], neff [N,Hq])."""
    N, Hq, D = q.shape
    P_, _, Hkv, _, _ = kv_pages.shape
    max_pages = page_table.shape[1]
    if page_table.dtype != torch.int32 or seqlens.dtype != torch.int32:
        raise TypeError("page_table and seqlens must be int32")
    p = make_params(0, 0, Hq, Hkv, _dt(q), s, alpha, L, beta, window=window)
    p.head_dim = D
    ws_need = int(lib().polar_attn_decode_workspace_size(N, max_pages, ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(ws_need, 16), device=q.device, dtype=torch.uint8)
    if out is None:
        out = torch.empty_like(q)
    if neff is None and want_neff:
        neff = torch.empty((N, Hq), device=q.device, dtype=torch.float32)
    _check(lib().polar_attn_decode_paged(
        _ptr(q), _ptr(kv_pages), P_, _ptr(page_table), max_pages, _ptr(seqlens), N, _ptr(u),
        ctypes.byref(p), _ptr(out), _ptr(neff), _ptr(workspace), workspace.numel(),
        _stream(stream)), "polar_attn_decode_paged")
    return out, neff


def decode_chunk_workspace_size(num_seqs: int, max_pages: int, chunk: int, Hq: int,
                                Hkv: int) -> int:
    p = make_params(0, 0, Hq, Hkv, POLAR_BF16)
    return int(lib().polar_attn_decode_chunk_workspace_size(num_seqs, max_pages, chunk,
                                                            ctypes.byref(p)))


def decode_paged_chunk(q, kv_pages, page_table, seqlens, u, out=None, neff=None, workspace=None,
                       *, s=8.0, alpha=0.3, L=2048, beta=1.0, stream=None, want_neff=True,
                       window=0):
    """Multi-token paged decode.  q [N,C,Hq,64] bf16: token t of sequence n is
    the query at cache position seqlens[n] - C + t.  Returns (out [N,C,Hq,64],
    neff [N,C,Hq])."""
    N, C, Hq, D = q.shape
    P_, _, Hkv, _, _ = kv_pages.shape
    max_pages = page_table.shape[1]
    if page_table.dtype != torch.int32 or seqlens.dtype != torch.int32:
        raise TypeError("page_table and seqlens must be int32")
    p = make_params(0, 0, Hq, Hkv, _dt(q), s, alpha, L, beta, window=window)
    p.head_dim = D
    ws_need = int(lib().polar_attn_decode_chunk_workspace_size(N, max_pages, C, ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(ws_need, 16), device=q.device, dtype=torch.uint8)
    if out is None:
        out = torch.empty_like(q)
    if neff is None and want_neff:
        neff = torch.empty((N, C, Hq), device=q.device, dtype=torch.float32)
    _check(lib().polar_attn_decode_paged_chunk(
        _ptr(q), _ptr(kv_pages), P_, _ptr(page_table), max_pages, _ptr(seqlens), N, C, _ptr(u),
        ctypes.byref(p), _ptr(out), _ptr(neff), _ptr(workspace), workspace.numel(),
        _stream(stream)), "polar_attn_decode_paged_chunk")
    return out, neff


# Bytes of the fixed device scratch behind decode_paged_noalloc (POLAR_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 16 << 20


def decode_paged_noalloc(q, kv_pages, page_table, seqlens, u, out, neff=None, *, s=8.0,
                         alpha=0.3, L=2048, beta=1.0, stream=None, window=0):
    """polar_attn_decode_paged_noalloc: the paged decode with no workspace, for
    callers that cannot allocate device memory.  out (and neff, if given) must
    be preallocated by the caller; this wrapper allocates nothing."""
    N, Hq, D = q.shape
    P_, _, Hkv, _, _ = kv_pages.shape
    p = make_params(0, 0, Hq, Hkv, _dt(q), s, alpha, L, beta, window=window)
    p.head_dim = D
    _check(lib().polar_attn_decode_paged_noalloc(
        _ptr(q), _ptr(kv_pages), P_, _ptr(page_table), page_table.shape[1], _ptr(seqlens), N,
        _ptr(u), ctypes.byref(p), _ptr(out), _ptr(neff), _stream(stream)),
        "polar_attn_decode_paged_noalloc")
    return out, neff


def fwd_staging_size(B, T, Hq, Hkv, dtype=POLAR_BF16) -> int:
    p = make_params(B, T, Hq, Hkv, dtype)
    return int(lib().polar_attn_fwd_staging_size(ctypes.byref(p)))


def fwd_host(q_h, k_h, v_h, u_h, out_h, neff_h, staging, *, s=8.0, alpha=0.3, L=2048, beta=1.0,
             impl="auto", stream=None, window=0):
    """polar_attn_fwd_host on (pinned) host tensors; staging is a CUDA uint8
    tensor of at least fwd_staging_size bytes.  Synchronises the stream."""
    B, T, Hq, D = q_h.shape
    p = make_params(B, T, Hq, k_h.shape[2], _dt(q_h), s, alpha, L, beta, impl, window)
    p.head_dim = D
    _check(lib().polar_attn_fwd_host(_ptr(q_h), _ptr(k_h), _ptr(v_h), _ptr(u_h), ctypes.byref(p),
                                     _ptr(out_h), _ptr(neff_h), _ptr(staging), staging.numel(),
                                     _stream(stream)), "polar_attn_fwd_host")


def decode_staging_size(num_seqs, max_pages, Hq, Hkv) -> int:
    p = make_params(0, 0, Hq, Hkv, POLAR_BF16)
    return int(lib().polar_attn_decode_staging_size(num_seqs, max_pages, ctypes.byref(p)))


def decode_paged_host(q_h, kv_pages, page_table_h, seqlens_h, u_h, out_h, neff_h, staging, *,
                      s=8.0, alpha=0.3, L=2048, beta=1.0, stream=None, window=0):
    """polar_attn_decode_paged_host: per-step inputs and outputs in (pinned)
    host memory, the KV pool resident on the device.  Synchronises the stream."""
    N, Hq, D = q_h.shape
    P_, _, Hkv, _, _ = kv_pages.shape
    p = make_params(0, 0, Hq, Hkv, _dt(q_h), s, alpha, L, beta, window=window)
    p.head_dim = D
    _check(lib().polar_attn_decode_paged_host(
        _ptr(q_h), _ptr(kv_pages), P_, _ptr(page_table_h), page_table_h.shape[1], _ptr(seqlens_h),
        N, _ptr(u_h), ctypes.byref(p), _ptr(out_h), _ptr(neff_h), _ptr(staging), staging.numel(),
        _stream(stream)), "polar_attn_decode_paged_host")


def selftest_exp2(x, stream=None):
    """The prefill kernel's FMA-pipe 2^x and MUFU ex2.approx on a CUDA fp32
    tensor x (even length).  Returns (poly, mufu)."""
    poly, mufu = torch.empty_like(x), torch.empty_like(x)
    _check(lib().polar_attn_selftest_exp2(_ptr(x), _ptr(poly), _ptr(mufu), x.numel(),
                                          _stream(stream)), "polar_attn_selftest_exp2")
    return poly, mufu


def _gd_params(B, T, H, dtype, zero_init, accumulate) -> GdeltaParams:
    return GdeltaParams(int(B), int(T), int(H), 64, int(dtype), int(bool(zero_init)),
                        int(bool(accumulate)))


def gdelta_workspace_size(B: int, T: int, H: int) -> int:
    p = _gd_params(B, T, H, POLAR_BF16, 0, 0)
    return int(lib().polar_gdelta_prefill_workspace_size(ctypes.byref(p)))


def gdelta_prefill(q, k, v, alpha, beta, state=None, out=None, workspace=None, *,
                   accumulate=False, stream=None):
    """Memory channel over whole sequences.  q, k, v [B,T,H,64] (bf16 or fp32,
    CUDA, contiguous), alpha, beta [B,T,H] fp32.  ``state`` [B,H,64,64] fp32 is
    updated in place (S_0 in, final state out); None starts from zero and
    returns a fresh final-state tensor.  With accumulate, ``out`` (required)
    gets the memory read added to it.  Returns (out, state)."""
    B, T, H, D = q.shape
    for t in (q, k, v, alpha, beta):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    zero_init = state is None
    if state is None:
        state = torch.empty((B, H, D, D), device=q.device, dtype=torch.float32)
    if out is None:
        if accumulate:
            raise ValueError("accumulate needs the output tensor to add into")
        out = torch.empty_like(q)
    p = _gd_params(B, T, H, _dt(q), zero_init, accumulate)
    p.head_dim = D
    need = int(lib().polar_gdelta_prefill_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    _check(lib().polar_gdelta_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                      _ptr(state), ctypes.byref(p), _ptr(out), _ptr(workspace),
                                      workspace.numel(), _stream(stream)), "polar_gdelta_prefill")
    return out, state


def gdelta_step(q, k, v, alpha, beta, state_pool, slots, out=None, *, accumulate=False,
                stream=None):
    """One decode token per sequence with the states updated in place in their
    pool slots.  q, k, v [N,H,64]; alpha, beta [N,H] fp32; state_pool
    [num_slots,H,64,64] fp32; slots [N] int32 (negative: skip).  Returns out."""
    N, H, D = q.shape
    for t in (q, k, v, alpha, beta, state_pool, slots):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if slots.dtype != torch.int32:
        raise TypeError("slots must be int32")
    if out is None:
        if accumulate:
            raise ValueError("accumulate needs the output tensor to add into")
        out = torch.empty_like(q)
    p = _gd_params(0, 0, H, _dt(q), 0, accumulate)
    p.head_dim = D
    _check(lib().polar_gdelta_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                   _ptr(state_pool), state_pool.shape[0], _ptr(slots), N,
                                   ctypes.byref(p), _ptr(out), _stream(stream)),
           "polar_gdelta_step")
    return out


def selftest_decode_per_head(q, kv_pages, page_table, seqlens, u, out=None, neff=None,
                             workspace=None, *, s=8.0, alpha=0.3, L=2048, beta=1.0, stream=None,
                             window=0):
    """polar_attn_selftest_decode_per_head: decode_paged with one query head per
    CTA (pages read once per query head).  Returns (out, neff)."""
    N, Hq, D = q.shape
    P_, _, Hkv, _, _ = kv_pages.shape
    max_pages = page_table.shape[1]
    p = make_params(0, 0, Hq, Hkv, _dt(q), s, alpha, L, beta, window=window)
    p.head_dim = D
    ws_need = int(lib().polar_attn_decode_workspace_size(N, max_pages, ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(ws_need, 16), device=q.device, dtype=torch.uint8)
    if out is None:
        out = torch.empty_like(q)
    if neff is None:
        neff = torch.empty((N, Hq), device=q.device, dtype=torch.float32)
    _check(lib().polar_attn_selftest_decode_per_head(
        _ptr(q), _ptr(kv_pages), P_, _ptr(page_table), max_pages, _ptr(seqlens), N, _ptr(u),
        ctypes.byref(p), _ptr(out), _ptr(neff), _ptr(workspace), workspace.numel(),
        _stream(stream)), "polar_attn_selftest_decode_per_head")
    return out, neff


def selftest_timeout(stream=None):
    """Launches one bounded wait that can never complete; afterwards
    get_status() returns POLAR_ERR_TIMEOUT (5)."""
    _check(lib().polar_attn_selftest_timeout(_stream(stream)), "polar_attn_selftest_timeout")


def get_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device status word."""
    return int(lib().polar_attn_get_status(_stream(stream)))


def launch_count() -> int:
    return int(lib().polar_attn_launch_count())
