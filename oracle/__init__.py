"""fp64 CPU oracle for the Polar Attention mixing step (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The CUDA library never calls it, and the two share no
code.  The arithmetic lives in ``polar_oracle.c``; this module only compiles
it with gcc (``-O2 -fopenmp -ffp-contract=off``, no fast-math) and marshals numpy
arrays through ctypes.

The memory channel (a gated-delta associative memory, the third additive
stream) lives in ``gdelta_oracle.c``, compiled into the same library.

Method source: "ATMA: Length-Invariant Language Modeling via Polar Attention
and Gated-Delta Compression Memory" (gist.science technical summary, section
2.1 "Polar Attention: A Three-Channel Decomposition"; section 2.2, "Fused Polar
Attention Kernel" and "GQA-Grouped Paged Decode Kernel").  The C file's header
states every formula and every reading taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "polar_oracle.c")
_SRC_GD = os.path.join(_HERE, "gdelta_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LOCK = threading.Lock()
_LIBS: dict = {}

MODES = {"two_pass": 0, "brute": 1, "stream": 2}
PAGE = 64


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("D", ctypes.c_int), ("s", ctypes.c_double), ("alpha", ctypes.c_double),
        ("L", ctypes.c_int), ("beta", ctypes.c_double), ("causal", ctypes.c_int),
        ("window", ctypes.c_int),
    ]


class _GdCfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int)]


@dataclass
class Params:
    """Method constants.  s: logit scale; alpha: length-temperature slope;
    L: training length; beta: gate slope."""
    s: float = 8.0
    alpha: float = 0.3
    L: int = 2048
    beta: float = 1.0
    causal: bool = True
    window: int = 0    # 0: every causal key; W > 0: the last W of them


def lib_path(mutant: int = 0, build_dir: str | None = None) -> str:
    d = build_dir or _BUILD
    return os.path.join(d, f"libpolar_oracle{'' if mutant == 0 else f'_m{mutant}'}.so")


def build(mutant: int = 0, build_dir: str | None = None, force: bool = False) -> str:
    """Compile the oracle (or a planted-mistake mutant of it) with gcc."""
    out = lib_path(mutant, build_dir)
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_GD))):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
           f"-DORACLE_MUTANT={int(mutant)}", "-o", tmp, _SRC, _SRC_GD, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    os.replace(tmp, out)
    return out


def _load(mutant: int = 0, build_dir: str | None = None) -> ctypes.CDLL:
    key = (mutant, build_dir)
    with _LOCK:
        if key not in _LIBS:
            lib = ctypes.CDLL(build(mutant, build_dir))
            P = ctypes.c_void_p
            lib.oracle_polar_fwd.argtypes = [
                ctypes.POINTER(_Cfg), P, P, P, ctypes.c_int, P, P, ctypes.c_int64, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, P, P, P]
            lib.oracle_polar_fwd.restype = ctypes.c_int
            lib.oracle_polar_decode.argtypes = [
                ctypes.POINTER(_Cfg), P, P, ctypes.c_int64, P, ctypes.c_int, P, ctypes.c_int,
                ctypes.c_int, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                P, P, P]
            lib.oracle_polar_decode.restype = ctypes.c_int
            lib.oracle_polar_bwd.argtypes = [
                ctypes.POINTER(_Cfg), P, P, P, ctypes.c_int, P, P, P, P, P, P]
            lib.oracle_polar_bwd.restype = ctypes.c_int
            lib.oracle_gdelta.argtypes = [ctypes.POINTER(_GdCfg), P, P, P, ctypes.c_int, P, P, P,
                                          P, ctypes.c_int]
            lib.oracle_gdelta.restype = ctypes.c_int
            lib.oracle_mutant_id.restype = ctypes.c_int
            _LIBS[key] = lib
        return _LIBS[key]


def _as_input(x: np.ndarray):
    """fp32 arrays pass as dtype 0; bf16 bit patterns (uint16) as dtype 1."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, 0
    if x.dtype == np.uint16:
        return x, 1
    raise TypeError(f"oracle inputs must be float32 or bf16 bits (uint16), got {x.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


@dataclass
class Result:
    out: np.ndarray    # [nrows, D] fp64
    neff: np.ndarray   # [nrows] fp64
    stats: np.ndarray  # [nrows, 8] fp64: m, mu, sigma, z0, gate, l, l2, c


def polar_fwd(q, k, v, u, p: Params = Params(), rows=None, mode: str = "two_pass",
              block: int = 128, theta: float = 0.0, mutant: int = 0,
              build_dir: str | None = None) -> Result:
    """Prefill rows.  q: [B,T,Hq,D]; k, v: [B,T,Hkv,D]; u: [Hq,D] float32.

    ``rows`` are flat indices ((b*Hq + h)*T + i); None means every row, in that
    order, and the result is then reshaped by the caller as [B,Hq,T,...]."""
    q, dt = _as_input(q)
    k, dk = _as_input(k)
    v, dv = _as_input(v)
    if not (dt == dk == dv):
        raise TypeError("q, k, v must share a dtype")
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, D) or v.shape != k.shape:
        raise ValueError("k/v shape mismatch")
    u = np.ascontiguousarray(u, dtype=np.float32)
    cfg = _Cfg(B, T, Hq, Hkv, D, p.s, p.alpha, p.L, p.beta, int(p.causal),
               int(p.window))
    if rows is None:
        n = B * Hq * T
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows_arr.size
    out = np.zeros((n, D), np.float64)
    neff = np.zeros(n, np.float64)
    stats = np.zeros((n, 8), np.float64)
    rc = _load(mutant, build_dir).oracle_polar_fwd(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), dt, _ptr(u), _ptr(rows_arr), n,
        MODES[mode], block, theta, _ptr(out), _ptr(neff), _ptr(stats))
    if rc != 0:
        raise ValueError(f"oracle_polar_fwd rejected its arguments (rc={rc})")
    return Result(out, neff, stats)


def polar_bwd(q, k, v, u, gout, p: Params = Params(), mutant: int = 0,
              build_dir: str | None = None):
    """Backward of the prefill: (dq, dk, dv, du) as fp64 arrays shaped like q,
    k, v and u, for the upstream gradient gout = dL/dout [B,T,Hq,D]."""
    q, dt = _as_input(q)
    k, dk_ = _as_input(k)
    v, dv_ = _as_input(v)
    if not (dt == dk_ == dv_):
        raise TypeError("q, k, v must share a dtype")
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    u = np.ascontiguousarray(u, dtype=np.float32)
    g = np.ascontiguousarray(gout, dtype=np.float64)
    if g.shape != (B, T, Hq, D):
        raise ValueError("gout shape mismatch")
    cfg = _Cfg(B, T, Hq, Hkv, D, p.s, p.alpha, p.L, p.beta, int(p.causal),
               int(p.window))
    dq = np.zeros((B, T, Hq, D), np.float64)
    dk = np.zeros((B, T, Hkv, D), np.float64)
    dv = np.zeros((B, T, Hkv, D), np.float64)
    du = np.zeros((Hq, D), np.float64)
    rc = _load(mutant, build_dir).oracle_polar_bwd(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), dt,
                                                   _ptr(u), _ptr(g), _ptr(dq), _ptr(dk), _ptr(dv),
                                                   _ptr(du))
    if rc != 0:
        raise ValueError(f"oracle_polar_bwd rejected its arguments (rc={rc})")
    return dq, dk, dv, du


def polar_decode(q, kv_pages, page_table, seqlens, u, p: Params = Params(), rows=None,
                 mode: str = "two_pass", block: int = 64, theta: float = 0.0, mutant: int = 0,
                 build_dir: str | None = None) -> Result:
    """Paged decode.  q: [N,Hq,D]; kv_pages: [P,2,Hkv,64,D]; page_table:
    [N,max_pages] int32; seqlens: [N] int32; rows: flat (s*Hq + h) or None."""
    q, dt = _as_input(q)
    kv_pages, dk = _as_input(kv_pages)
    if dt != dk:
        raise TypeError("q and kv_pages must share a dtype")
    N, Hq, D = q.shape
    P_, two, Hkv, page, D2 = kv_pages.shape
    if two != 2 or page != PAGE or D2 != D:
        raise ValueError("kv_pages must be [num_pages, 2, Hkv, 64, D]")
    page_table = np.ascontiguousarray(page_table, dtype=np.int32)
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    u = np.ascontiguousarray(u, dtype=np.float32)
    cfg = _Cfg(N, 0, Hq, Hkv, D, p.s, p.alpha, p.L, p.beta, 1, int(p.window))
    if rows is None:
        n = N * Hq
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows_arr.size
    out = np.zeros((n, D), np.float64)
    neff = np.zeros(n, np.float64)
    stats = np.zeros((n, 8), np.float64)
    rc = _load(mutant, build_dir).oracle_polar_decode(
        ctypes.byref(cfg), _ptr(q), _ptr(kv_pages), P_, _ptr(page_table), page_table.shape[1],
        _ptr(seqlens), N, dt, _ptr(u), _ptr(rows_arr), n, MODES[mode], block, theta,
        _ptr(out), _ptr(neff), _ptr(stats))
    if rc == -2:
        raise ValueError("oracle_polar_decode: page id out of range")
    if rc != 0:
        raise ValueError(f"oracle_polar_decode rejected its arguments (rc={rc})")
    return Result(out, neff, stats)


def gdelta(q, k, v, alpha, beta, state=None, literal: bool = False, mutant: int = 0,
           build_dir: str | None = None):
    """Gated-delta memory channel over whole sequences.

    q, k, v: [B,T,H,D] float32 or bf16 bits (uint16); alpha, beta: [B,T,H]
    (any float dtype, widened exactly); state: [B,H,D,D] initial state S_0
    (row = value dim, column = key dim), None for zeros.  Returns (o, S_T):
    o [B,T,H,D] and the final state [B,H,D,D], both fp64."""
    q, dt = _as_input(q)
    k, dk_ = _as_input(k)
    v, dv_ = _as_input(v)
    if not (dt == dk_ == dv_):
        raise TypeError("q, k, v must share a dtype")
    B, T, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share a shape")
    a = np.ascontiguousarray(alpha, dtype=np.float64)
    b = np.ascontiguousarray(beta, dtype=np.float64)
    if a.shape != (B, T, H) or b.shape != (B, T, H):
        raise ValueError("alpha and beta must be [B, T, H]")
    S = (np.zeros((B, H, D, D), np.float64) if state is None
         else np.array(state, dtype=np.float64, copy=True, order="C"))
    if S.shape != (B, H, D, D):
        raise ValueError("state must be [B, H, D, D]")
    out = np.zeros((B, T, H, D), np.float64)
    cfg = _GdCfg(B, T, H, D)
    rc = _load(mutant, build_dir).oracle_gdelta(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), dt,
                                                _ptr(a), _ptr(b), _ptr(S), _ptr(out), int(literal))
    if rc != 0:
        raise ValueError(f"oracle_gdelta rejected its arguments (rc={rc})")
    return out, S


def mutant_id(mutant: int = 0, build_dir: str | None = None) -> int:
    return int(_load(mutant, build_dir).oracle_mutant_id())
