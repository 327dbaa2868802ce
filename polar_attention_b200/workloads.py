"""Seeded synthetic inputs for the Polar Attention prefill and paged decode.

This module holds no step of the method: it draws Gaussian rows, L2-normalises
them (the method's stated precondition on queries and keys, "Stability
Mechanism" in section 2.1 of the ATMA technical summary), plants near-copies of
queries among the keys, and lays out a shuffled page table.  Both the CUDA path
and the CPU oracle receive the exact same bits from here.

The pages evaluate on FineWeb-Edu, induction needle-in-a-haystack and BABILong,
none of which is present; these generators stand in for them with the shapes
of the 378M-parameter model's attention (head_dim 64, 16 query heads over 4
key/value heads, training length 2048) and with planted matches so that the
participation ratio and the gate see real signal, not only noise.

All randomness comes from ``torch.Generator(device).manual_seed(seed)``; a
given (config, seed, device type) always yields the same bits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

PAGE = 64  # tokens per KV page


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int = 64
    dtype: str = "bf16"         # "bf16" or "fp32"
    plant: str = "none"         # "block" | "frac" | "needle" | "none"
    plant_frac: float = 0.0
    s: float = 8.0              # logit scale
    alpha: float = 0.3          # length-temperature slope
    L: int = 2048               # training length
    beta: float = 1.0           # gate slope
    seed: int = 0
    window: int = 0             # sliding window (0: every causal key)

    @property
    def visible_pairs(self) -> float:
        """(query, key) pairs a row sees, summed over the rows of one head:
        the causal triangle, or with a window W the rows' min(i + 1, W)."""
        T, W = self.T, self.window
        if W <= 0 or W >= T:
            return T * (T + 1) / 2.0
        return W * (W + 1) / 2.0 + (T - W) * float(W)

    @property
    def flops(self) -> float:
        """Algorithmic MMA flops of the visible pairs: 4*D per visible
        (query, key) pair (QK^T and PV, 2 flops per MAC each)."""
        return 4.0 * self.D * self.B * self.Hq * self.visible_pairs

    def describe(self) -> str:
        return (f"causal prefill B={self.B} T={self.T} Hq={self.Hq} Hkv={self.Hkv} "
                f"d={self.D} {self.dtype}")


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    num_seqs: int
    min_len: int
    max_len: int
    Hq: int = 16
    Hkv: int = 4
    D: int = 64
    dtype: str = "bf16"
    s: float = 8.0
    alpha: float = 0.3
    L: int = 2048
    beta: float = 1.0
    seed: int = 0
    plant: int = 0              # near-copies of the group's first query per (seq, kv head)
    window: int = 0             # sliding window (0: every cached position)

    def describe(self) -> str:
        return (f"paged GQA decode {self.num_seqs} seqs ctx {self.min_len}-{self.max_len} "
                f"Hq={self.Hq} Hkv={self.Hkv} d={self.D} {self.dtype} pages of {PAGE}")


# The five workloads the method is measured on (sizes of the 378M model's
# attention; the first is small enough for the oracle to finish in seconds).
TINY = PrefillWorkload("tiny_fp32_T256", B=1, T=256, Hq=2, Hkv=2, dtype="fp32", plant="block")
TRAIN = PrefillWorkload("train_len_T2048", B=8, T=2048, Hq=16, Hkv=4, plant="frac",
                        plant_frac=0.01)
EXTRAP = PrefillWorkload("extrapolation_T16384", B=2, T=16384, Hq=16, Hkv=4, plant="frac",
                         plant_frac=0.001)
LONG = PrefillWorkload("long_T65536", B=1, T=65536, Hq=16, Hkv=4, plant="needle")
DECODE = DecodeWorkload("paged_decode_128k_256k", num_seqs=32, min_len=131072, max_len=262144)

PREFILL_WORKLOADS = {w.name: w for w in (TINY, TRAIN, EXTRAP, LONG)}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def _cast(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(torch.bfloat16 if dtype == "bf16" else torch.float32).contiguous()


def prefill_inputs(w: PrefillWorkload, device="cpu", seed: int | None = None) -> dict:
    """q [B,T,Hq,D], k/v [B,T,Hkv,D] (bf16 or fp32, rows of unit norm) and
    u [Hq,D] fp32 ~ N(0, 0.02^2)."""
    device = torch.device(device)
    g = _gen(device, w.seed if seed is None else seed)
    B, T, Hq, Hkv, D = w.B, w.T, w.Hq, w.Hkv, w.D
    f32 = torch.float32
    q = _unit(torch.randn((B, T, Hq, D), generator=g, device=device, dtype=f32))
    k = _unit(torch.randn((B, T, Hkv, D), generator=g, device=device, dtype=f32))
    v = _unit(torch.randn((B, T, Hkv, D), generator=g, device=device, dtype=f32))
    u = 0.02 * torch.randn((Hq, D), generator=g, device=device, dtype=f32)
    grp = Hq // Hkv
    noise = 0.1 / math.sqrt(D)

    def rint(hi, n):  # n draws uniform in [0, hi) (hi may be a tensor)
        r = torch.rand((n,), generator=g, device=device, dtype=torch.float64)
        return (r * hi).floor().long()

    if w.plant == "block" and T > 0:
        # per 64-row query block and head: 2 keys planted at a visible position
        for b in range(B):
            for h in range(Hq):
                gk = h // grp
                for blk0 in range(0, T, 64):
                    blen = min(64, T - blk0)
                    for _ in range(2):
                        r = blk0 + int(rint(blen, 1))
                        j = int(rint(r + 1, 1))
                        eps = torch.randn((D,), generator=g, device=device, dtype=f32)
                        k[b, j, gk] = _unit(q[b, r, h] + noise * eps)
    elif w.plant == "frac" and T > 0:
        n_pl = max(1, int(round(w.plant_frac * T)))
        for b in range(B):
            for gk in range(Hkv):
                js = torch.randperm(T, generator=g, device=device)[:n_pl]
                rs = js + rint((T - js).to(torch.float64), n_pl)
                hs = gk * grp + rint(grp, n_pl)
                eps = torch.randn((n_pl, D), generator=g, device=device, dtype=f32)
                k[b, js, gk] = _unit(q[b, rs, hs] + noise * eps)
    elif w.plant == "needle" and T > 0:
        nq = min(64, T)
        for b in range(B):
            for gk in range(Hkv):
                nu = _unit(torch.randn((D,), generator=g, device=device, dtype=f32))
                p0 = int(rint(max(1, T // 2 - 16), 1))
                nk = min(16, T - p0)
                eps = torch.randn((nk, D), generator=g, device=device, dtype=f32)
                k[b, p0:p0 + nk, gk] = _unit(nu + noise * eps)
                eps = torch.randn((nq, grp, D), generator=g, device=device, dtype=f32)
                q[b, T - nq:, gk * grp:(gk + 1) * grp] = _unit(nu + noise * eps)
    return {"q": _cast(q, w.dtype), "k": _cast(k, w.dtype), "v": _cast(v, w.dtype), "u": u}


def decode_lengths(w: DecodeWorkload, seed: int | None = None) -> np.ndarray:
    rng = np.random.default_rng(w.seed if seed is None else seed)
    return rng.integers(w.min_len, w.max_len + 1, size=w.num_seqs).astype(np.int32)


def decode_inputs(w: DecodeWorkload, device="cpu", seed: int | None = None,
                  seqlens=None, chunk_pages: int = 2048) -> dict:
    """q [N,Hq,D], kv_pages [P,2,Hkv,64,D] (the physical pool), page_table
    [N,max_pages] int32 (a random permutation of the pool; -1 past the end of
    a sequence), seqlens [N] int32 and u [Hq,D] fp32.

    The pool is drawn ``chunk_pages`` pages at a time so that full-size pools
    (about 98K pages, 6.4 GB in bf16) never need an fp32 copy."""
    device = torch.device(device)
    s = w.seed if seed is None else seed
    lens = decode_lengths(w, s) if seqlens is None else np.asarray(seqlens, np.int32)
    N = int(lens.size)
    npg = (lens.astype(np.int64) + PAGE - 1) // PAGE
    P = int(npg.sum())
    max_pages = int(npg.max()) if N else 0
    rng = np.random.default_rng(s + 1)
    perm = rng.permutation(P).astype(np.int32)
    pt = np.full((N, max_pages), -1, np.int32)
    o = 0
    for i in range(N):
        pt[i, :npg[i]] = perm[o:o + npg[i]]
        o += int(npg[i])
    g = _gen(device, s)
    f32 = torch.float32
    q = _unit(torch.randn((N, w.Hq, w.D), generator=g, device=device, dtype=f32))
    u = 0.02 * torch.randn((w.Hq, w.D), generator=g, device=device, dtype=f32)
    kv = torch.empty((P, 2, w.Hkv, PAGE, w.D), device=device,
                     dtype=torch.bfloat16 if w.dtype == "bf16" else f32)
    for p0 in range(0, P, chunk_pages):
        p1 = min(P, p0 + chunk_pages)
        x = torch.randn((p1 - p0, 2, w.Hkv, PAGE, w.D), generator=g, device=device, dtype=f32)
        kv[p0:p1] = _unit(x).to(kv.dtype)
    if w.plant > 0:
        grp = w.Hq // w.Hkv
        pt_t = torch.from_numpy(pt).to(device)
        noise = 0.1 / math.sqrt(w.D)
        for i in range(N):
            pos = rng.integers(0, int(lens[i]), size=(w.Hkv, w.plant))
            for gk in range(w.Hkv):
                for j in pos[gk]:
                    eps = torch.randn((w.D,), generator=g, device=device, dtype=f32)
                    kv[pt_t[i, j // PAGE], 0, gk, j % PAGE] = _unit(
                        q[i, gk * grp] + noise * eps).to(kv.dtype)
    return {"q": _cast(q, w.dtype), "kv_pages": kv.contiguous(),
            "page_table": torch.from_numpy(pt).to(device), "seqlens": torch.from_numpy(lens).to(device),
            "u": u, "num_pages": P, "max_pages": max_pages}


def decode_chunk_queries(w: DecodeWorkload, x: dict, chunk: int, seed: int | None = None) -> torch.Tensor:
    """Queries of a multi-token decode: q [N, chunk, Hq, D], unit rows.  The
    last token of each sequence is the single-token decode query x["q"] (whose
    planted keys sit in the cache); the earlier tokens are fresh random rows."""
    q1 = x["q"]
    N = q1.shape[0]
    g = _gen(q1.device, (w.seed if seed is None else seed) + 7)
    fresh = _unit(torch.randn((N, chunk, w.Hq, w.D), generator=g, device=q1.device,
                              dtype=torch.float32))
    q = _cast(fresh, w.dtype).clone()
    q[:, chunk - 1] = q1
    return q.contiguous()


@dataclass(frozen=True)
class GdeltaWorkload:
    """The memory channel (gated-delta memory, one state per (sequence, head)).

    Inputs: q, k ~ N(0, 1) rows of arbitrary length (the channel normalises
    them itself), v unit rows, decay gates alpha = 1 - 10^U(lg_lo, lg_hi)
    (between 0.9 and 0.999 by default: memories from about ten to about a
    thousand tokens), write strengths beta = sigmoid(N(0, 1))."""
    name: str
    B: int
    T: int
    H: int = 16
    D: int = 64
    dtype: str = "bf16"
    seed: int = 0
    lg_lo: float = -3.0
    lg_hi: float = -1.0

    @property
    def flops(self) -> float:
        """Flops of the token-by-token recurrence: S k, the rank-one write and
        S q, 2 D^2 each (2 flops per multiply-add), per (token, head)."""
        return 6.0 * self.D * self.D * self.B * self.T * self.H

    def describe(self) -> str:
        return f"gated-delta memory B={self.B} T={self.T} H={self.H} d={self.D} {self.dtype}"


@dataclass(frozen=True)
class GdeltaStepWorkload:
    """One decode token per sequence against a pool of state slots (random
    distinct slots, states ~ N(0, 0.1^2))."""
    name: str
    num_seqs: int
    num_slots: int
    H: int = 16
    D: int = 64
    dtype: str = "bf16"
    seed: int = 0

    @property
    def state_bytes(self) -> int:
        """Bytes the step must move: every state read once and written once."""
        return 2 * self.num_seqs * self.H * self.D * self.D * 4

    def describe(self) -> str:
        return (f"gated-delta step {self.num_seqs} seqs x {self.H} heads, pool of "
                f"{self.num_slots} slots, {self.dtype}")


GD_TRAIN = GdeltaWorkload("gdelta_train_T2048", B=8, T=2048, H=16)
GD_STEP = GdeltaStepWorkload("gdelta_step_1024seqs", num_seqs=1024, num_slots=1024, H=16)


def gdelta_inputs(w: GdeltaWorkload, device="cpu", seed: int | None = None) -> dict:
    """q, k, v [B,T,H,D] (dtype), alpha, beta [B,T,H] fp32."""
    device = torch.device(device)
    g = _gen(device, w.seed if seed is None else seed)
    f32 = torch.float32
    shp = (w.B, w.T, w.H, w.D)
    q = torch.randn(shp, generator=g, device=device, dtype=f32)
    k = torch.randn(shp, generator=g, device=device, dtype=f32)
    v = _unit(torch.randn(shp, generator=g, device=device, dtype=f32))
    u = torch.rand((w.B, w.T, w.H), generator=g, device=device, dtype=f32)
    alpha = 1.0 - torch.pow(10.0, w.lg_lo + (w.lg_hi - w.lg_lo) * u)
    beta = torch.sigmoid(torch.randn((w.B, w.T, w.H), generator=g, device=device, dtype=f32))
    return {"q": _cast(q, w.dtype), "k": _cast(k, w.dtype), "v": _cast(v, w.dtype),
            "alpha": alpha.contiguous(), "beta": beta.contiguous()}


def gdelta_step_inputs(w: GdeltaStepWorkload, device="cpu", seed: int | None = None) -> dict:
    """q, k, v [N,H,D], alpha, beta [N,H], state_pool [num_slots,H,D,D] fp32,
    slots [N] int32 (distinct)."""
    device = torch.device(device)
    s = w.seed if seed is None else seed
    g = _gen(device, s)
    f32 = torch.float32
    shp = (w.num_seqs, w.H, w.D)
    q = torch.randn(shp, generator=g, device=device, dtype=f32)
    k = torch.randn(shp, generator=g, device=device, dtype=f32)
    v = _unit(torch.randn(shp, generator=g, device=device, dtype=f32))
    u = torch.rand((w.num_seqs, w.H), generator=g, device=device, dtype=f32)
    alpha = 1.0 - torch.pow(10.0, -3.0 + 2.0 * u)
    beta = torch.sigmoid(torch.randn((w.num_seqs, w.H), generator=g, device=device, dtype=f32))
    pool = 0.1 * torch.randn((w.num_slots, w.H, w.D, w.D), generator=g, device=device, dtype=f32)
    perm = np.random.default_rng(s + 1).permutation(w.num_slots)[:w.num_seqs].astype(np.int32)
    return {"q": _cast(q, w.dtype), "k": _cast(k, w.dtype), "v": _cast(v, w.dtype),
            "alpha": alpha.contiguous(), "beta": beta.contiguous(), "state_pool": pool.contiguous(),
            "slots": torch.from_numpy(perm).to(device)}


def small_gdelta(B=1, T=300, H=2, dtype="bf16", seed=0, **kw) -> GdeltaWorkload:
    return GdeltaWorkload(f"custom_gdelta_B{B}_T{T}_H{H}", B=B, T=T, H=H, dtype=dtype, seed=seed,
                          **kw)


def small_prefill(B=1, T=300, Hq=4, Hkv=2, D=64, dtype="fp32", seed=0, **kw) -> PrefillWorkload:
    return PrefillWorkload(f"custom_B{B}_T{T}_H{Hq}x{Hkv}", B=B, T=T, Hq=Hq, Hkv=Hkv, D=D,
                           dtype=dtype, seed=seed, **kw)


def small_decode(num_seqs=3, min_len=1, max_len=700, Hq=8, Hkv=2, dtype="bf16", seed=0,
                 **kw) -> DecodeWorkload:
    return DecodeWorkload(f"custom_decode_{num_seqs}x{min_len}_{max_len}", num_seqs=num_seqs,
                          min_len=min_len, max_len=max_len, Hq=Hq, Hkv=Hkv, dtype=dtype,
                          seed=seed, **kw)


def with_seed(w, seed: int):
    return replace(w, seed=seed)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """Exact host copy for the oracle: fp32 values, or bf16 bit patterns as uint16."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.int32:
        return t.numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")
