"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each ``pin_*`` function returns normally when the oracle (or a planted-mistake
mutant of it, ``mutant=k``) agrees with an independent fact, and raises
``AssertionError`` otherwise.  The facts are closed forms derived by hand from
the definitions (below each pin), invariants the pages state for the method
(ATMA technical summary, section 2.1: the direction is count-blind and of unit
norm; the participation ratio is an inverse Simpson index; the magnitude map is
bounded), and brute force on tiny inputs.  ``test_oracle_pins.py`` runs them
on the real oracle; ``test_oracle_mutants.py`` shows that every planted
mistake fails at least one of them.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from oracle import Params

RTOL = 1e-12


def _close(a, b, rtol=RTOL, atol=1e-13, what=""):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if not np.allclose(a, b, rtol=rtol, atol=atol):
        err = np.max(np.abs(a - b))
        raise AssertionError(f"{what}: max abs diff {err:.3e}")


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_inputs(rng, B, T, Hq, Hkv, D=64):
    q = _unit(rng.standard_normal((B, T, Hq, D))).astype(np.float32)
    k = _unit(rng.standard_normal((B, T, Hkv, D))).astype(np.float32)
    v = _unit(rng.standard_normal((B, T, Hkv, D))).astype(np.float32)
    u = (0.02 * rng.standard_normal((Hq, D))).astype(np.float32)
    # plant a few strong matches so the max moves between blocks
    for b in range(B):
        for g in range(Hkv):
            for j in rng.integers(0, T, size=3):
                r = int(rng.integers(j, T))
                h = g * (Hq // Hkv)
                k[b, j, g] = _unit(q[b, r, h] + 0.05 * rng.standard_normal(D)).astype(np.float32)
    return q, k, v, u


def _paged_from_dense(k, v, b, perm_seed=0):
    """One sequence's dense k/v [T,Hkv,D] as a shuffled page pool."""
    T, Hkv, D = k.shape[1], k.shape[2], k.shape[3]
    npg = (T + 63) // 64
    rng = np.random.default_rng(perm_seed)
    perm = rng.permutation(npg + 2)[:npg]  # two spare pages never referenced
    pool = np.zeros((npg + 2, 2, Hkv, 64, D), k.dtype)
    for p in range(npg):
        t0, t1 = p * 64, min(T, p * 64 + 64)
        pool[perm[p], 0, :, :t1 - t0] = np.transpose(k[b, t0:t1], (1, 0, 2))
        pool[perm[p], 1, :, :t1 - t0] = np.transpose(v[b, t0:t1], (1, 0, 2))
    return pool, perm.astype(np.int32)[None, :]


# --------------------------------------------------------------------------
# 1. brute force == two-pass == streaming (blocks 1/7/64/128, lazy or not)
#    Brute force materialises p_j = e^{z_j}/sum e^z and n_eff = 1/sum p^2.
# --------------------------------------------------------------------------
def pin_modes_agree(mutant=0, bd=None):
    rng = np.random.default_rng(1)
    q, k, v, u = _rand_inputs(rng, B=2, T=300, Hq=4, Hkv=2)
    p = Params(s=8.0, alpha=0.3, L=64, beta=1.0)  # L=64 so the temperature acts
    ref = oracle.polar_fwd(q, k, v, u, p, mode="brute", mutant=mutant, build_dir=bd)
    for mode, blk, th in [("two_pass", 0, 0.0), ("stream", 1, 0.0), ("stream", 7, 0.0),
                          ("stream", 64, 0.0), ("stream", 128, 0.0), ("stream", 128, 8 * math.log(2)),
                          ("stream", 1, 8 * math.log(2))]:
        got = oracle.polar_fwd(q, k, v, u, p, mode=mode, block=max(blk, 1), theta=th,
                               mutant=mutant, build_dir=bd)
        _close(got.neff, ref.neff, what=f"neff {mode}/{blk}/{th}")
        _close(got.out, ref.out, what=f"out {mode}/{blk}/{th}")
        _close(got.stats[:, :5], ref.stats[:, :5], rtol=1e-11, what=f"stats {mode}/{blk}")
        # l and l2 relative to the true max agree too
        _close(got.stats[:, 5:7], ref.stats[:, 5:7], rtol=1e-11, what=f"l,l2 {mode}/{blk}")


# --------------------------------------------------------------------------
# 2. uniform logits: all keys equal => every p_j = 1/n => n_eff = n exactly,
#    sigma = 0 => z0 = mu = m => gate = 1/2, count = tanh(ln n / ln L)/2 * u_h,
#    content = sum_j v_j / |sum_j v_j|.  Causal row i sees n = i + 1 keys.
# --------------------------------------------------------------------------
def pin_uniform(mutant=0, bd=None):
    rng = np.random.default_rng(2)
    B, T, Hq, Hkv, D = 1, 200, 2, 1, 64
    q = _unit(rng.standard_normal((B, T, Hq, D))).astype(np.float32)
    kstar = _unit(rng.standard_normal(D)).astype(np.float32)
    k = np.broadcast_to(kstar, (B, T, Hkv, D)).copy()
    v = _unit(rng.standard_normal((B, T, Hkv, D))).astype(np.float32)
    u = (0.02 * rng.standard_normal((Hq, D))).astype(np.float32)
    L = 128
    res = oracle.polar_fwd(q, k, v, u, Params(L=L, alpha=0.0), mutant=mutant, build_dir=bd)
    neff = res.neff.reshape(B, Hq, T)
    out = res.out.reshape(B, Hq, T, D)
    vs = v.astype(np.float64)
    for h in range(Hq):
        for i in [0, 1, 2, 63, 127, 128, 199]:
            n = i + 1
            assert abs(neff[0, h, i] - n) <= 1e-9 * n, f"n_eff at n={n}: {neff[0, h, i]}"
            acc = vs[0, :n, 0].sum(0)
            content = acc / np.linalg.norm(acc)
            count = 0.5 * math.tanh(math.log(n) / math.log(L)) * u[h].astype(np.float64)
            _close(out[0, h, i], content + count, rtol=1e-10, atol=1e-12, what=f"uniform h{h} i{i}")


def pin_uniform_train_length_constant(mutant=0, bd=None):
    """At n = L = 2048 the uniform count factor is tanh(1)/2 = 0.380797077977882."""
    rng = np.random.default_rng(3)
    n, D, Hq, Hkv = 2048, 64, 1, 1
    q = _unit(rng.standard_normal((1, Hq, D))).astype(np.float32)
    kstar = _unit(rng.standard_normal(D)).astype(np.float32)
    k = np.broadcast_to(kstar, (1, n, Hkv, D)).copy()
    v = np.zeros((1, n, Hkv, D), np.float32)
    v[..., 0] = 1.0  # content = e_0 exactly
    u = np.ones((Hq, D), np.float32)
    pool, pt = _paged_from_dense(k, v, 0)
    res = oracle.polar_decode(q, pool, pt, np.array([n], np.int32), u, Params(L=2048),
                              mutant=mutant, build_dir=bd)
    count = res.out[0].copy()
    count[0] -= 1.0
    _close(count, np.full(D, 0.3807970779778824), rtol=1e-12, what="tanh(1)/2")


# --------------------------------------------------------------------------
# 3. closed form of the whole pipeline.  q = e_0; `km` matched keys equal e_0
#    (raw dot 1, logit c); the other n-km keys are unit vectors orthogonal to
#    e_0 (logit 0).  With p = km/n:
#      m = c, mu = c p, sigma = c sqrt(p(1-p)), z0 = mu + sigma sqrt(2 ln n),
#      gate = 1/(1+exp(-beta (c - z0))),
#      n_eff = (km + (n-km) e^{-c})^2 / (km + (n-km) e^{-2c}),
#      content = normalize(sum_match v + e^{-c} sum_other v),
#      out = content + gate tanh(ln n_eff / ln L) u_h,
#    with c = s (1 + alpha ln(n/L)) when n > L.  Runs through decode with two
#    query heads per kv head and distinct u per head.
# --------------------------------------------------------------------------
def _closed_form_case(n, km, s, alpha, L, beta, seed, mutant, bd):
    rng = np.random.default_rng(seed)
    D, Hq, Hkv = 64, 2, 1
    q = np.zeros((1, Hq, D), np.float32)
    q[0, :, 0] = 1.0
    match = np.sort(rng.choice(n, size=km, replace=False))
    k = np.zeros((1, n, Hkv, D), np.float32)
    other = np.ones(n, bool)
    other[match] = False
    k[0, match, 0, 0] = 1.0
    ax = 1 + (np.arange(n) % (D - 1))
    k[0, other, 0, ax[other]] = 1.0
    v = _unit(rng.standard_normal((1, n, Hkv, D))).astype(np.float32)
    u = (0.02 * rng.standard_normal((Hq, D))).astype(np.float32)
    pool, pt = _paged_from_dense(k, v, 0, perm_seed=seed)
    res = oracle.polar_decode(q, pool, pt, np.array([n], np.int32), u,
                              Params(s=s, alpha=alpha, L=L, beta=beta), mutant=mutant, build_dir=bd)
    tau = 1.0 + alpha * math.log(n / L) if n > L else 1.0
    c = s * tau
    p = km / n
    mu, sigma = c * p, c * math.sqrt(p * (1 - p))
    z0 = mu + sigma * math.sqrt(2 * math.log(n))
    gate = 1.0 / (1.0 + math.exp(-beta * (c - z0)))
    e1, e2 = math.exp(-c), math.exp(-2 * c)
    neff = (km + (n - km) * e1) ** 2 / (km + (n - km) * e2)
    vv = v[0, :, 0].astype(np.float64)
    acc = vv[match].sum(0) + e1 * vv[other].sum(0)
    content = acc / np.linalg.norm(acc)
    for h in range(Hq):
        want = content + gate * math.tanh(math.log(neff) / math.log(L)) * u[h].astype(np.float64)
        _close(res.neff[h], neff, rtol=1e-11, what=f"closed-form n_eff n={n} km={km}")
        _close(res.stats[h, :5], [c, mu, sigma, z0, gate], rtol=1e-11, atol=1e-12,
               what=f"closed-form stats n={n} km={km}")
        _close(res.out[h], want, rtol=1e-11, atol=1e-13, what=f"closed-form out n={n} km={km} h={h}")


def pin_closed_form(mutant=0, bd=None):
    _closed_form_case(n=1000, km=7, s=8.0, alpha=0.3, L=2048, beta=1.0, seed=4, mutant=mutant, bd=bd)
    _closed_form_case(n=5000, km=3, s=8.0, alpha=0.3, L=2048, beta=1.5, seed=5, mutant=mutant, bd=bd)
    _closed_form_case(n=4097, km=100, s=4.0, alpha=0.5, L=1024, beta=0.7, seed=6, mutant=mutant, bd=bd)
    # one dominant logit: n_eff -> 1 as the gap grows
    _closed_form_case(n=300, km=1, s=30.0, alpha=0.0, L=2048, beta=1.0, seed=7, mutant=mutant, bd=bd)


# --------------------------------------------------------------------------
# 4. length-temperature and null-floor constants at n = 4096, L = 2048,
#    alpha = 0.3: tau = 1 + 0.3 ln 2 = 1.2079441541679836,
#    sqrt(2 ln 4096) = 4.078667960675236  (z0 = mu + sigma * that).
# --------------------------------------------------------------------------
def pin_temperature_constants(mutant=0, bd=None):
    rng = np.random.default_rng(8)
    n, D = 4096, 64
    q = _unit(rng.standard_normal((1, 1, D))).astype(np.float32)
    k = _unit(rng.standard_normal((1, n, 1, D))).astype(np.float32)
    v = _unit(rng.standard_normal((1, n, 1, D))).astype(np.float32)
    u = np.zeros((1, D), np.float32)
    pool, pt = _paged_from_dense(k, v, 0)
    res = oracle.polar_decode(q, pool, pt, np.array([n], np.int32), u, Params(alpha=0.3, L=2048),
                              mutant=mutant, build_dir=bd)
    m, mu, sigma, z0, gate, l, l2, c = res.stats[0]
    _close(c, 8.0 * 1.2079441541679836, what="c = s*tau(4096)")
    _close(z0, mu + sigma * 4.078667960675236, what="z0 = mu + sigma*sqrt(2 ln 4096)")
    # the mean and the population std of the logits, from the inputs directly
    z = c * (k[0, :, 0].astype(np.float64) @ q[0, 0].astype(np.float64))
    _close([mu, sigma, m], [z.mean(), z.std(), z.max()], rtol=1e-11, what="mu, sigma, max")


# --------------------------------------------------------------------------
# 5. direction channel has unit norm (u = 0 isolates it) and the count channel
#    is bounded by |u_h| for every n (checked up to n = 262144).
# --------------------------------------------------------------------------
def pin_unit_norm_and_bounded(mutant=0, bd=None):
    rng = np.random.default_rng(9)
    q, k, v, u = _rand_inputs(rng, B=1, T=257, Hq=2, Hkv=1)
    zero = np.zeros_like(u)
    r0 = oracle.polar_fwd(q, k, v, zero, Params(L=64), mutant=mutant, build_dir=bd)
    _close(np.linalg.norm(r0.out, axis=1), 1.0, what="|content| = 1")
    for n in [1, 2, 100, 262144]:
        D = 64
        kk = _unit(rng.standard_normal((1, n, 1, D))).astype(np.float32)
        vv = _unit(rng.standard_normal((1, n, 1, D))).astype(np.float32)
        qq = _unit(rng.standard_normal((1, 1, D))).astype(np.float32)
        uu = (0.02 * rng.standard_normal((1, D))).astype(np.float32)
        pool, pt = _paged_from_dense(kk, vv, 0)
        sl = np.array([n], np.int32)
        a = oracle.polar_decode(qq, pool, pt, sl, uu, Params(), mutant=mutant, build_dir=bd)
        b = oracle.polar_decode(qq, pool, pt, sl, np.zeros_like(uu), Params(), mutant=mutant, build_dir=bd)
        count = a.out[0] - b.out[0]
        assert np.all(np.abs(count) < np.abs(uu[0]) + 1e-15), f"count unbounded at n={n}"
        assert 1.0 - 1e-12 <= a.neff[0] <= n * (1 + 1e-12), f"n_eff outside [1, n] at n={n}"
        _close(np.linalg.norm(b.out[0]), 1.0, what=f"|content| = 1 at n={n}")


# --------------------------------------------------------------------------
# 6. duplication: repeating every (k, v) pair leaves the direction unchanged
#    and doubles n_eff exactly (temperature inactive: n, 2n <= L).
# --------------------------------------------------------------------------
def pin_duplication(mutant=0, bd=None):
    rng = np.random.default_rng(10)
    n, D = 500, 64
    q = _unit(rng.standard_normal((1, 2, D))).astype(np.float32)
    k = _unit(rng.standard_normal((1, n, 1, D))).astype(np.float32)
    v = _unit(rng.standard_normal((1, n, 1, D))).astype(np.float32)
    k[0, 17, 0] = q[0, 0]
    u = np.zeros((2, D), np.float32)
    k2 = np.concatenate([k, k[:, ::-1]], axis=1)
    v2 = np.concatenate([v, v[:, ::-1]], axis=1)
    p1, t1 = _paged_from_dense(k, v, 0)
    p2, t2 = _paged_from_dense(k2, v2, 0, perm_seed=3)
    a = oracle.polar_decode(q, p1, t1, np.array([n], np.int32), u, Params(), mutant=mutant, build_dir=bd)
    b = oracle.polar_decode(q, p2, t2, np.array([2 * n], np.int32), u, Params(), mutant=mutant, build_dir=bd)
    _close(b.neff, 2 * a.neff, rtol=1e-11, what="n_eff doubles")
    _close(b.out, a.out, rtol=1e-11, atol=1e-13, what="direction unchanged")


# --------------------------------------------------------------------------
# 7. causality: changing keys/values after row i leaves row i bit-identical,
#    and row 0 (n = 1: gate 1/2, n_eff 1, count 0) returns v_0 itself.
# --------------------------------------------------------------------------
def pin_causality(mutant=0, bd=None):
    rng = np.random.default_rng(11)
    q, k, v, u = _rand_inputs(rng, B=1, T=130, Hq=2, Hkv=1)
    base = oracle.polar_fwd(q, k, v, u, Params(L=64), mutant=mutant, build_dir=bd)
    i = 77
    k2, v2 = k.copy(), v.copy()
    k2[0, i + 1:] = _unit(rng.standard_normal(k2[0, i + 1:].shape)).astype(np.float32)
    v2[0, i + 1:] = _unit(rng.standard_normal(v2[0, i + 1:].shape)).astype(np.float32)
    pert = oracle.polar_fwd(q, k2, v2, u, Params(L=64), mutant=mutant, build_dir=bd)
    T = 130
    for h in range(2):
        r = h * T + i
        assert np.array_equal(base.out[r], pert.out[r]) and base.neff[r] == pert.neff[r], \
            "row depends on future keys"
        r0 = h * T
        _close(base.out[r0], v[0, 0, 0].astype(np.float64) / np.linalg.norm(v[0, 0, 0].astype(np.float64)),
               rtol=1e-14, atol=1e-15, what="row 0 = v_0")
        assert base.neff[r0] == 1.0
    # a row does change when a visible key changes
    k3 = k.copy()
    k3[0, i] = q[0, i, 0]
    ch = oracle.polar_fwd(q, k3, v, u, Params(L=64), rows=[i], mutant=mutant, build_dir=bd)
    assert not np.array_equal(ch.out[0], base.out[i]), "row ignores its own diagonal key"


# --------------------------------------------------------------------------
# 8. GQA mapping: q heads g*G .. g*G+G-1 share kv head g; the same computation
#    with kv heads repeated explicitly (Hq = Hkv) gives identical results.
# --------------------------------------------------------------------------
def pin_gqa(mutant=0, bd=None):
    rng = np.random.default_rng(12)
    q, k, v, u = _rand_inputs(rng, B=1, T=90, Hq=8, Hkv=2)
    a = oracle.polar_fwd(q, k, v, u, Params(L=64), mutant=mutant, build_dir=bd)
    kr = np.repeat(k, 4, axis=2)
    vr = np.repeat(v, 4, axis=2)
    b = oracle.polar_fwd(q, kr, vr, u, Params(L=64), mutant=mutant, build_dir=bd)
    _close(a.out, b.out, rtol=0, atol=0, what="GQA vs repeated heads")


# --------------------------------------------------------------------------
# 9. decode over a shuffled page pool == prefill's last row on the same keys.
# --------------------------------------------------------------------------
def pin_decode_matches_prefill(mutant=0, bd=None):
    rng = np.random.default_rng(13)
    T = 333
    q, k, v, u = _rand_inputs(rng, B=1, T=T, Hq=4, Hkv=2)
    pf = oracle.polar_fwd(q, k, v, u, Params(L=64), mutant=mutant, build_dir=bd)
    pool, pt = _paged_from_dense(k, v, 0, perm_seed=5)
    dq = np.ascontiguousarray(q[:, T - 1])
    dc = oracle.polar_decode(dq, pool, pt, np.array([T], np.int32), u, Params(L=64),
                             mutant=mutant, build_dir=bd)
    last = [h * T + T - 1 for h in range(4)]
    _close(dc.out, pf.out[last], rtol=0, atol=0, what="decode vs prefill last row")
    _close(dc.neff, pf.neff[last], rtol=0, atol=0, what="decode vs prefill n_eff")


# --------------------------------------------------------------------------
# 10. sliding window W: a window no shorter than the sequence changes nothing;
#     W = 1 leaves each row only its own key (out = v_i / |v_i|, n_eff = 1,
#     gate 1/2, count 0); row i >= W-1 equals the unwindowed last row of the
#     slice of keys i-W+1 .. i taken as a sequence of its own (same keys, same
#     count n = W, so the same temperature), bit for bit, and earlier rows
#     equal their unwindowed selves; a windowed decode equals the windowed
#     prefill's last row.
# --------------------------------------------------------------------------
def pin_window(mutant=0, bd=None):
    rng = np.random.default_rng(14)
    T, W = 150, 37
    q, k, v, u = _rand_inputs(rng, B=1, T=T, Hq=2, Hkv=1)
    full = oracle.polar_fwd(q, k, v, u, Params(L=16), mutant=mutant, build_dir=bd)
    big = oracle.polar_fwd(q, k, v, u, Params(L=16, window=T), mutant=mutant, build_dir=bd)
    _close(big.out, full.out, rtol=0, atol=0, what="window >= T")
    one = oracle.polar_fwd(q, k, v, u, Params(L=16, window=1), mutant=mutant, build_dir=bd)
    vv = v[0, :, 0].astype(np.float64)
    for h in range(2):
        _close(one.out[h * T:(h + 1) * T], vv / np.linalg.norm(vv, axis=1, keepdims=True),
               rtol=1e-14, atol=1e-15, what="window 1 = v_i")
    assert np.all(one.neff == 1.0)
    win = oracle.polar_fwd(q, k, v, u, Params(L=16, window=W), mutant=mutant, build_dir=bd)
    for h in range(2):
        r = [h * T + i for i in range(W - 1)]
        _close(win.out[r], full.out[r], rtol=0, atol=0, what="rows inside the first window")
    for i in (W - 1, W, 90, T - 1):
        sl = slice(i - W + 1, i + 1)
        qs, ks, vs = (np.ascontiguousarray(x[:, sl]) for x in (q, k, v))
        ref = oracle.polar_fwd(qs, ks, vs, u, Params(L=16), mutant=mutant, build_dir=bd,
                               rows=[h * W + W - 1 for h in range(2)])
        got = [h * T + i for h in range(2)]
        _close(win.out[got], ref.out, rtol=0, atol=0, what=f"window row {i} vs slice")
        _close(win.neff[got], ref.neff, rtol=0, atol=0, what=f"window n_eff {i} vs slice")
    pool, pt = _paged_from_dense(k, v, 0, perm_seed=6)
    dc = oracle.polar_decode(np.ascontiguousarray(q[:, T - 1]), pool, pt,
                             np.array([T], np.int32), u, Params(L=16, window=W),
                             mutant=mutant, build_dir=bd)
    _close(dc.out, win.out[[T - 1, 2 * T - 1]], rtol=0, atol=0, what="windowed decode")


# --------------------------------------------------------------------------
# 11. backward: the oracle's analytic gradients of L = <out, G> (G random)
#     against central finite differences of the oracle's own forward, for
#     coordinates of q, k, v and u, with and without a window.  The forward is
#     pinned by 1-10, so this ties the gradient to the pages' forms.
# --------------------------------------------------------------------------
def pin_backward_finite_differences(mutant=0, bd=None):
    rng = np.random.default_rng(15)
    T, Hq, Hkv = 24, 4, 2
    q, k, v, u = _rand_inputs(rng, B=1, T=T, Hq=Hq, Hkv=Hkv)
    u = (0.5 * rng.standard_normal(u.shape)).astype(np.float32)  # a count large enough to matter
    G = rng.standard_normal((1, T, Hq, 64))
    for p in (Params(L=4, alpha=0.3), Params(L=4, alpha=0.3, window=9)):
        dq, dk, dv, du = oracle.polar_bwd(q, k, v, u, G, p, mutant=mutant, build_dir=bd)

        def loss(qq, kk, vv, uu):
            r = oracle.polar_fwd(qq, kk, vv, uu, p, mutant=mutant, build_dir=bd)
            out = r.out.reshape(1, Hq, T, 64).transpose(0, 2, 1, 3)
            return float(np.sum(out * G))

        def fd(arrs, which, idx, eps=1e-3):
            a = list(arrs)
            x = a[which]
            xp, xm = x.copy(), x.copy()
            xp[idx] = np.float32(x[idx] + eps)
            xm[idx] = np.float32(x[idx] - eps)
            step = float(xp[idx]) - float(xm[idx])  # exact: both ends are fp32 values
            a[which] = xp
            lp = loss(*a)
            a[which] = xm
            lm = loss(*a)
            return (lp - lm) / step

        arrs = (q, k, v, u)
        grads = (dq, dk, dv, du)
        for which in range(4):
            for _ in range(6):
                idx = tuple(int(rng.integers(0, n)) for n in arrs[which].shape)
                num = fd(arrs, which, idx)
                ana = grads[which][idx]
                scale = max(1e-3, np.max(np.abs(grads[which])))
                assert abs(num - ana) <= 2e-4 * scale, \
                    f"grad {'qkvu'[which]}{idx} window={p.window}: fd {num:.6e} vs {ana:.6e}"


# ---- memory channel (gated-delta associative memory) ---------------------
# The pages name the rule (ATMA technical summary, section 2.1, "Recurrent
# Memory Channel": gated-delta memory with L2-normalised keys and queries);
# the facts below follow from the delta rule itself, not from the oracle.

def _gd_rand(rng, B, T, H, D=64, scale_rows=True):
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, H, D))
    if scale_rows:  # rows of arbitrary length: the channel normalises them
        q *= rng.uniform(0.2, 5.0, (B, T, H, 1))
        k *= rng.uniform(0.2, 5.0, (B, T, H, 1))
    v = rng.standard_normal((B, T, H, D))
    return q.astype(np.float32), k.astype(np.float32), v.astype(np.float32)


def pin_gdelta_orders_agree(mutant=0, bd=None):
    """The literal update S (alpha (I - beta k k^T)) + beta v k^T with the
    matrix built, and its rank-one expansion, agree to rounding."""
    rng = np.random.default_rng(31)
    B, T, H = 2, 40, 2
    q, k, v = _gd_rand(rng, B, T, H)
    a = rng.uniform(0.3, 1.0, (B, T, H))
    b = rng.uniform(0.0, 1.0, (B, T, H))
    S0 = rng.standard_normal((B, H, 64, 64)) * 0.3
    o1, S1 = oracle.gdelta(q, k, v, a, b, S0, literal=True, mutant=mutant, build_dir=bd)
    o0, S0_ = oracle.gdelta(q, k, v, a, b, S0, literal=False, mutant=mutant, build_dir=bd)
    _close(o0, o1, rtol=1e-10, atol=1e-11, what="gdelta orders: o")
    _close(S0_, S1, rtol=1e-10, atol=1e-11, what="gdelta orders: state")


def pin_gdelta_last_write_retrieved(mutant=0, bd=None):
    """With beta = 1 the write replaces whatever the memory returned for the
    (unit) key: S_t k_t = alpha S (k - k (k.k)) + v (k.k) = v_t, whatever the
    history, the decay or S_0.  So a query equal to the key reads v_t back."""
    rng = np.random.default_rng(32)
    B, T, H = 1, 50, 2
    q, k, v = _gd_rand(rng, B, T, H)
    q = (k * 2.0 ** rng.integers(-2, 3, (B, T, H, 1))).astype(np.float32)  # exact rescale
    a = rng.uniform(0.5, 1.0, (B, T, H))
    b = np.ones((B, T, H))
    S0 = rng.standard_normal((B, H, 64, 64))
    for literal in (False, True):
        o, _ = oracle.gdelta(q, k, v, a, b, S0, literal=literal, mutant=mutant, build_dir=bd)
        _close(o, v, rtol=1e-10, atol=1e-10, what=f"gdelta last write (literal={literal})")


def pin_gdelta_orthonormal_store(mutant=0, bd=None):
    """alpha = beta = 1 and keys drawn from a scaled orthonormal basis: the
    memory is a key -> value table.  A query along basis vector e returns the
    value last written under e (an overwrite, not a sum), or zero."""
    rng = np.random.default_rng(33)
    T, D = 60, 64
    basis, _ = np.linalg.qr(rng.standard_normal((D, D)))
    slots = rng.integers(0, 12, size=T)       # repeated slots: overwrites
    qslots = rng.integers(0, 16, size=T)      # 12..15 are never written
    k = (basis[:, slots].T * rng.uniform(0.3, 3.0, (T, 1)))[None, :, None]
    q = (basis[:, qslots].T * rng.uniform(0.3, 3.0, (T, 1)))[None, :, None]
    v = rng.standard_normal((1, T, 1, D))
    ones = np.ones((1, T, 1))
    expect = np.zeros((T, D))
    last = {}
    for t in range(T):
        last[int(slots[t])] = v[0, t, 0]
        expect[t] = last.get(int(qslots[t]), np.zeros(D))
    for literal in (False, True):
        o, _ = oracle.gdelta(q.astype(np.float32), k.astype(np.float32), v.astype(np.float32),
                             ones, ones, literal=literal, mutant=mutant, build_dir=bd)
        _close(o[0, :, 0], expect.astype(np.float32).astype(np.float64), rtol=1e-6, atol=1e-6,
               what=f"gdelta orthonormal store (literal={literal})")


def pin_gdelta_partial_writes(mutant=0, bd=None):
    """alpha = 1, beta = 1/2, the same key and value written n times from an
    empty memory: S_n = (1 - 2^-n) v k^T (each write closes half of the gap),
    so the read with q = k is (1 - 2^-n) v."""
    rng = np.random.default_rng(34)
    T, D = 10, 64
    kk = rng.standard_normal(D)
    vv = rng.standard_normal(D)
    k = np.tile(kk, (1, T, 1, 1)).astype(np.float32)
    v = np.tile(vv, (1, T, 1, 1)).astype(np.float32)
    o, _ = oracle.gdelta(k, k, v, np.ones((1, T, 1)), np.full((1, T, 1), 0.5), mutant=mutant,
                         build_dir=bd)
    vf = vv.astype(np.float32).astype(np.float64)
    for n in range(1, T + 1):
        _close(o[0, n - 1, 0], (1 - 0.5 ** n) * vf, rtol=1e-10, atol=1e-12,
               what=f"gdelta partial write n={n}")


def pin_gdelta_decay_and_reset(mutant=0, bd=None):
    """beta = 0: nothing is written, the state only decays, S_t = (prod alpha)
    S_0 and o_t = (prod_{s<=t} alpha_s) S_0 q_t/|q_t|.  alpha = 0: everything
    is forgotten before the write, S_t = beta_t v_t k_t^T/|k_t|, so
    o_t = beta_t v_t <k_t, q_t>/(|k_t||q_t|)."""
    rng = np.random.default_rng(35)
    B, T, H = 1, 30, 2
    q, k, v = _gd_rand(rng, B, T, H)
    a = rng.uniform(0.7, 1.0, (B, T, H))
    S0 = rng.standard_normal((B, H, 64, 64))
    o, S = oracle.gdelta(q, k, v, a, np.zeros((B, T, H)), S0, mutant=mutant, build_dir=bd)
    qn = q.astype(np.float64) / np.linalg.norm(q.astype(np.float64), axis=-1, keepdims=True)
    cum = np.cumprod(a, axis=1)
    for h in range(H):
        exp = cum[0, :, h, None] * (qn[0, :, h] @ S0[0, h].T)
        _close(o[0, :, h], exp, rtol=1e-10, atol=1e-11, what="gdelta decay only")
        _close(S[0, h], cum[0, -1, h] * S0[0, h], rtol=1e-10, atol=1e-12, what="gdelta decay state")
    b = rng.uniform(0.1, 1.0, (B, T, H))
    o, _ = oracle.gdelta(q, k, v, np.zeros((B, T, H)), b, S0, mutant=mutant, build_dir=bd)
    kn = k.astype(np.float64) / np.linalg.norm(k.astype(np.float64), axis=-1, keepdims=True)
    exp = b[..., None] * v.astype(np.float64) * np.sum(kn * qn, axis=-1, keepdims=True)
    _close(o, exp, rtol=1e-10, atol=1e-12, what="gdelta reset")


def pin_gdelta_invariances(mutant=0, bd=None):
    """The channel sees only the directions of q and k (it normalises them):
    rescaling their rows changes nothing, a common rotation R of every q and k
    leaves o unchanged and turns the final state into S R^T, and the output is
    linear in v (from an empty memory)."""
    rng = np.random.default_rng(36)
    B, T, H = 1, 24, 2
    q, k, v = _gd_rand(rng, B, T, H, scale_rows=False)
    a = rng.uniform(0.5, 1.0, (B, T, H))
    b = rng.uniform(0.0, 1.0, (B, T, H))
    o, S = oracle.gdelta(q, k, v, a, b, mutant=mutant, build_dir=bd)
    sq = rng.uniform(0.1, 10.0, (B, T, H, 1))
    sk = rng.uniform(0.1, 10.0, (B, T, H, 1))
    # powers of two keep the rescaled fp32 rows exact
    sq, sk = 2.0 ** np.round(np.log2(sq)), 2.0 ** np.round(np.log2(sk))
    o2, _ = oracle.gdelta((q * sq).astype(np.float32), (k * sk).astype(np.float32), v, a, b,
                          mutant=mutant, build_dir=bd)
    _close(o2, o, rtol=1e-12, atol=1e-13, what="gdelta row scale")
    R, _ = np.linalg.qr(rng.standard_normal((64, 64)))
    qr = (q.astype(np.float64) @ R.T)
    kr = (k.astype(np.float64) @ R.T)
    # the rotated rows are not fp32-exact: compare against the unrotated run on
    # the same rounded inputs rotated back, within fp32 input rounding
    o3, S3 = oracle.gdelta(qr.astype(np.float32), kr.astype(np.float32), v, a, b,
                           mutant=mutant, build_dir=bd)
    _close(o3, o, rtol=1e-5, atol=1e-5, what="gdelta rotation: o")
    _close(S3, S @ R.T, rtol=1e-5, atol=1e-5, what="gdelta rotation: state")
    o4, _ = oracle.gdelta(q, k, (4.0 * v).astype(np.float32), a, b, mutant=mutant, build_dir=bd)
    _close(o4, 4.0 * o, rtol=1e-12, atol=1e-13, what="gdelta linear in v")


def pin_gdelta_state_carries(mutant=0, bd=None):
    """Running T tokens equals running the first T1 and then the rest from
    the returned state (the state is the whole of the channel's memory)."""
    rng = np.random.default_rng(37)
    B, T, H, T1 = 2, 33, 2, 14
    q, k, v = _gd_rand(rng, B, T, H)
    a = rng.uniform(0.5, 1.0, (B, T, H))
    b = rng.uniform(0.0, 1.0, (B, T, H))
    o, S = oracle.gdelta(q, k, v, a, b, mutant=mutant, build_dir=bd)
    oa, Sa = oracle.gdelta(q[:, :T1], k[:, :T1], v[:, :T1], a[:, :T1], b[:, :T1], mutant=mutant,
                           build_dir=bd)
    ob, Sb = oracle.gdelta(q[:, T1:], k[:, T1:], v[:, T1:], a[:, T1:], b[:, T1:], Sa,
                           mutant=mutant, build_dir=bd)
    _close(np.concatenate([oa, ob], axis=1), o, rtol=1e-12, atol=1e-13, what="gdelta split: o")
    _close(Sb, S, rtol=1e-12, atol=1e-13, what="gdelta split: state")


GDELTA_PINS = [pin_gdelta_orders_agree, pin_gdelta_last_write_retrieved,
               pin_gdelta_orthonormal_store, pin_gdelta_partial_writes,
               pin_gdelta_decay_and_reset, pin_gdelta_invariances, pin_gdelta_state_carries]


ALL_PINS = [pin_modes_agree, pin_uniform, pin_uniform_train_length_constant, pin_closed_form,
            pin_temperature_constants, pin_unit_norm_and_bounded, pin_duplication,
            pin_causality, pin_gqa, pin_decode_matches_prefill, pin_window,
            pin_backward_finite_differences] + GDELTA_PINS
