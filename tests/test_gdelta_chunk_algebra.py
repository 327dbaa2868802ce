"""The chunk-parallel form the memory-channel prefill kernels compute, written
out in fp64 numpy, equals the oracle's token-by-token gated-delta recurrence.

This checks the reformulation (per 64-token chunk: the triangular solve for
the writes, then the three products with the carried state), not the CUDA
code: a wrong decay ratio, mask or sign in the algebra fails here on the CPU.
"""
import numpy as np
import pytest

import oracle

C = 64


def _unit0(x):
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)


def chunked(q, k, v, alpha, beta, S0):
    """One (sequence, head): q, k, v [T, D]; alpha, beta [T]; S0 [D, D]."""
    T, D = q.shape
    S = S0.copy()
    out = np.zeros((T, D))
    for t0 in range(0, T, C):
        n = min(C, T - t0)
        Q = _unit0(q[t0:t0 + n])
        K = _unit0(k[t0:t0 + n])
        V = v[t0:t0 + n]
        be = beta[t0:t0 + n]
        g = np.cumsum(np.maximum(np.log(np.maximum(alpha[t0:t0 + n], 1e-300)), -87.0))
        b = np.exp(g)
        ratio = np.exp(np.tril(g[:, None] - g[None, :]))  # e^{g_t - g_j}, j <= t
        A = np.tril(be[:, None] * ratio * (K @ K.T), -1)
        P = np.tril(ratio * (Q @ K.T))
        Minv = np.linalg.inv(np.eye(n) + A)
        W = Minv @ ((be * b)[:, None] * K)
        Ut = Minv @ (be[:, None] * V)
        U = Ut - W @ S.T
        out[t0:t0 + n] = b[:, None] * (Q @ S.T) + P @ U
        S = b[-1] * S + U.T @ (np.exp(g[-1] - g)[:, None] * K)
    return out, S


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_chunked_form_equals_recurrence(T):
    rng = np.random.default_rng(T)
    H, D = 2, 64
    q = rng.standard_normal((1, T, H, D)).astype(np.float32)
    k = (rng.standard_normal((1, T, H, D)) * rng.uniform(0.2, 4, (1, T, H, 1))).astype(np.float32)
    v = rng.standard_normal((1, T, H, D)).astype(np.float32)
    alpha = rng.uniform(0.5, 1.0, (1, T, H))
    beta = rng.uniform(0.0, 1.0, (1, T, H))
    S0 = 0.3 * rng.standard_normal((1, H, D, D))
    o_ref, S_ref = oracle.gdelta(q, k, v, alpha, beta, S0)
    for h in range(H):
        o, S = chunked(q[0, :, h].astype(np.float64), k[0, :, h].astype(np.float64),
                       v[0, :, h].astype(np.float64), alpha[0, :, h], beta[0, :, h], S0[0, h])
        np.testing.assert_allclose(o, o_ref[0, :, h], rtol=1e-9, atol=1e-10)
        np.testing.assert_allclose(S, S_ref[0, h], rtol=1e-9, atol=1e-10)


def test_chunked_form_with_closed_gates():
    """alpha = 0 somewhere inside a chunk (a full reset there) and beta = 0
    rows: the clamped log gate leaves a factor e^-87 where the recurrence has
    0, far below fp32 resolution of the results."""
    rng = np.random.default_rng(5)
    T, D = 150, 64
    q = rng.standard_normal((1, T, 1, D)).astype(np.float32)
    k = rng.standard_normal((1, T, 1, D)).astype(np.float32)
    v = rng.standard_normal((1, T, 1, D)).astype(np.float32)
    alpha = rng.uniform(0.8, 1.0, (1, T, 1))
    alpha[0, [10, 70, 71, 149], 0] = 0.0
    beta = rng.uniform(0.0, 1.0, (1, T, 1))
    beta[0, [3, 64, 100], 0] = 0.0
    o_ref, S_ref = oracle.gdelta(q, k, v, alpha, beta)
    o, S = chunked(q[0, :, 0].astype(np.float64), k[0, :, 0].astype(np.float64),
                   v[0, :, 0].astype(np.float64), alpha[0, :, 0], beta[0, :, 0], np.zeros((D, D)))
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=1e-9, atol=1e-12)
