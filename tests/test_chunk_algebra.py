"""The chunkwise-parallel (WY / UT-transform) form used by the tensor-core prefill kernels,
written out in fp64 numpy and checked against the token-sequential oracle.

The pages define only the recurrence (eqs. 1-5 of "On the design of Qwen3.8-Next
architecture", section 2.1.1); the chunk form is derived from eq. (5).  Unrolling
eqs. (1)-(3) inside a chunk that starts from state S, with gamma_r the inclusive
prefix sum of g = log(alpha) inside the chunk and Gamma_r = exp(gamma_r):

    A[r,s] = beta_r exp(gamma_r - gamma_s) k_r.k_s       (s < r)
    T      = (I + A)^-1
    W      = T diag(beta Gamma) K,   U~ = T diag(beta) V,   U = U~ - W S
    M[r,s] = exp(gamma_r - gamma_s) q_r.k_s               (s <= r)
    Y      = diag(Gamma) Q S + M U
    S'     = Gamma_L S + (diag(Gamma_L / Gamma) K)^T U

Every decay factor used is exp(<= 0), so nothing overflows however fast the decay.
This test pins the derivation, not the oracle; it shares no code with the CUDA kernels.
"""
import numpy as np
import pytest

import oracle


def chunked_forward(q, k, v, g, beta, S0, cu, C):
    N, H, dk = q.shape
    dv = v.shape[2]
    y = np.zeros((N, H, dv))
    S_T = np.zeros((len(cu) - 1, H, dk, dv))
    for n in range(len(cu) - 1):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[n, h].copy()
            for c0 in range(cu[n], cu[n + 1], C):
                c1 = min(c0 + C, cu[n + 1])
                Q, K, V = q[c0:c1, h], k[c0:c1, h], v[c0:c1, h]
                b = beta[c0:c1, h]
                gam = np.cumsum(g[c0:c1, h])
                D = gam[:, None] - gam[None, :]
                low = np.tril(np.ones_like(D), -1) > 0
                A = np.where(low, b[:, None] * np.exp(np.where(low, D, 0.0)) * (K @ K.T), 0.0)
                T = np.linalg.inv(np.eye(c1 - c0) + A)
                W = T @ ((np.exp(gam) * b)[:, None] * K)
                Ut = T @ (b[:, None] * V)
                U = Ut - W @ S
                lowd = np.tril(np.ones_like(D)) > 0
                M = np.where(lowd, np.exp(np.where(lowd, D, 0.0)) * (Q @ K.T), 0.0)
                y[c0:c1, h] = np.exp(gam)[:, None] * (Q @ S) + M @ U
                Kt = np.exp(gam[-1] - gam)[:, None] * K
                S = np.exp(gam[-1]) * S + Kt.T @ U
            S_T[n, h] = S
    return y, S_T


def p_form_end_state(k, g, beta, v, S, C):
    """S' = (Gamma_L I - Kt^T W) S + Kt^T U~: the chunk's affine map on the state."""
    L = k.shape[0]
    gam = np.cumsum(g)
    D = gam[:, None] - gam[None, :]
    low = np.tril(np.ones_like(D), -1) > 0
    A = np.where(low, beta[:, None] * np.exp(np.where(low, D, 0.0)) * (k @ k.T), 0.0)
    T = np.linalg.inv(np.eye(L) + A)
    W = T @ ((np.exp(gam) * beta)[:, None] * k)
    Ut = T @ (beta[:, None] * v)
    Kt = np.exp(gam[-1] - gam)[:, None] * k
    P = np.exp(gam[-1]) * np.eye(k.shape[1]) - Kt.T @ W
    return P @ S + Kt.T @ Ut


def inputs(rng, lengths, H, dk, dv, expA_hi):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    N = int(cu[-1])
    q = rng.standard_normal((N, H, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((N, H, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, H, dv))
    expA = rng.uniform(1.0, expA_hi, H)
    g = -expA[None, :] * np.logaddexp(0.0, rng.standard_normal((N, H)))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((N, H))))
    S0 = rng.standard_normal((len(lengths), H, dk, dv)) * 0.5
    return q, k, v, g, beta, S0, cu


@pytest.mark.parametrize("C", [4, 16, 64])
@pytest.mark.parametrize("expA_hi", [1.001, 16.0, 64.0])
def test_chunk_form_equals_sequential(C, expA_hi):
    rng = np.random.default_rng(C * 100 + int(expA_hi))
    lengths = [3 * C + 5, C, 1, 2 * C - 1]
    q, k, v, g, beta, S0, cu = inputs(rng, lengths, 2, 8, 6, expA_hi)
    y_ref, S_ref = oracle.recurrence(q, k, v, g, beta, S0, cu_seqlens=cu)
    y, S_T = chunked_forward(q, k, v, g, beta, S0, cu, C)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(S_T))
    assert np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)) < 1e-11
    assert np.max(np.abs(S_T - S_ref)) / np.max(np.abs(S_ref)) < 1e-11


def test_affine_chunk_map_equals_sequential():
    rng = np.random.default_rng(7)
    q, k, v, g, beta, S0, cu = inputs(rng, [64], 1, 16, 8, 16.0)
    _, S_ref = oracle.recurrence(q, k, v, g, beta, S0, cu_seqlens=cu)
    S = p_form_end_state(k[:, 0], g[:, 0], beta[:, 0], v[:, 0], S0[0, 0], 64)
    assert np.max(np.abs(S - S_ref[0, 0])) / np.max(np.abs(S_ref)) < 1e-11
