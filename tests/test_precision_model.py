"""fp64 model of the chunked prefill's operand roundings (CPU, no GPU).

The chunk form of eqs. (1)-(4) (derived from eq. (5) of "On the design of Qwen3.8-Next
architecture", section 2.1.1; checked exactly in tests/test_chunk_algebra.py) evaluated in
fp64, with every operand the tensor-core kernels read rounded once to the 16-bit format
they use:
  q, k, v      as stored (bf16 inputs); V enters the U~ product converted to fp16 (exact)
  T_w, W, S    bf16 (the partners of q and k take the input's format)
  T_u, M, U    fp16 (products between computed values)
  U'           bf16 high part plus bf16 rounding remainder (16 significant bits)
Products accumulate in fp64 here (fp32 in TMEM on the GPU).  The model shows the scheme
stays well inside the 3e-3 bound of the GPU parity tests, and that entering U' as a single
bf16 value would cost several times more -- the reason for the hi + lo split.
"""
import numpy as np
import pytest

import oracle
from linear_attention_token_gdn_b200 import inputs

BOUND = 3e-3


def _f64(x):
    return x.double().numpy() if hasattr(x, "double") else np.asarray(x, np.float64)


def _chunk_model(q, k, v, g, beta, cu, u_prime="hi_lo", C=64):
    bf = lambda x: oracle.round_to_format(x, "bf16")
    hf = lambda x: oracle.round_to_format(x, "fp16")
    N, H, dk = q.shape
    dv = v.shape[2]
    y = np.zeros((N, H, dv))
    S_T = np.zeros((len(cu) - 1, H, dk, dv))
    for n in range(len(cu) - 1):
        for h in range(H):
            S = np.zeros((dk, dv))
            for c0 in range(cu[n], cu[n + 1], C):
                c1 = min(c0 + C, cu[n + 1])
                L = c1 - c0
                Q, K, V = q[c0:c1, h], k[c0:c1, h], v[c0:c1, h]
                b = beta[c0:c1, h]
                gam = np.cumsum(g[c0:c1, h])
                D = gam[:, None] - gam[None, :]
                strict = np.tril(np.ones((L, L), bool), -1)
                incl = np.tril(np.ones((L, L), bool))
                A = np.where(strict, b[:, None] * np.exp(np.where(strict, D, 0.0)) * (K @ K.T), 0.0)
                M = hf(np.where(incl, np.exp(np.where(incl, D, 0.0)) * (Q @ K.T), 0.0))
                T = np.linalg.inv(np.eye(L) + A)
                T_w = bf(T * (b * np.exp(gam))[None, :])
                T_u = hf(T * b[None, :])
                W = bf(T_w @ K)
                S_op = bf(S)
                U = T_u @ hf(V) - W @ S_op
                Up = np.exp(gam[-1] - gam)[:, None] * U
                if u_prime == "hi_lo":
                    hi = bf(Up)
                    Up = hi + bf(Up - hi)
                else:
                    Up = bf(Up)
                y[c0:c1, h] = np.exp(gam)[:, None] * (Q @ S_op) + M @ hf(U)
                S = np.exp(gam[-1]) * S + K.T @ Up
            S_T[n, h] = S
    return y, S_T


def _err(a, b):
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


@pytest.fixture(scope="module")
def case():
    # the prefill workload's statistics, shortened: 2 sequences x 1024 tokens, 2 heads
    x = inputs.make_prefill(inputs.PREFILL, "cpu", B=2, T=1024, H=2)
    q, k, v, g, beta = (_f64(x[n]) for n in ("q", "k", "v", "g", "beta"))
    cu = x["cu_seqlens"].numpy()
    y_ref, S_ref = oracle.recurrence(q, k, v, g, beta, None, cu)
    return q, k, v, g, beta, cu, y_ref, S_ref


def test_kernel_rounding_scheme_is_well_inside_the_bound(case):
    q, k, v, g, beta, cu, y_ref, S_ref = case
    y, S_T = _chunk_model(q, k, v, g, beta, cu, "hi_lo")
    ey, es = _err(y, y_ref), _err(S_T, S_ref)
    print(f"model, U' hi + lo: y {ey:.2e}, S_T {es:.2e}")
    assert ey < BOUND / 3 and es < BOUND / 3


def test_single_bf16_u_prime_costs_much_more(case):
    q, k, v, g, beta, cu, y_ref, S_ref = case
    _, S_hl = _chunk_model(q, k, v, g, beta, cu, "hi_lo")
    _, S_1 = _chunk_model(q, k, v, g, beta, cu, "single")
    e_hl, e_1 = _err(S_hl, S_ref), _err(S_1, S_ref)
    print(f"S_T error: U' hi + lo {e_hl:.2e}, single bf16 {e_1:.2e}")
    assert e_1 > 2 * e_hl
