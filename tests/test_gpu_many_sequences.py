"""Many packed sequences (300, lengths 0-200 with empty, one-token and chunk-multiple ones) through
the entry points whose kernels locate their sequence from cu_seqlens: the chunked prefill (its
records, chunk lookup and per-sequence state rows), the gated pass, the backward's checkpoint
blocks and the fused in-projection's conv boundaries; each against the fp64 oracle (eqs. (1)-(4),
(6)-(11) of "On the design of Qwen3.8-Next architecture", section 2.1.1)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs
from parity_metric import excess_rel_err

pytestmark = pytest.mark.gpu

TOL_16 = 3e-3
TOL_32 = 1e-4
UNIT_ROUNDOFF = {torch.float32: 0.0, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    gbuild.build()
    gdn.lib()


def err(gpu, ref):
    return excess_rel_err(gpu.detach().double().cpu().numpy(), np.asarray(ref), UNIT_ROUNDOFF[gpu.dtype])


def many_lengths(seed, n=300):
    rng = np.random.default_rng(seed)
    L = rng.integers(0, 201, n)
    L[rng.choice(n, 20, replace=False)] = 0
    L[rng.choice(n, 20, replace=False)] = 1
    L[rng.choice(n, 20, replace=False)] = 64 * rng.integers(1, 4, 20)
    return [int(x) for x in L]


def test_chunked_prefill_300_sequences():
    lengths = many_lengths(3)
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=31, lengths=lengths, H=2, S0_std=0.1)
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], chunk=64,
                           y_dtype=torch.float32)
    gdn.check_device_error()
    ry, rS = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"])
    ey, es = err(y, ry), err(S_T, rS)
    print(f"300 sequences, N={x['N']}: y {ey:.2e}, S_T {es:.2e}")
    assert ey < TOL_16 and es < TOL_16


def test_gated_prefill_300_sequences():
    lengths = many_lengths(4)
    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=lengths, H=2, seed=41)
    q, k, v, g, beta = gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                                m["alpha_logit"], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"])
    y, _ = gdn.chunk_fwd(q, k, v, g, beta, None, m["cu_seqlens"], chunk=64, y_dtype=torch.float32,
                         final_state=False)
    out, _ = gdn.chunk_fwd_gated(q, k, v, g, beta, m["z"], m["norm_w"], m["eps"], None, m["cu_seqlens"],
                                 final_state=False)
    gdn.check_device_error()
    ry, _ = oracle.recurrence(q, k, v, g, beta, None, m["cu_seqlens"])
    assert err(y, ry) < TOL_16
    # the fused epilogue against eq. (11) applied to the same pass's fp32 y
    assert err(out, oracle.out_gate(y.cpu(), m["z"].cpu(), m["norm_w"].cpu(), m["eps"])) < TOL_32


def test_backward_300_sequences():
    lengths = many_lengths(5)
    x = inputs.make_prefill(inputs.TINY, "cuda", seed=51, lengths=lengths, H=2, d=32, S0_std=0.1)
    dy = torch.randn(x["N"], 2, 32, device="cuda", generator=torch.Generator(device="cuda").manual_seed(9))
    got = gdn.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], dy, x["S0"], cu_seqlens=x["cu_seqlens"])
    gdn.check_device_error()
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dy, x["S0"], cu_seqlens=x["cu_seqlens"])
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert err(got[name], ref[name]) < TOL_32, name


def test_inproj_prep_300_sequences():
    lengths = many_lengths(6)
    m = inputs.make_inproj(device="cuda", lengths=lengths, D=128, seed=61)
    got = gdn.inproj_prep(m["x"], m["w"], m["H"], m["conv_q"], m["conv_k"], m["conv_v"], m["A_log"],
                          m["alpha_bias"], m["cu_seqlens"], eps=m["eps"])
    gdn.check_device_error()
    want = oracle.in_proj_prep(m["x"].cpu(), m["w"].cpu(), m["H"], m["d"], m["conv_q"].cpu(), m["conv_k"].cpu(),
                               m["conv_v"].cpu(), m["A_log"].cpu(), m["alpha_bias"].cpu(),
                               m["cu_seqlens"].cpu().numpy(), eps=m["eps"])
    for name, a, b in zip(("q", "k", "v", "g", "beta", "z"), got, want):
        assert err(a, b) < (TOL_32 if a.dtype == torch.float32 else TOL_16), name
