"""Metamorphic GPU checks of the state carry, at sizes where a single comparison with the
oracle could hide a carry bug.  Each compares two ways of computing the same thing through
the C ABI; the recurrence (eqs. (1)-(4) of "On the design of Qwen3.8-Next architecture",
section 2.1.1) fixes that they agree:

* splitting a sequence and passing S_T of the first part as S0 of the second equals one call
  (the state after a prefix is all the recurrence carries);
* packing sequences with cu_seqlens equals one call per sequence (sequences never interact);
* T decode steps equal one prefill over the same T tokens;
* permuting the heads permutes every output (heads never interact);
* the chunkwise form (chunk = 64) equals the token-sequential recurrence (chunk = 0).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs
from parity_metric import excess_rel_err

pytestmark = pytest.mark.gpu

TOL_16 = 3e-3


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    gbuild.build()
    gdn.lib()


def rel(a, b):
    return excess_rel_err(a.double().cpu().numpy(), b.double().cpu().numpy(), 0.0)


@pytest.mark.parametrize("split", [1024, 1000])
def test_split_sequence_chained_through_the_state_equals_one_call(split):
    """Two sequences of 2048 tokens, H=4, S0 != 0: [0, split) then [split, 2048) with S0 = S_T of
    the first part.  At a split on a chunk boundary (1024) both ways run the same chunks on
    the same fp32 state, so they agree bit for bit; elsewhere (1000) the chunks differ and
    they agree within the tensor-core bound.  Both also meet the oracle."""
    T, H = 2048, 4
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=51, B=2, T=T, H=H, S0_std=0.1)
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], None, num_seqs=2, chunk=64,
                           y_dtype=torch.float32)
    parts = []
    for n in range(2):
        sl = slice(n * T, (n + 1) * T)
        xs = {k: x[k][sl] for k in ("q", "k", "v", "g", "beta")}
        a, b = slice(0, split), slice(split, T)
        # fresh copies: every pointer of the ABI is 16-byte aligned
        ya, Sa = gdn.chunk_fwd(*(xs[k][a].clone() for k in ("q", "k", "v", "g", "beta")), x["S0"][n:n + 1].clone(),
                               None, num_seqs=1, chunk=64, y_dtype=torch.float32)
        yb, Sb = gdn.chunk_fwd(*(xs[k][b].clone() for k in ("q", "k", "v", "g", "beta")), Sa, None, num_seqs=1,
                               chunk=64, y_dtype=torch.float32)
        parts.append((torch.cat([ya, yb]), Sb))
    y2 = torch.cat([p[0] for p in parts])
    S2 = torch.cat([p[1] for p in parts])
    gdn.check_device_error()
    if split % 64 == 0:
        assert torch.equal(y2, y) and torch.equal(S2, S_T)
    else:
        assert rel(y2, y) < TOL_16 and rel(S2, S_T) < TOL_16
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], num_seqs=2)
    assert excess_rel_err(y2.cpu().numpy(), y_ref, 0.0) < TOL_16
    assert excess_rel_err(S2.cpu().numpy(), S_ref, 0.0) < TOL_16


@pytest.mark.parametrize("path", ["chunk64", "chunk0"])
def test_packed_sequences_equal_separate_calls(path):
    """Five packed sequences (ragged, one empty, one of a single token) against one call per
    sequence with its own S0 row: the same numbers, bit for bit (a chunk never reads another
    sequence's tokens into its result)."""
    lengths = [300, 1, 0, 129, 64]
    H = 3
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=52, lengths=lengths, H=H, S0_std=0.1)
    chunk = 64 if path == "chunk64" else 0
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], chunk=chunk,
                           y_dtype=torch.float32)
    cu = x["cu_seqlens"].cpu().tolist()
    for n, L in enumerate(lengths):
        a, b = cu[n], cu[n + 1]
        S0n = x["S0"][n:n + 1].clone()
        if L == 0:
            assert torch.equal(S_T[n:n + 1], S0n)
            continue
        yn, Sn = gdn.chunk_fwd(*(x[k][a:b].clone() for k in ("q", "k", "v", "g", "beta")), S0n, None,
                               num_seqs=1, chunk=chunk, y_dtype=torch.float32)
        assert torch.equal(yn, y[a:b]), n
        assert torch.equal(Sn, S_T[n:n + 1]), n
    gdn.check_device_error()


def test_decode_steps_equal_one_prefill():
    """Three sequences of 200 tokens, H=4, S0 != 0: 200 gdn_decode_step calls (fp32 state in
    place) against one gdn_chunk_fwd (chunk 64, tensor cores) over the same tokens: y of every
    step and the final state within the tensor-core bound, and the decode side within fp32
    rounding of the oracle."""
    T, H, B = 200, 4, 3
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=53, B=B, T=T, H=H, S0_std=0.1)
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], None, num_seqs=B, chunk=64,
                           y_dtype=torch.float32)
    state = x["S0"].clone()
    ys = torch.empty_like(y)
    idx = lambda t: torch.arange(B, device="cuda") * T + t  # token t of every sequence
    for t in range(T):
        r = idx(t)
        ys[r] = gdn.decode_step(*(x[k][r].contiguous() for k in ("q", "k", "v", "g", "beta")), state,
                                y_dtype=torch.float32)
    gdn.check_device_error()
    assert rel(ys, y) < TOL_16 and rel(state, S_T) < TOL_16
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], num_seqs=B)
    assert excess_rel_err(ys.cpu().numpy(), y_ref, 0.0) < 1e-4
    assert excess_rel_err(state.cpu().numpy(), S_ref, 0.0) < 1e-4


@pytest.mark.parametrize("chunk", [64, 0])
def test_permuting_heads_permutes_outputs(chunk):
    """Heads are independent recurrences: a permutation of the heads of q, k, v, g, beta and S0
    gives the same permutation of y and S_T, bit for bit (each head's arithmetic is unchanged)."""
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=17, lengths=[300, 77], H=8)
    perm = torch.tensor([5, 2, 7, 0, 3, 6, 1, 4], device="cuda")
    S0 = torch.randn(2, 8, 128, 128, device="cuda") * 0.02
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, x["cu_seqlens"], chunk=chunk,
                           y_dtype=torch.float32)
    px = {n: x[n][:, perm].contiguous() for n in ("q", "k", "v", "g", "beta")}
    yp, S_Tp = gdn.chunk_fwd(px["q"], px["k"], px["v"], px["g"], px["beta"], S0[:, perm].contiguous(),
                             x["cu_seqlens"], chunk=chunk, y_dtype=torch.float32)
    gdn.check_device_error()
    assert torch.equal(yp, y[:, perm]) and torch.equal(S_Tp, S_T[:, perm])


def test_chunkwise_form_equals_token_sequential():
    """gdn_chunk_fwd with chunk = 64 (the tensor-core UT form derived from eq. (5)) against chunk = 0
    (eqs. (1)-(4) token by token in fp32) on the same bf16 inputs, ragged sequences and S0 != 0:
    the tensor-core bound on y and S_T."""
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=23, lengths=[1, 200, 0, 777], H=4)
    S0 = torch.randn(4, 4, 128, 128, device="cuda") * 0.02
    y64, S64 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, x["cu_seqlens"], chunk=64,
                             y_dtype=torch.float32)
    y0, S0_ = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, x["cu_seqlens"], chunk=0,
                            y_dtype=torch.float32)
    gdn.check_device_error()
    ey, es = rel(y64, y0), rel(S64, S0_)
    print(f"chunk 64 vs chunk 0: y {ey:.2e}, S_T {es:.2e}")
    assert ey < TOL_16 and es < TOL_16
