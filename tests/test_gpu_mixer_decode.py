"""GPU parity of gdn_mixer_decode_step: one token per row through the whole mixer (eqs.
(6)-(11) of "On the design of Qwen3.8-Next architecture", section 2.1.1) in one kernel,
against the fp64 oracle mixer run over the same tokens as whole sequences.

Feeding a sequence to the decode step token by token, starting from a zero conv history and
the sequence's initial state, must give the mixer's output for every token: the conv history
the kernel keeps is exactly the W-1 previous raw inputs the causal ShortConv of eqs. (6)-(8)
reads.  q, k, v stay fp32 inside the kernel, so the oracle keeps them in fp64 (no storage
rounding) and the fp32 bound applies."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs
from parity_metric import excess_rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
UNIT_ROUNDOFF = {torch.float32: 0.0, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    gbuild.build()
    gdn.lib()


def err(gpu, ref):
    return excess_rel_err(gpu.detach().double().cpu().numpy(), ref, UNIT_ROUNDOFF[gpu.dtype])


def run_decode(m, B, T, S0, slots=None, num_slots=None, out_dtype=torch.float32):
    """Rows b = 0..B-1 are sequences of T tokens packed one after another in m's tensors."""
    H, d, W = m["H"], m["d"], m["W"]
    ns = B if num_slots is None else num_slots
    conv = torch.zeros(ns, max(W - 1, 0), H, 3 * d, device="cuda", dtype=m["x_q"].dtype)
    state = torch.zeros(ns, H, d, d, device="cuda")
    rows = torch.arange(B, device="cuda") if slots is None else slots.long()
    if S0 is not None:
        state[rows] = S0
    outs = torch.empty(B * T, H, d, device="cuda", dtype=out_dtype)
    for t in range(T):
        idx = torch.arange(B, device="cuda") * T + t
        pick = lambda x: x[idx].contiguous()
        outs[idx] = gdn.mixer_decode_step(pick(m["x_q"]), pick(m["x_k"]), pick(m["x_v"]), m["w_q"], m["w_k"],
                                          m["w_v"], pick(m["beta_logit"]), pick(m["alpha_logit"]), m["A_log"],
                                          m["alpha_bias"], pick(m["z"]), m["norm_w"],
                                          conv if W > 1 else None, state, slots, l2_eps=m["eps"], rms_eps=m["eps"],
                                          out_dtype=out_dtype)
    gdn.check_device_error()
    return outs, state[rows], conv[rows] if W > 1 else None


def oracle_mixer(m, S0):
    return oracle.mixer(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                        m["alpha_logit"], m["A_log"], m["alpha_bias"], m["z"], m["norm_w"], m["cu_seqlens"], S0=S0,
                        eps_l2=m["eps"], eps_rms=m["eps"])


@pytest.mark.parametrize("d,W", [(128, 4), (32, 4), (64, 6), (16, 1)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_mixer_decode_matches_the_oracle_mixer_token_by_token(d, W, out_dtype):
    B, T, H = 3, 40, 2
    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[T] * B, d=d, H=H, W=W, seed=61 + d + W)
    gen = torch.Generator(device="cuda").manual_seed(62)
    S0 = torch.randn(B, H, d, d, device="cuda", generator=gen) * 0.05
    outs, S_T, conv = run_decode(m, B, T, S0, out_dtype=out_dtype)
    ref_out, _, ref_S = oracle_mixer(m, S0)
    eo, es = err(outs, ref_out), err(S_T, ref_S)
    print(f"mixer decode d={d} W={W} {out_dtype}: out err {eo:.2e}, state err {es:.2e}")
    assert eo < TOL_F32 and es < TOL_F32
    if W > 1:  # the history is the last W-1 raw inputs of each row, bit for bit
        last = torch.arange(B, device="cuda")[:, None] * T + torch.arange(T - (W - 1), T, device="cuda")[None, :]
        want = torch.cat([m["x_q"][last], m["x_k"][last], m["x_v"][last]], dim=-1)  # [B, W-1, H, 3d]
        assert torch.equal(conv, want)


def test_mixer_decode_with_state_slots_and_a_short_sequence():
    """Rows map to permuted slots of larger state and conv-history pools; the oracle runs the
    same sequences.  Eight steps with conv width 4 cover the warm-up of the history."""
    B, T, H, d = 4, 8, 3, 128
    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[T] * B, d=d, H=H, seed=63)
    slots = torch.tensor([5, 0, 3, 6], dtype=torch.int32, device="cuda")
    outs, S_T, _ = run_decode(m, B, T, None, slots=slots, num_slots=7)
    ref_out, _, ref_S = oracle_mixer(m, None)
    assert err(outs, ref_out) < TOL_F32 and err(S_T, ref_S) < TOL_F32


def test_mixer_decode_rejects_an_out_of_range_slot_on_device():
    B, H, d = 1, 1, 16
    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[1], d=d, H=H, seed=64)
    conv = torch.zeros(2, 3, H, 3 * d, device="cuda", dtype=m["x_q"].dtype)
    state = torch.zeros(2, H, d, d, device="cuda")
    gdn.mixer_decode_step(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                          m["alpha_logit"], m["A_log"], m["alpha_bias"], m["z"], m["norm_w"], conv, state,
                          torch.tensor([9], dtype=torch.int32, device="cuda"))
    with pytest.raises(gdn.GDNError) as e:
        gdn.check_device_error()
    assert e.value.status == gdn.GDN_ERR_INVALID_ARG
    assert torch.all(state == 0) and torch.all(conv == 0)


def test_mixer_decode_full_workload_every_row_and_head():
    """The benchmarked launch: 256 rows x 32 heads (8,192 CTAs), d = 128, conv width 4, bf16
    inputs, a resident state ~ N(0, 0.05).  Four steps per row fill the conv history; every
    output of every step and the whole final state are checked against the oracle mixer."""
    B, T, H, d = 256, 4, 32, 128
    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[T] * B, d=d, H=H, seed=65)
    S0 = inputs.make_decode_state(inputs.DECODE, "cuda", B=B, H=H)
    outs, S_T, _ = run_decode(m, B, T, S0)
    ref_out, _, ref_S = oracle_mixer(m, S0)
    eo, es = err(outs, ref_out), err(S_T, ref_S)
    print(f"full mixer decode: out {eo:.2e}, state {es:.2e}")
    assert eo < TOL_F32 and es < TOL_F32
