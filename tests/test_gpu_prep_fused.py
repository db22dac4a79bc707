"""gdn_chunk_fwd_prep: eqs. (6)-(10) of "On the design of Qwen3.8-Next architecture", section
2.1.1, fused into the chunked pass (q, k, v computed inside the chunk kernel from the projection
outputs), against the fp64 oracle mixer that rounds q, k, v to the same 16-bit format at the same
point, and against the unfused gdn_prep -> gdn_chunk_fwd on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs
from parity_metric import excess_rel_err

pytestmark = pytest.mark.gpu

TOL_16 = 3e-3
UNIT_ROUNDOFF = {torch.float32: 0.0, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    gbuild.build()
    gdn.lib()


def err(gpu, ref):
    return excess_rel_err(gpu.detach().double().cpu().numpy(), np.asarray(ref), UNIT_ROUNDOFF[gpu.dtype])


def run_both(m, inter, S0=None):
    fused = gdn.chunk_fwd_prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                               m["alpha_logit"], m["A_log"], m["alpha_bias"], S0=S0, cu_seqlens=m["cu_seqlens"],
                               l2_eps=m["eps"], qkv_dtype=inter, y_dtype=torch.float32)
    q, k, v, g, beta = gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                                m["alpha_logit"], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"],
                                out_dtype=inter)
    unfused = gdn.chunk_fwd(q, k, v, g, beta, S0, m["cu_seqlens"], chunk=64, y_dtype=torch.float32)
    gdn.check_device_error()
    return fused, unfused


def oracle_mixer(m, inter, S0=None):
    return oracle.mixer(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                        m["alpha_logit"], m["A_log"], m["alpha_bias"], m["z"], m["norm_w"], m["cu_seqlens"],
                        S0=S0, eps_l2=m["eps"], eps_rms=m["eps"], inter_dtype=inter)


@pytest.mark.parametrize("inter", [torch.float16, torch.bfloat16])
def test_fused_prep_full_mixer_workload(inter):
    """The mixer workload (4 packed sequences, ragged lengths, H=16): y and S_T within the
    tensor-core bound of the oracle on every head, and within it of the unfused path."""
    m = inputs.make_mixer(inputs.MIXER, "cuda")
    (y, S_T), (yu, Su) = run_both(m, inter)
    _, ref_y, ref_S = oracle_mixer(m, inter)
    ey, es = err(y, ref_y), err(S_T, ref_S)
    print(f"fused prep ({inter}): y err {ey:.2e}, S_T err {es:.2e}; "
          f"vs unfused: y {err(y, yu.double().cpu().numpy()):.2e}, S_T {err(S_T, Su.double().cpu().numpy()):.2e}")
    assert ey < TOL_16 and es < TOL_16
    for h in range(m["H"]):
        assert err(y[:, h], ref_y[:, h]) < TOL_16, h
    assert err(y, yu.double().cpu().numpy()) < TOL_16 and err(S_T, Su.double().cpu().numpy()) < TOL_16


@pytest.mark.parametrize("W", [4, 1, 8])
def test_fused_prep_ragged_short_sequences(W):
    """Sequences shorter than a chunk, one token long and empty, conv widths 1, 4 and 8 (the
    zero history at every sequence start), with S0 != 0."""
    lengths = [1, 70, 0, 130, 5, 64]
    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=lengths, H=3, W=W, seed=81 + W)
    gen = torch.Generator(device="cuda").manual_seed(82)
    S0 = torch.randn(len(lengths), 3, 128, 128, device="cuda", generator=gen) * 0.02
    (y, S_T), _ = run_both(m, torch.float16, S0=S0)
    _, ref_y, ref_S = oracle_mixer(m, torch.float16, S0=S0)
    ey, es = err(y, ref_y), err(S_T, ref_S)
    print(f"fused prep W={W}: y err {ey:.2e}, S_T err {es:.2e}")
    assert ey < TOL_16 and es < TOL_16
