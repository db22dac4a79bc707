"""gdn_chunk_bwd: the reverse-mode derivative of eqs. (1)-(4) of "On the design of Qwen3.8-Next
architecture", section 2.1.1, against the oracle's (itself pinned by central finite differences),
element by element: every input's gradient, for packed ragged sequences, S0 and dS_T given or
not, fp32 and bf16 inputs, every supported head size, and the full prefill workload."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs
from parity_metric import excess_rel_err

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dS0")


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    gbuild.build()
    gdn.lib()


def run(x, dy, dS_T, scale=1.0):
    got = gdn.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], dy, S0=x["S0"], dS_T=dS_T,
                        cu_seqlens=x["cu_seqlens"], scale=scale)
    gdn.check_device_error()
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dy, S0=x["S0"], dS_T=dS_T,
                          cu_seqlens=x["cu_seqlens"], scale=scale)
    return {n: excess_rel_err(got[n].double().cpu().numpy(), ref[n], 0.0) for n in NAMES}


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (128, 16)])
def test_backward_fp32_ragged_matches_the_oracle(dk, dv):
    lengths = [1, 0, 37, 8, 70]
    x = inputs.make_prefill(inputs.TINY, "cuda", lengths=lengths, H=2, dk=dk, dv=dv, S0_std=0.1, seed=95 + dk + dv)
    gen = torch.Generator(device="cuda").manual_seed(96)
    dy = torch.randn(x["N"], 2, dv, device="cuda", generator=gen)
    dS_T = torch.randn(len(lengths), 2, dk, dv, device="cuda", generator=gen) * 0.1
    e = run(x, dy, dS_T, scale=0.9)
    print(f"bwd fp32 dk={dk} dv={dv}: " + ", ".join(f"{n} {v:.1e}" for n, v in e.items()))
    assert all(v < 1e-4 for v in e.values()), e


def test_backward_bf16_without_final_state_gradient():
    x = inputs.make_prefill(inputs.PREFILL, "cuda", B=2, T=300, H=3, seed=97)
    gen = torch.Generator(device="cuda").manual_seed(98)
    dy = torch.randn(x["N"], 3, 128, device="cuda", generator=gen).to(torch.bfloat16)
    e = run(x, dy, None)
    print("bwd bf16: " + ", ".join(f"{n} {v:.1e}" for n, v in e.items()))
    assert all(v < 1e-4 for v in e.values()), e


def test_backward_full_prefill_workload():
    """B=2, H=16, T=4096, dk=dv=128, bf16 q/k/v: every gradient of every head."""
    x = inputs.make_prefill(inputs.PREFILL, "cuda")
    gen = torch.Generator(device="cuda").manual_seed(99)
    dy = torch.randn(x["N"], x["H"], 128, device="cuda", generator=gen).to(torch.bfloat16)
    dS_T = torch.randn(x["num_seqs"], x["H"], 128, 128, device="cuda", generator=gen) * 0.01
    e = run(x, dy, dS_T)
    print("bwd prefill workload: " + ", ".join(f"{n} {v:.1e}" for n, v in e.items()))
    assert all(v < 1e-4 for v in e.values()), e
