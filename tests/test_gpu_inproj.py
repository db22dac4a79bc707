"""gdn_inproj_prep: the input projections that eqs. (6)-(11) of "On the design of Qwen3.8-Next
architecture", section 2.1.1, apply to the residual stream x_t (W_q, W_k, W_v, W_z, W_beta,
W_alpha), fused with eqs. (6)-(10), against the fp64 oracle (one fp64 matrix product, then the
pinned prep) on the same bf16 / fp16 bytes."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs
from parity_metric import excess_rel_err

pytestmark = pytest.mark.gpu

TOL_16 = 3e-3   # 16-bit inputs (the stated bound), beyond the output's own rounding
TOL_32 = 1e-4   # fp32 outputs g and beta: only fp32 accumulation and the gate functions differ
UNIT_ROUNDOFF = {torch.float32: 0.0, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}
NAMES = ("q", "k", "v", "g", "beta", "z")


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    gbuild.build()
    gdn.lib()


def err(gpu, ref):
    return excess_rel_err(gpu.detach().double().cpu().numpy(), np.asarray(ref), UNIT_ROUNDOFF[gpu.dtype])


def run(m, out_dtype=None, with_z=True):
    out = gdn.inproj_prep(m["x"], m["w"], m["H"], m["conv_q"], m["conv_k"], m["conv_v"], m["A_log"],
                          m["alpha_bias"], m["cu_seqlens"], eps=m["eps"], out_dtype=out_dtype, with_z=with_z)
    gdn.check_device_error()
    return out


def ref(m):
    return oracle.in_proj_prep(m["x"].cpu(), m["w"].cpu(), m["H"], m["d"], m["conv_q"].cpu(), m["conv_k"].cpu(),
                               m["conv_v"].cpu(), m["A_log"].cpu(), m["alpha_bias"].cpu(), m["cu_seqlens"].cpu().numpy(),
                               eps=m["eps"])


def check_all(got, want, per_head=False, label=""):
    errs = {n: err(a, b) for n, a, b in zip(NAMES, got, want)}
    print(label, " ".join(f"{n} {e:.2e}" for n, e in errs.items()))
    for n in ("q", "k", "v", "z"):
        assert errs[n] < TOL_16, (n, errs[n])
    for n in ("g", "beta"):
        assert errs[n] < TOL_32, (n, errs[n])
    if per_head:
        H = got[0].shape[1]
        for n, a, b in zip(NAMES, got, want):
            for h in range(H):
                assert err(a[:, h], b[:, h]) < (TOL_32 if n in ("g", "beta") else TOL_16), (n, h)


@pytest.mark.parametrize("W", [1, 3, 4, 5, 8])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_inproj_ragged_sequences_every_conv_width(W, dt):
    """Six packed sequences (one empty, one of a single token) over several token blocks, so
    each CTA walks more than one tile and both accumulators; conv widths 1-8 (4- and 8-tap
    kernels); x and w in bf16 and fp16, outputs in the same format."""
    m = inputs.make_inproj(device="cuda", lengths=[1, 700, 0, 411, 3, 388], D=128, W=W, dtype=dt, seed=91 + W)
    check_all(run(m), ref(m), per_head=True, label=f"W={W} {dt}")


@pytest.mark.parametrize("D", [64, 320])
def test_inproj_model_widths(D):
    """One K step (D = 64) and an odd number of them (D = 320)."""
    m = inputs.make_inproj(device="cuda", lengths=[257, 130], D=D, seed=7)
    check_all(run(m), ref(m), label=f"D={D}")


def test_inproj_full_workload_every_head():
    """The workload itself: the mixer's four packed sequences, H = 16, D = 2048, bf16."""
    m = inputs.make_inproj(inputs.INPROJ, "cuda")
    check_all(run(m), ref(m), per_head=True, label="full")


def test_inproj_tokens_past_the_last_sequence_and_no_z():
    """q, k, v of tokens past cu_seqlens[num_seqs] stay as they were; z, g and beta are formed
    for every token.  Without z the other outputs are the same bits."""
    m = inputs.make_inproj(device="cuda", lengths=[100, 160], D=128, seed=3)
    N = m["N"]
    m["x"] = torch.cat([m["x"], torch.randn(60, m["D"], device="cuda").to(m["x"].dtype)])
    cu = m["cu_seqlens"]
    sentinel = 7.0
    H, d = m["H"], m["d"]
    out = tuple(torch.full((N + 60, H, d), sentinel, device="cuda", dtype=torch.bfloat16) for _ in range(3)) + (
        torch.empty(N + 60, H, device="cuda"), torch.empty(N + 60, H, device="cuda"),
        torch.empty(N + 60, H, d, device="cuda", dtype=torch.bfloat16))
    got = gdn.inproj_prep(m["x"], m["w"], H, m["conv_q"], m["conv_k"], m["conv_v"], m["A_log"], m["alpha_bias"], cu,
                          eps=m["eps"], out=out)
    gdn.check_device_error()
    for t in got[:3]:
        assert torch.all(t[N:] == sentinel)
    m2 = dict(m, cu_seqlens=torch.tensor([0, 100, 260, N + 60], dtype=torch.int32, device="cuda"))
    want = ref(m2)  # the oracle over a third sequence holding the extra tokens: its z, g, beta rows
    for n, a, b in zip(NAMES[3:], got[3:], want[3:]):
        assert err(a, b) < (TOL_32 if n != "z" else TOL_16), n
    check_all(tuple(t[:N] for t in got[:3]) + got[3:], tuple(np.asarray(t)[:N] for t in want[:3]) + want[3:],
              label="past-end")
    noz = gdn.inproj_prep(m["x"], m["w"], H, m["conv_q"], m["conv_k"], m["conv_v"], m["A_log"], m["alpha_bias"], cu,
                          eps=m["eps"], with_z=False)
    gdn.check_device_error()
    assert noz[5] is None
    for a, b in zip(noz[:5], got[:5]):
        assert torch.equal(a[:N], b[:N])
