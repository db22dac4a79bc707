"""Context-parallel prefill on one GPU: the sequences are split into segments as ranks would
hold them, each segment's affine maps are formed through gdn_chunk_fwd, and the ranks' final
passes start from the states that gdn_state_map_apply folds from the earlier segments' maps (the
all-gather is replaced by the list of all segments' maps, which is what it delivers).  Compared
with the oracle's single pass over the whole sequences (eq. 5 of "On the design of Qwen3.8-Next
architecture", section 2.1.1, makes each segment affine in its start state)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import cp, gdn, inputs
from parity_metric import excess_rel_err

pytestmark = pytest.mark.gpu

TOL_TC = 3e-3
UNIT_ROUNDOFF = {torch.float32: 0.0, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    gbuild.build()
    gdn.lib()


def err(gpu, ref):
    return excess_rel_err(gpu.detach().double().cpu().numpy(), np.asarray(ref), UNIT_ROUNDOFF[gpu.dtype])


@pytest.mark.parametrize("rows,dk,dv,with_b", [(3, 128, 128, True), (2, 64, 32, True), (5, 16, 128, False)])
def test_state_map_apply_is_m_s_plus_b(rows, dk, dv, with_b):
    gen = torch.Generator(device="cuda").manual_seed(71 + dk + dv)
    M = torch.randn(rows, dk, dk, device="cuda", generator=gen) / dk ** 0.5
    S = torch.randn(rows, dk, dv, device="cuda", generator=gen)
    B = torch.randn(rows, dk, dv, device="cuda", generator=gen) if with_b else None
    out = gdn.state_map_apply(M, B, S)
    ref = M.double().cpu().numpy() @ S.double().cpu().numpy()
    if with_b:
        ref = ref + B.double().cpu().numpy()
    assert np.abs(out.double().cpu().numpy() - ref).max() <= 1e-5 * np.abs(ref).max()


def test_state_map_apply_refuses_in_place():
    M = torch.zeros(1, 16, 16, device="cuda")
    S = torch.zeros(1, 16, 16, device="cuda")
    with pytest.raises(gdn.GDNError):
        gdn.state_map_apply(M, None, S, S_out=S)


def part(x, T, a, b):
    """Tokens [a, b) of each of the sequences (all T long) packed in x, as one rank holds them."""
    idx = torch.cat([torch.arange(a, b) + s * T for s in range(x["num_seqs"])]).to(x["q"].device)
    p = {n: x[n].index_select(0, idx).contiguous() for n in ("q", "k", "v", "g", "beta")}
    n = b - a
    p["cu_seqlens"] = torch.arange(x["num_seqs"] + 1, device=x["q"].device, dtype=torch.int32) * n
    return p


def test_segment_maps_match_the_oracle():
    """M = the segment from S0 = I with v = 0, B = the segment from S0 = 0 (tensor-core path)."""
    x = inputs.make_prefill(inputs.PREFILL, "cuda", B=2, T=320, H=2, seed=72)
    M, B = cp.segment_maps(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=x["cu_seqlens"])
    eye = np.broadcast_to(np.eye(128), (2, 2, 128, 128)).copy()
    _, M_ref = oracle.recurrence(x["q"], x["k"], torch.zeros_like(x["v"]), x["g"], x["beta"], eye, x["cu_seqlens"])
    _, B_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
    assert err(M, M_ref) < TOL_TC and err(B, B_ref) < TOL_TC


@pytest.mark.parametrize("segs,S0_std", [([256, 200, 312], 0.02), ([448, 320], 0.0)])
def test_emulated_context_parallel_prefill_matches_one_pass(segs, S0_std):
    T = sum(segs)
    x = inputs.make_prefill(inputs.PREFILL, "cuda", B=2, T=T, H=4, S0_std=S0_std, seed=73 + len(segs))
    bounds = np.concatenate([[0], np.cumsum(segs)])
    parts = [part(x, T, int(bounds[r]), int(bounds[r + 1])) for r in range(len(segs))]
    maps = [cp.segment_maps(p["q"], p["k"], p["v"], p["g"], p["beta"], cu_seqlens=p["cu_seqlens"]) for p in parts]
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"])
    S_T = None
    for r, p in enumerate(parts):
        y, S_T = cp.finish(maps, r, p["q"], p["k"], p["v"], p["g"], p["beta"], S0=x["S0"], cu_seqlens=p["cu_seqlens"])
        a, b = int(bounds[r]), int(bounds[r + 1])
        ref = np.concatenate([y_ref[s * T + a:s * T + b] for s in range(2)])
        e = err(y, ref)
        print(f"segments {segs}, rank {r}: y err {e:.2e}")
        assert e < TOL_TC
    e = err(S_T, S_ref)
    print(f"segments {segs}: final state err {e:.2e}")
    assert e < TOL_TC
