"""GPU parity: every entry point of libgdn.so (called through the C ABI via the ctypes
binding) against the fp64 oracle on the same seeded inputs.

Error metric (per output tensor): max over elements of
    max(|gpu - oracle| - u |oracle|, 0) / max |oracle|
where u is the unit roundoff of the output's own storage type (0 for fp32, 2^-11 for
fp16, 2^-8 for bf16): a 16-bit output is a rounding of the computed value, and that
final rounding alone can exceed the arithmetic bounds below.  Bounds:
  * 1e-4 for fp32 inputs (fp32 arithmetic on CUDA cores);
  * 3e-3 for bf16/fp16 inputs with the fp32 state (tensor-core path: fp16 operands,
    fp32 accumulation, fp32 state).
The oracle receives the exact values the GPU receives (16-bit inputs upcast exactly).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs
from parity_metric import excess_rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_16 = 3e-3


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    gbuild.build()
    gdn.lib()


UNIT_ROUNDOFF = {torch.float32: 0.0, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


def err(gpu, ref):
    """The parity metric (tests/parity_metric.py) of a GPU tensor against the oracle."""
    return excess_rel_err(gpu.detach().double().cpu().numpy(), ref, UNIT_ROUNDOFF[gpu.dtype])


# --------------------------------------------------------------- recurrent (chunk=0)

def test_recurrent_tiny_fp32_workload():
    """The tiny workload: B=1, H=2, T=64, dk=dv=16, fp32, S0 = 0."""
    x = inputs.make_prefill(inputs.TINY, "cuda")
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=0)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
    assert err(y, y_ref) < TOL_F32
    assert err(S_T, S_ref) < TOL_F32
    gdn.check_device_error()


@pytest.mark.parametrize("dk,dv", [(16, 32), (64, 16), (128, 128), (32, 64)])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16, torch.float16])
def test_recurrent_varlen_shapes_dtypes(dk, dv, dt):
    lengths = [37, 1, 0, 70]
    x = inputs.make_prefill(inputs.PREFILL, "cuda", seed=11 + dk + dv, lengths=lengths, H=3, dk=dk, dv=dv, dtype=dt,
                            S0_std=0.3)
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], chunk=0,
                           y_dtype=torch.float32)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"])
    assert err(y, y_ref) < TOL_F32
    assert err(S_T, S_ref) < TOL_F32
    gdn.check_device_error()


# --------------------------------------------------------------------- decode

@pytest.mark.parametrize("dk,dv", [(128, 128), (16, 16), (64, 32), (32, 128)])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_decode_steps_with_slots(dk, dv, dt):
    B, H, slots = 5, 3, 9
    state = inputs.make_decode_state(inputs.DECODE, "cuda", seed=5, B=slots, H=H, dk=dk, dv=dv)
    slot = torch.tensor([7, 0, 3, 8, 1], dtype=torch.int32, device="cuda")
    ref_state = state.double().cpu().numpy()
    for step in range(3):
        x = inputs.make_decode_step(inputs.DECODE, "cuda", step=step, seed=5, B=B, H=H, dk=dk, dv=dv, dtype=dt)
        y = gdn.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state, slot, y_dtype=torch.float32)
        y_ref, ref_state = oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], ref_state, slot)
        assert err(y, y_ref) < TOL_F32
        assert err(state, ref_state) < TOL_F32
    gdn.check_device_error()


def test_decode_full_workload_every_head():
    """256 x 32 heads, dk = dv = 128, 100 in-place steps (bf16 q/k/v, bf16 y): the oracle steps
    every (row, head) pair alongside (fp64, in place); y of every pair is checked on four of
    the steps and the whole state after the last one."""
    c = inputs.WORKLOAD_SPECS[inputs.DECODE]
    state = inputs.make_decode_state(inputs.DECODE, "cuda")
    ref = state.double().cpu().numpy()
    checked = {0, 37, 71, c["steps"] - 1}
    for step in range(c["steps"]):
        x = inputs.make_decode_step(inputs.DECODE, "cuda", step=step)
        y = gdn.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state)
        y_ref, ref = oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], ref, inplace=True)
        if step in checked:
            ey = err(y, y_ref)
            assert ey < TOL_F32, (step, ey)
    es = err(state, ref)
    print(f"decode workload: state err {es:.2e} after {c['steps']} steps")
    assert es < TOL_F32
    gdn.check_device_error()


def test_decode_rejects_out_of_range_slot_on_device():
    state = torch.zeros(2, 1, 16, 16, device="cuda")
    x = inputs.make_decode_step(inputs.DECODE, "cuda", B=1, H=1, dk=16, dv=16, dtype=torch.float32)
    gdn.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state,
                    torch.tensor([5], dtype=torch.int32, device="cuda"))
    with pytest.raises(gdn.GDNError) as e:
        gdn.check_device_error()
    assert e.value.status == gdn.GDN_ERR_INVALID_ARG
    assert torch.all(state == 0)


# ------------------------------------------------------------- prep / out gate

@pytest.mark.parametrize("d", [128, 64, 32, 16])
@pytest.mark.parametrize("out_dt", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", ["three_seqs", "edge"])
def test_prep_matches_oracle(d, out_dt, case):
    """Sequences that start inside a 64-token run and runs that start inside a sequence; the
    edge case adds an empty and a one-token sequence, conv width 3 and a ragged last run."""
    if case == "three_seqs":
        m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[33, 5, 64], d=d, H=3)
    else:
        m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[70, 0, 1, 129], d=d, H=2, W=3, seed=77)
    q, k, v, g, beta = gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                                m["alpha_logit"], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"],
                                out_dtype=out_dt)
    ref = oracle.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                      m["alpha_logit"], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"])
    for got, want in zip((q, k, v), ref[:3]):
        assert err(got, want) < TOL_F32
    assert err(g, ref[3]) < TOL_F32
    assert err(beta, ref[4]) < TOL_F32
    gdn.check_device_error()


@pytest.mark.parametrize("dv", [128, 64, 32, 16])
@pytest.mark.parametrize("y_dt,io", [(torch.float32, torch.float32), (torch.float32, torch.bfloat16),
                                     (torch.bfloat16, torch.bfloat16), (torch.float16, torch.float16),
                                     (torch.bfloat16, torch.float32)])
def test_out_gate_matches_oracle(dv, y_dt, io):
    """Every (y, z/out) storage pair and head size; 301 x 3 rows, so the last block is ragged."""
    gen = torch.Generator(device="cuda").manual_seed(3 + dv)
    y = (torch.randn(301, 3, dv, device="cuda", generator=gen) * 2).to(y_dt)
    z = torch.randn(301, 3, dv, device="cuda", generator=gen).to(io)
    w = torch.randn(dv, device="cuda", generator=gen) * 0.02
    out = gdn.out_gate(y, z, w, 1e-6)
    assert out.dtype == io
    ref = oracle.out_gate(y, z, w, 1e-6)
    assert err(out, ref) < TOL_F32


# ---------------------------------------------------------- tensor-core chunked path

@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("y_dt", [torch.float32, torch.bfloat16])
def test_chunk_tc_small_ragged(dt, y_dt):
    """Several chunks per sequence, ragged tails, an empty and a one-token sequence, S0 != 0."""
    lengths = [3 * 64 + 17, 64, 1, 0, 130]
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=21, lengths=lengths, H=3, dtype=dt, S0_std=0.2)
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], chunk=64,
                           y_dtype=y_dt)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"])
    assert err(y, y_ref) < TOL_16
    assert err(S_T, S_ref) < TOL_16
    gdn.check_device_error()


@pytest.mark.parametrize("chunk", [64, 0, "gated"])
def test_chunk_fwd_all_sequences_empty_carries_the_state(chunk):
    """N = 0 with S_T requested: every sequence is empty, so S_T = S0 (zeros without S0)."""
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=27, lengths=[0, 0, 0], H=2, S0_std=0.2)
    assert x["q"].shape[0] == 0
    for S0 in (x["S0"], None):
        if chunk == "gated":
            z = torch.empty(0, 2, 128, device="cuda", dtype=x["q"].dtype)
            w = torch.zeros(128, device="cuda")
            _, S_T = gdn.chunk_fwd_gated(x["q"], x["k"], x["v"], x["g"], x["beta"], z, w, 1e-6, S0, x["cu_seqlens"])
        else:
            _, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, x["cu_seqlens"], chunk=chunk)
        want = torch.zeros_like(S_T) if S0 is None else S0
        assert torch.equal(S_T, want)
    gdn.check_device_error()


@pytest.mark.parametrize("case", ["beta0", "alpha1_beta1", "reset", "mixed"])
def test_chunk_tc_degenerate_gates(case):
    """The chunked tensor-core path at the method's degenerate points, against the oracle:
    beta = 0 (pure decay of S0), alpha = beta = 1 (no decay, full overwrite), g = -60 on every
    token (the state resets each token: decay factors underflow to zero inside the chunk
    masks), and a mix of all three across heads.  Two sequences, ragged tail, S0 != 0."""
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=28, lengths=[150, 77], H=4, S0_std=0.2)
    g, beta = x["g"].clone(), x["beta"].clone()
    if case == "beta0":
        beta.zero_()
    elif case == "alpha1_beta1":
        g.zero_()
        beta.fill_(1.0)
    elif case == "reset":
        g.fill_(-60.0)
    else:
        beta[:, 0] = 0.0
        g[:, 1] = 0.0
        beta[:, 1] = 1.0
        g[:, 2] = -60.0
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], g, beta, x["S0"], x["cu_seqlens"], chunk=64, y_dtype=torch.float32)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], g, beta, x["S0"], x["cu_seqlens"])
    ey, es = err(y, y_ref), err(S_T, S_ref)
    assert ey < TOL_16 and es < TOL_16, (case, ey, es)
    gdn.check_device_error()


@pytest.mark.parametrize("path", ["chunk64", "gated", "chunk0", "prep"])
def test_malformed_cu_seqlens_is_reported(path):
    """cu_seqlens = [0, 640, 0, 640] over N = 640 tokens: the middle sequence runs backwards
    and the third overlaps the first, describing 20 chunks where the workspace holds 13
    records.  Every path clamps the bounds (the chunked pass also its chunk count to the
    workspace), flags GDN_ERR_INVALID_ARG in the device error word and leaves the context
    usable."""
    N, H, d = 640, 2, 128
    gen = torch.Generator(device="cuda").manual_seed(29)
    cu = torch.tensor([0, 640, 0, 640], dtype=torch.int32, device="cuda")
    bf = lambda *shape: torch.randn(*shape, device="cuda", generator=gen).to(torch.bfloat16)
    if path == "prep":
        w = lambda: torch.randn(H * d, 4, device="cuda", generator=gen) * 0.5
        gdn.prep(bf(N, H, d), bf(N, H, d), bf(N, H, d), w(), w(), w(), bf(N, H), bf(N, H),
                 torch.zeros(H, device="cuda"), torch.zeros(H, device="cuda"), cu)
    else:
        x = inputs.make_prefill(inputs.PREFILL, "cuda", seed=29, B=1, T=N, H=H)
        if path == "gated":
            gdn.chunk_fwd_gated(x["q"], x["k"], x["v"], x["g"], x["beta"], bf(N, H, d),
                                torch.zeros(d, device="cuda"), 1e-6, None, cu)
        else:
            gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, cu, chunk=64 if path == "chunk64" else 0)
    with pytest.raises(gdn.GDNError) as e:
        gdn.check_device_error()
    assert e.value.status == gdn.GDN_ERR_INVALID_ARG
    gdn.check_device_error()  # the word was cleared
    # a well-formed call right after is correct
    x = inputs.make_prefill(inputs.PREFILL, "cuda", seed=30, lengths=[100, 28], H=2)
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=64,
                           y_dtype=torch.float32)
    gdn.check_device_error()
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
    assert err(y, y_ref) < TOL_16 and err(S_T, S_ref) < TOL_16


@pytest.mark.parametrize("d", [128, 32])
def test_prep_wide_conv(d):
    """Conv widths 5-8 take the wider (8-tap) kernel instantiation: width 6 against the oracle."""
    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[40, 3, 70], d=d, H=2, W=6, seed=78)
    q, k, v, g, beta = gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                                m["alpha_logit"], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"],
                                out_dtype=torch.float32)
    ref = oracle.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                      m["alpha_logit"], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"])
    for got, want in zip((q, k, v), ref[:3]):
        assert err(got, want) < TOL_F32
    gdn.check_device_error()


def test_chunk_tc_matches_recurrent_path_no_initial_state():
    x = inputs.make_prefill(inputs.PREFILL, "cuda", seed=22, T=256, H=4)
    y1, S1 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=64,
                           y_dtype=torch.float32)
    y0, S0 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=0,
                           y_dtype=torch.float32)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
    assert err(y0, y_ref) < TOL_F32
    assert err(y1, y_ref) < TOL_16 and err(S1, S_ref) < TOL_16


def test_chunk_tc_prefill_workload_full():
    """B=2, H=16, T=4096, dk=dv=128, bf16, S0 = 0, chunk 64: every output checked."""
    x = inputs.make_prefill(inputs.PREFILL, "cuda")
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=64)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
    ey, es = err(y, y_ref), err(S_T, S_ref)
    print(f"prefill workload: y err {ey:.2e}, S_T err {es:.2e}")
    assert ey < TOL_16 and es < TOL_16
    gdn.check_device_error()


def test_chunk_tc_long_prefill_every_head():
    """B=1, H=32, T=32768, S0 ~ N(0, 0.02), exp(A) up to 64: every head and every output."""
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda")
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], chunk=64)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"])
    ey, es = err(y, y_ref), err(S_T, S_ref)
    print(f"long prefill workload: y err {ey:.2e}, S_T err {es:.2e}")
    assert ey < TOL_16 and es < TOL_16
    # per head as well: a head whose outputs are small must not hide behind the global max
    for h in range(x["H"]):
        assert err(y[:, h], y_ref[:, h]) < TOL_16, h
        assert err(S_T[:, h], S_ref[:, h]) < TOL_16, h
    gdn.check_device_error()


def _mixer_call(m, inter):
    """prep with q, k, v stored in `inter` (bf16 or fp16), then the unfused chunked pass
    (fp32 and bf16 y) with the out gate, and the pass with the gate fused, on the same q, k, v."""
    q, k, v, g, beta = gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                                m["alpha_logit"], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"],
                                out_dtype=inter)
    res = {}
    for y_dt in (torch.float32, torch.bfloat16):
        y, S_T = gdn.chunk_fwd(q, k, v, g, beta, None, m["cu_seqlens"], chunk=64, y_dtype=y_dt)
        res[y_dt] = (y, S_T, gdn.out_gate(y, m["z"], m["norm_w"], m["eps"]))
    res["fused"] = gdn.chunk_fwd_gated(q, k, v, g, beta, m["z"], m["norm_w"], m["eps"], None, m["cu_seqlens"])
    gdn.check_device_error()
    return res


@pytest.mark.parametrize("inter", [torch.float16, torch.bfloat16])
def test_full_mixer_workload_every_head(inter):
    """Packed variable-length sequences, H=16, d=128: prep -> chunked recurrence -> out gate
    through the C ABI, and prep -> the chunked pass with the gate fused, against the fp64
    oracle mixer on every head.  q, k, v are stored in `inter` between prep and the
    recurrence, and the oracle rounds them to the same format at the same point.  y and S_T
    meet the tensor-core bound (3e-3, beyond the output's own rounding) in both formats.

    The gated output meets the same bound with fp16 storage, the mixer's configuration.  With
    bf16 storage it is not compared: the GPU's fp32 prep and the oracle's fp64 prep round about
    one stored element in 10^5 to neighbouring bf16 values, and eq. (11)'s per-row RMS
    normalisation amplifies such a one-ulp (0.4 %) input difference past 3e-3 on rows whose y
    is small -- a property of comparing two roundings of different approximations, shown on the
    CPU by tests/test_precision_model.py::test_bf16_storage_double_rounding_alone_exceeds_the_out_bound.
    The fused epilogue is checked on its own in both formats: eq. (11) applied by the oracle to
    the fp32 y of the same chunked pass, within the fp32 bound."""
    m = inputs.make_mixer(inputs.MIXER, "cuda")
    res = _mixer_call(m, inter)
    ref_out, ref_y, ref_S = oracle.mixer(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"],
                                         m["beta_logit"], m["alpha_logit"], m["A_log"], m["alpha_bias"], m["z"],
                                         m["norm_w"], m["cu_seqlens"], eps_l2=m["eps"], eps_rms=m["eps"],
                                         inter_dtype=inter)
    for y_dt in (torch.float32, torch.bfloat16):
        y, S_T, out = res[y_dt]
        ey, es, eo = err(y, ref_y), err(S_T, ref_S), err(out, ref_out)
        print(f"mixer ({inter}, y {y_dt}): y err {ey:.2e}, S_T err {es:.2e}, out err {eo:.2e}")
        assert ey < TOL_16 and es < TOL_16, (y_dt, ey, es)
        if inter == torch.float16:
            assert eo < TOL_16, (y_dt, eo)
            for h in range(m["H"]):
                assert err(out[:, h], ref_out[:, h]) < TOL_16, (y_dt, h)
    out_f, S_f = res["fused"]
    y32 = res[torch.float32][0]
    ef_epi = err(out_f, oracle.out_gate(y32, m["z"], m["norm_w"], m["eps"]))
    ef = err(out_f, ref_out)
    print(f"mixer ({inter}), gate fused: epilogue err {ef_epi:.2e}, out err {ef:.2e}")
    assert ef_epi < TOL_F32
    if inter == torch.float16:
        assert ef < TOL_16
    assert torch.equal(S_f, res[torch.float32][1])


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_chunk_fwd_gated_small_ragged(dt):
    """The fused out gate: ragged tails, an empty and a one-token sequence, S0 != 0.  Its
    epilogue against eq. (11) applied by the oracle to the fp32 y of the unfused pass (fp32
    bound), its output against the oracle's (tensor-core bound), S_T equal to the unfused
    pass's."""
    lengths = [3 * 64 + 17, 64, 1, 0, 130]
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=24, lengths=lengths, H=3, dtype=dt, S0_std=0.2)
    gen = torch.Generator(device="cuda").manual_seed(25)
    N, H, dv = x["v"].shape
    z = torch.randn(N, H, dv, device="cuda", generator=gen).to(dt)
    w = torch.randn(dv, device="cuda", generator=gen) * 0.5
    out, S_T = gdn.chunk_fwd_gated(x["q"], x["k"], x["v"], x["g"], x["beta"], z, w, 1e-6, x["S0"],
                                   x["cu_seqlens"])
    y32, S32 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], chunk=64,
                             y_dtype=torch.float32)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"])
    assert err(out, oracle.out_gate(y32, z, w, 1e-6)) < TOL_F32
    assert err(out, oracle.out_gate(y_ref, z, w, 1e-6)) < TOL_16
    assert err(S_T, S_ref) < TOL_16
    assert torch.equal(S_T, S32)
    gdn.check_device_error()


def test_chunk_fwd_gated_bounded_wait_reports_timeout():
    """The gated variant's cluster exchange waits are bounded too: with a one-cycle budget the
    call flags GDN_ERR_TIMEOUT and every CTA of every cluster still leaves; the next call is
    correct."""
    x = inputs.make_prefill(inputs.PREFILL, "cuda", seed=26, T=256, H=2)
    N, H, dv = x["v"].shape
    z = torch.ones(N, H, dv, device="cuda", dtype=x["q"].dtype)
    w = torch.zeros(dv, device="cuda")
    try:
        gdn.set_wait_budget(1)
        gdn.chunk_fwd_gated(x["q"], x["k"], x["v"], x["g"], x["beta"], z, w, 1e-6, None, x["cu_seqlens"])
        with pytest.raises(gdn.GDNError) as e:
            gdn.check_device_error()
        assert e.value.status == gdn.GDN_ERR_TIMEOUT
    finally:
        gdn.set_wait_budget(0)
    out, _ = gdn.chunk_fwd_gated(x["q"], x["k"], x["v"], x["g"], x["beta"], z, w, 1e-6, None, x["cu_seqlens"])
    gdn.check_device_error()
    y32, _ = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=64,
                           y_dtype=torch.float32)
    y_ref, _ = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
    assert err(out, oracle.out_gate(y32, z, w, 1e-6)) < TOL_F32
    assert err(out, oracle.out_gate(y_ref, z, w, 1e-6)) < TOL_16


def test_bounded_wait_reports_timeout_and_context_survives():
    """Failure detection without a GPU fault: with a one-cycle wait budget every mbarrier
    wait of the chunked kernel gives up, the kernel flags GDN_ERR_TIMEOUT, drains its MMAs,
    frees TMEM and returns; the next call with the default budget is correct again."""
    x = inputs.make_prefill(inputs.PREFILL, "cuda", seed=23, T=256, H=2)
    try:
        gdn.set_wait_budget(1)
        gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=64)
        with pytest.raises(gdn.GDNError) as e:
            gdn.check_device_error()
        assert e.value.status == gdn.GDN_ERR_TIMEOUT
    finally:
        gdn.set_wait_budget(0)
    y, S_T = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=64,
                           y_dtype=torch.float32)
    gdn.check_device_error()
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
    assert err(y, y_ref) < TOL_16 and err(S_T, S_ref) < TOL_16


def test_launch_timing_reports_each_kernel():
    """gdn_timing_start/stop bracket every library launch with events on its stream."""
    x = inputs.make_prefill(inputs.PREFILL, "cuda", seed=31, T=512, H=2)
    gdn.timing_start(16)
    for _ in range(2):
        gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=64)
    gdn.decode_step(*(inputs.make_decode_step(inputs.DECODE, "cuda", B=2, H=2)[k] for k in ("q", "k", "v", "g", "beta")),
                    inputs.make_decode_state(inputs.DECODE, "cuda", B=2, H=2))
    t = gdn.timing_stop()
    assert list(t) == ["chunk_ut_kernel", "chunk_chain_kernel", "decode_step_kernel"]
    assert [c for c, _ in t.values()] == [2, 2, 1]
    assert all(ms > 0 for _, ms in t.values())
    with pytest.raises(gdn.GDNError):
        gdn.timing_stop()  # timing is off again
    gdn.check_device_error()
