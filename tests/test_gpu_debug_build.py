"""The bounds-checking build (libgdn_debug.so, -DGDN_BOUNDS_CHECK): every entry point on small
ragged inputs runs through it with its device-side index checks compiled in, trips none of
them (the error word stays clear), and returns the release build's results."""
import pytest
import torch

from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def debug_lib(cuda_device):
    gbuild.build()
    gbuild.build(debug=True)
    gdn.lib()
    L = gdn.load(gdn.DEBUG_LIB_PATH)
    assert L.gdn_bounds_checked() == 1 and gdn.lib().gdn_bounds_checked() == 0
    return L


def both(debug_lib, fn):
    """fn() through the release build, then through the debug build (fresh outputs each time)."""
    rel = fn()
    gdn.check_device_error()
    with gdn.using(debug_lib):
        dbg = fn()
        gdn.check_device_error()  # raises GDNError if a bounds check tripped
    return rel, dbg


def same(a, b):
    if isinstance(a, dict):
        for n in a:
            same(a[n], b[n])
        return
    if isinstance(a, (tuple, list)):
        for x, y in zip(a, b):
            same(x, y)
        return
    if a is None:
        assert b is None
        return
    # the checks only add branches; the arithmetic is the release build's
    torch.testing.assert_close(b, a, rtol=1e-6, atol=1e-6)


def prefill(lengths, H=2, d=128, dt=torch.bfloat16, seed=5):
    return inputs.make_prefill(inputs.PREFILL, "cuda", seed=seed, lengths=lengths, H=H, d=d, dtype=dt)


def test_debug_build_chunked_and_sequential_prefill(debug_lib):
    x = prefill([70, 0, 1, 130])
    S0 = torch.randn(4, 2, 128, 128, device="cuda") * 0.02
    for chunk in (64, 0):
        rel, dbg = both(debug_lib, lambda: gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], S0,
                                                          x["cu_seqlens"], chunk=chunk, y_dtype=torch.float32))
        same(rel, dbg)


def test_debug_build_gated_and_prep_fused_prefill(debug_lib):
    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[65, 3, 200], H=2)
    q, k, v, g, beta = gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                                m["alpha_logit"], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"])
    same(*both(debug_lib, lambda: gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"],
                                           m["beta_logit"], m["alpha_logit"], m["A_log"], m["alpha_bias"],
                                           m["cu_seqlens"], eps=m["eps"])))
    same(*both(debug_lib, lambda: gdn.chunk_fwd_gated(q, k, v, g, beta, m["z"], m["norm_w"], m["eps"], None,
                                                      m["cu_seqlens"])))
    same(*both(debug_lib, lambda: gdn.chunk_fwd_prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"],
                                                     m["beta_logit"], m["alpha_logit"], m["A_log"], m["alpha_bias"],
                                                     cu_seqlens=m["cu_seqlens"], l2_eps=m["eps"],
                                                     y_dtype=torch.float32)))
    y = torch.randn(m["N"], 2, 128, device="cuda").to(torch.bfloat16)
    same(*both(debug_lib, lambda: gdn.out_gate(y, m["z"], m["norm_w"], m["eps"])))


def test_debug_build_decode_steps(debug_lib):
    st0 = inputs.make_decode_state(inputs.DECODE, "cuda", B=6, H=2)
    d = inputs.make_decode_step(inputs.DECODE, "cuda", B=4, H=2)
    slots = torch.tensor([5, 0, 3, 2], dtype=torch.int32, device="cuda")
    states = []

    def dec():
        st = st0.clone()
        states.append(st)
        return gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], st, slots, y_dtype=torch.float32)
    same(*both(debug_lib, dec))
    same(states[0], states[1])

    m = inputs.make_mixer(inputs.MIXER, "cuda", lengths=[4], H=2)
    conv0 = torch.randn(6, m["W"] - 1, 2, 3 * 128, device="cuda").to(m["x_q"].dtype)
    kept = []

    def mdec():
        conv, st = conv0.clone(), st0.clone()
        kept.append((conv, st))
        return gdn.mixer_decode_step(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                                     m["alpha_logit"], m["A_log"], m["alpha_bias"], m["z"], m["norm_w"], conv, st,
                                     slots, l2_eps=m["eps"], rms_eps=m["eps"], out_dtype=torch.float32)
    same(*both(debug_lib, mdec))
    same(kept[0], kept[1])


def test_debug_build_backward_state_maps_and_inproj(debug_lib):
    x = prefill([9, 0, 21], d=32, dt=torch.float32)
    dy = torch.randn(x["N"], 2, 32, device="cuda")
    same(*both(debug_lib, lambda: gdn.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], dy,
                                                cu_seqlens=x["cu_seqlens"])))
    M = torch.randn(3, 2, 128, 128, device="cuda") * 0.05
    B = torch.randn(3, 2, 128, 128, device="cuda")
    S = torch.randn(3, 2, 128, 128, device="cuda")
    same(*both(debug_lib, lambda: gdn.state_map_apply(M, B, S)))
    p = inputs.make_inproj(device="cuda", lengths=[5, 300], D=128)
    same(*both(debug_lib, lambda: gdn.inproj_prep(p["x"], p["w"], p["H"], p["conv_q"], p["conv_k"], p["conv_v"],
                                                  p["A_log"], p["alpha_bias"], p["cu_seqlens"], eps=p["eps"])))
