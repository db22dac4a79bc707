"""The seeded input recipes: shapes, dtypes, ranges and determinism (CPU, small overrides)."""
import numpy as np
import torch

from linear_attention_token_gdn_b200 import inputs


def test_prefill_recipe_small():
    a = inputs.make_prefill(inputs.PREFILL, "cpu", T=64, H=3)
    b = inputs.make_prefill(inputs.PREFILL, "cpu", T=64, H=3)
    assert a["q"].dtype == torch.bfloat16 and a["q"].shape == (128, 3, 128)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["g"], b["g"])
    n = a["k"].float().norm(dim=-1)
    assert torch.all((n - 1).abs() < 1e-2)
    alpha = a["g"].exp()
    assert torch.all(alpha > 0) and torch.all(alpha < 1)
    assert torch.all(a["beta"] > 0) and torch.all(a["beta"] < 1)
    assert a["S0"] is None and a["cu_seqlens"].tolist() == [0, 64, 128]


def test_long_prefill_has_initial_state_and_fast_decay():
    a = inputs.make_prefill(inputs.LONG_PREFILL, "cpu", T=256)
    assert a["S0"].shape == (1, 32, 128, 128)
    assert abs(float(a["S0"].std()) - 0.02) < 1e-3
    assert float(a["g"].min()) < -20.0  # exp(A) up to 64 makes some heads decay fast


def test_mixer_lengths_and_packing():
    L = inputs.mixer_lengths(inputs.MIXER)
    assert len(L) == 4 and all(1024 <= x <= 8192 for x in L) and sum(L) <= 32768
    m = inputs.make_mixer(inputs.MIXER, "cpu", lengths=[5, 3])
    assert m["cu_seqlens"].tolist() == [0, 5, 8] and m["x_q"].shape == (8, 16, 128)
    assert m["w_q"].shape == (16 * 128, 4)


def test_decode_recipe():
    st = inputs.make_decode_state(inputs.DECODE, "cpu", B=2, H=2)
    s0 = inputs.make_decode_step(inputs.DECODE, "cpu", step=0, B=2, H=2)
    s1 = inputs.make_decode_step(inputs.DECODE, "cpu", step=1, B=2, H=2)
    assert st.shape == (2, 2, 128, 128) and st.dtype == torch.float32
    assert not torch.equal(s0["q"], s1["q"])
