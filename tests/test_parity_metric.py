"""CPU checks of the parity metric itself (no GPU): it forgives exactly the output's own
storage rounding and nothing more, so a gain error of a few percent in the gated output of
eq. (11) ("On the design of Qwen3.8-Next architecture", section 2.1.1) cannot pass.  Each
mistake is planted in the oracle's own output on the CPU."""
import numpy as np

import oracle
from parity_metric import UNIT_ROUNDOFF_BY_NAME, excess_rel_err

TOL_16 = 3e-3


def _small_mixer(seed=40):
    rng = np.random.default_rng(seed)
    lengths = [90, 41]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    N, H, d = int(cu[-1]), 2, 16
    c = dict(x_q=rng.standard_normal((N, H, d)), x_k=rng.standard_normal((N, H, d)),
             x_v=rng.standard_normal((N, H, d)), w_q=rng.standard_normal((H * d, 4)) * 0.5,
             w_k=rng.standard_normal((H * d, 4)) * 0.5, w_v=rng.standard_normal((H * d, 4)) * 0.5,
             beta_logit=rng.standard_normal((N, H)), alpha_logit=rng.standard_normal((N, H)),
             A_log=np.log(rng.uniform(1, 16, H)), alpha_bias=rng.standard_normal(H) * 0.5,
             z=rng.standard_normal((N, H, d)), norm_w=rng.standard_normal(d) * 0.02, cu_seqlens=cu)
    out, y, S_T = oracle.mixer(**c)
    return c, out, y


def test_metric_forgives_only_the_storage_rounding():
    _, out, _ = _small_mixer()
    u = UNIT_ROUNDOFF_BY_NAME["bfloat16"]
    rounded = oracle.round_to_format(out, "bf16")
    assert excess_rel_err(rounded, out, u) == 0.0
    # the same rounding judged as an fp32 output is an error of about 2^-9 of max |out|
    assert excess_rel_err(rounded, out, 0.0) > 1e-4


def test_metric_rejects_a_five_percent_gain_error_in_the_gated_output():
    """(1 + w) replaced by (1.05 + w): every element off by about 5 %."""
    c, out, y = _small_mixer()
    wrong = oracle.out_gate(y, c["z"], c["norm_w"] + 0.05)
    u = UNIT_ROUNDOFF_BY_NAME["bfloat16"]
    assert excess_rel_err(oracle.round_to_format(wrong, "bf16"), out, u) > 10 * TOL_16


def test_metric_rejects_one_wrong_row():
    """A single (token, head) row of the gated output scaled by 1 %: still above the bound,
    because the metric is a maximum over elements."""
    _, out, _ = _small_mixer()
    r = np.unravel_index(np.argmax(np.abs(out)), out.shape)
    wrong = out.copy()
    wrong[r[0], r[1], :] *= 1.01
    assert excess_rel_err(wrong, out, 0.0) > TOL_16
    assert excess_rel_err(oracle.round_to_format(wrong, "bf16"), out, UNIT_ROUNDOFF_BY_NAME["bfloat16"]) > TOL_16
