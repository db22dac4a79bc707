"""Pins for the fp64 oracle, none of which re-types the oracle's own loop.

Each test ties one oracle function to something the page or the mathematics
fixes independently ("On the design of Qwen3.8-Next architecture", section
2.1.1): the closed form eq. (5), pure decay, exact retrieval with orthonormal
keys, the delta-rule overwrite property, brute-force unrolled products, the
contraction bound, a hand-worked two-token example, and library routines
(scipy FIR filter, logistic function) for the pieces of eqs. (6)-(11).
"""
import math
import os

import numpy as np
import pytest
import scipy.signal
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RTOL = 1e-12


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def rand_inputs(rng, T, H, dk, dv, unit_k=False, S0=True, nseq=1):
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    alpha = rng.uniform(0.05, 0.999, (T, H))
    beta = rng.uniform(0.01, 0.99, (T, H))
    S0a = rng.standard_normal((nseq, H, dk, dv)) * 0.3 if S0 else None
    return q, k, v, np.log(alpha), beta, S0a


# ---------------------------------------------------------------- eq. (5)

@pytest.mark.parametrize("dk,dv", [(5, 3), (3, 7), (16, 16)])
def test_recurrence_matches_closed_form_eq5(dk, dv):
    """Eq. (5): S_t = alpha_t (I - beta_t k k^T) S_{t-1} + beta_t k v^T, an algebraically
    independent restatement of eqs. (1)-(3); y_t = S_t^T q_t (eq. 4).  Unnormalised keys,
    dk != dv so that a transposed state or operand fails."""
    rng = np.random.default_rng(1)
    T, H = 13, 3
    q, k, v, g, beta, S0 = rand_inputs(rng, T, H, dk, dv)
    y, S_T = oracle.recurrence(q, k, v, g, beta, S0)
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kt = k[t, h][:, None]
            S = np.exp(g[t, h]) * (np.eye(dk) - beta[t, h] * kt @ kt.T) @ S + beta[t, h] * kt @ v[t, h][None, :]
            assert rel(y[t, h], S.T @ q[t, h]) < RTOL
        assert rel(S_T[0, h], S) < RTOL


def test_packed_sequences_restart_state():
    """Varlen packing: each sequence starts from its own S0 row and never sees another's tokens."""
    rng = np.random.default_rng(2)
    lengths = [5, 1, 0, 9]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T, H, dk, dv = int(cu[-1]), 2, 4, 6
    q, k, v, g, beta, S0 = rand_inputs(rng, T, H, dk, dv, nseq=len(lengths))
    y, S_T = oracle.recurrence(q, k, v, g, beta, S0, cu_seqlens=cu)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        for h in range(H):
            S = S0[n, h].copy()
            for t in range(a, b):
                kt = k[t, h][:, None]
                S = np.exp(g[t, h]) * (np.eye(dk) - beta[t, h] * kt @ kt.T) @ S + beta[t, h] * kt @ v[t, h][None, :]
                assert rel(y[t, h], S.T @ q[t, h]) < RTOL
            assert rel(S_T[n, h], S) < RTOL


# ------------------------------------------------------------ pure decay

def test_beta_zero_is_pure_decay():
    """beta = 0 leaves only eq. (1): S_t = (prod_{s<=t} alpha_s) S0, y_t = that S_t^T q_t."""
    rng = np.random.default_rng(3)
    T, H, dk, dv = 20, 2, 6, 5
    q, k, v, g, beta, S0 = rand_inputs(rng, T, H, dk, dv)
    beta[:] = 0.0
    y, S_T = oracle.recurrence(q, k, v, g, beta, S0)
    decay = np.cumprod(np.exp(g), axis=0)  # [T, H]
    for h in range(H):
        for t in range(T):
            assert rel(y[t, h], decay[t, h] * S0[0, h].T @ q[t, h]) < RTOL
        assert rel(S_T[0, h], decay[-1, h] * S0[0, h]) < RTOL


# ------------------------------------------------------- exact retrieval

def test_orthonormal_keys_give_exact_retrieval():
    """alpha = beta = 1 with orthonormal keys and S0 = 0: S_t = sum_s k_s v_s^T, so querying
    with an earlier (or the current) key returns exactly that token's value (readout after the
    update, eq. 4)."""
    rng = np.random.default_rng(4)
    dk, dv, T = 16, 9, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :T].T.reshape(T, 1, dk).copy()
    v = rng.standard_normal((T, 1, dv))
    src = np.array([rng.integers(0, t + 1) for t in range(T)])
    src[0] = 0
    src[5] = 5  # the current token itself: needs the post-update state
    q = k[src].copy()
    g = np.zeros((T, 1))
    beta = np.ones((T, 1))
    y, S_T = oracle.recurrence(q, k, v, g, beta)
    assert rel(y[:, 0], v[src, 0]) < 1e-12
    assert rel(S_T[0, 0], k[:, 0].T @ v[:, 0]) < 1e-12


def test_repeated_key_overwrites_association():
    """Delta-rule property (section 2.1.1, after eq. 5): with alpha = beta = 1 and a unit key,
    writing (k, v1) and then (k, v2) leaves S^T k = v2 instead of v1 + v2."""
    rng = np.random.default_rng(5)
    dk, dv = 8, 4
    kk = rng.standard_normal(dk)
    kk /= np.linalg.norm(kk)
    k = np.stack([kk, kk])[:, None, :]
    v = rng.standard_normal((2, 1, dv))
    y, S_T = oracle.recurrence(k, k, v, np.zeros((2, 1)), np.ones((2, 1)))
    assert rel(S_T[0, 0].T @ kk, v[1, 0]) < 1e-12
    assert rel(y[1, 0], v[1, 0]) < 1e-12
    assert rel(y[0, 0], v[0, 0]) < 1e-12


# ---------------------------------------------------- brute-force products

@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_bruteforce_unrolled_products(T):
    """S_T = P_{T:1} S0 + sum_s P_{T:s+1} beta_s k_s v_s^T with P_{b:a} = prod_{r=a..b}
    alpha_r (I - beta_r k_r k_r^T), every product formed as an explicit dk x dk matrix;
    the same for every prefix gives y_t."""
    rng = np.random.default_rng(10 + T)
    H, dk, dv = 2, 4, 3
    q, k, v, g, beta, S0 = rand_inputs(rng, T, H, dk, dv)
    y, S_T = oracle.recurrence(q, k, v, g, beta, S0)
    for h in range(H):
        F = [np.exp(g[r, h]) * (np.eye(dk) - beta[r, h] * np.outer(k[r, h], k[r, h])) for r in range(T)]

        def P(b, a):  # product F_b F_{b-1} ... F_a (identity when a > b)
            M = np.eye(dk)
            for r in range(a, b + 1):
                M = F[r] @ M
            return M

        for t in range(T):
            St = P(t, 0) @ S0[0, h]
            for s in range(t + 1):
                St = St + P(t, s + 1) @ (beta[s, h] * np.outer(k[s, h], v[s, h]))
            assert rel(y[t, h], St.T @ q[t, h]) < 1e-11
            if t == T - 1:
                assert rel(S_T[0, h], St) < 1e-11


# ------------------------------------------------------- contraction bound

def test_contraction_bound_unit_keys():
    """For ||k|| = 1 and alpha, beta in (0,1) (section 2.1.1 after eq. 4):
    ||S_t||_2 <= alpha_t ||S_{t-1}||_2 + beta_t ||v_t||, checked on every prefix."""
    rng = np.random.default_rng(6)
    T, H, dk, dv = 16, 2, 8, 8
    q, k, v, g, beta, S0 = rand_inputs(rng, T, H, dk, dv, unit_k=True)
    prev = np.array([np.linalg.norm(S0[0, h], 2) for h in range(H)])
    for t in range(1, T + 1):
        _, S_t = oracle.recurrence(q[:t], k[:t], v[:t], g[:t], beta[:t], S0)
        for h in range(H):
            n = np.linalg.norm(S_t[0, h], 2)
            assert n <= np.exp(g[t - 1, h]) * prev[h] + beta[t - 1, h] * np.linalg.norm(v[t - 1, h]) + 1e-12
            prev[h] = n


# -------------------------------------------------------- hand-worked case

def test_permuting_heads_permutes_outputs():
    """Heads never interact (each runs its own recurrence): permuting the heads of every input
    permutes y and S_T exactly."""
    rng = np.random.default_rng(61)
    q, k, v, g, beta, S0 = rand_inputs(rng, 13, 4, 5, 3, nseq=2)
    cu = np.array([0, 6, 13])
    perm = np.array([2, 0, 3, 1])
    y, S_T = oracle.recurrence(q, k, v, g, beta, S0, cu)
    yp, S_Tp = oracle.recurrence(q[:, perm], k[:, perm], v[:, perm], g[:, perm], beta[:, perm], S0[:, perm], cu)
    assert np.array_equal(yp, y[:, perm]) and np.array_equal(S_Tp, S_T[:, perm])


def test_hand_worked_two_token_example():
    rows, S_rows = [], []
    with open(os.path.join(GOLDEN, "hand_worked_two_tokens.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("S"):
                S_rows.append([float(x) for x in line.split()[1:]])
            else:
                rows.append([float(x) for x in line.split()[1:]])
    r = np.array(rows)
    k = r[:, 0:2][:, None, :]
    v = r[:, 2:4][:, None, :]
    q = r[:, 4:6][:, None, :]
    g = np.log(r[:, 6:7])
    beta = r[:, 7:8]
    y, S_T = oracle.recurrence(q, k, v, g, beta)
    assert np.max(np.abs(y[:, 0] - r[:, 8:10])) < 1e-14
    assert np.max(np.abs(S_T[0, 0] - np.array(S_rows))) < 1e-14


# ------------------------------------------------------------- decode step

def test_decode_step_equals_one_token_recurrence_with_slots():
    """One decode step per row against state[slot[row]] = the recurrence over one token
    started from that state (eqs. 1-4), pinned here through eq. (5)."""
    rng = np.random.default_rng(7)
    B, H, dk, dv, slots = 3, 2, 5, 4, 6
    q, k, v, g, beta, _ = rand_inputs(rng, B, H, dk, dv)
    state = rng.standard_normal((slots, H, dk, dv))
    slot = np.array([4, 0, 2])
    y, new = oracle.decode_step(q, k, v, g, beta, state, slot)
    for b in range(B):
        for h in range(H):
            kt = k[b, h][:, None]
            S = np.exp(g[b, h]) * (np.eye(dk) - beta[b, h] * kt @ kt.T) @ state[slot[b], h] + beta[b, h] * kt @ v[b, h][None, :]
            assert rel(new[slot[b], h], S) < RTOL
            assert rel(y[b, h], S.T @ q[b, h]) < RTOL
    untouched = [s for s in range(slots) if s not in slot]
    assert np.array_equal(new[untouched], state[untouched])


# ------------------------------------------------------ eqs. (6)-(10): prep

def _prep_case(rng, lengths, H=2, dk=6, dv=5, W=4):
    cu = np.concatenate([[0], np.cumsum(lengths)])
    N = int(cu[-1])
    return dict(
        x_q=rng.standard_normal((N, H, dk)), x_k=rng.standard_normal((N, H, dk)),
        x_v=rng.standard_normal((N, H, dv)), w_q=rng.standard_normal((H * dk, W)) * 0.5,
        w_k=rng.standard_normal((H * dk, W)) * 0.5, w_v=rng.standard_normal((H * dv, W)) * 0.5,
        beta_logit=rng.standard_normal((N, H)), alpha_logit=rng.standard_normal((N, H)),
        A_log=np.log(rng.uniform(1, 16, H)), alpha_bias=rng.standard_normal(H) * 0.5,
        cu_seqlens=cu)


def test_prep_conv_is_causal_fir_filter_then_silu():
    """ShortConv (eqs. 6-8) = causal FIR filter per channel with zero history at each sequence
    start (scipy.signal.lfilter with the taps reversed, so tap W-1 meets the current token),
    then SiLU = x * logistic(x) (scipy.special.expit)."""
    rng = np.random.default_rng(20)
    lengths = [7, 2, 11]
    c = _prep_case(rng, lengths)
    q, k, v, g, beta = oracle.prep(**c)
    H, dv = c["x_v"].shape[1:]
    cu = c["cu_seqlens"]
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        for h in range(H):
            for ch in range(dv):
                taps = c["w_v"][h * dv + ch]
                pre = scipy.signal.lfilter(taps[::-1], [1.0], c["x_v"][a:b, h, ch])
                assert rel(v[a:b, h, ch], pre * scipy.special.expit(pre)) < RTOL


def _l2norm_reference(x, eps):
    """x / sqrt(sum_i x_i^2 + eps) over the last axis (the head dimension)."""
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


@pytest.mark.parametrize("eps", [1e-6, 1e-3])
def test_prep_q_k_are_conv_silu_then_l2norm(eps):
    """Eqs. (6)-(7) on the q and k branches: each channel of x_q (x_k) through its own causal
    FIR filter with w_q (w_k) (scipy.signal.lfilter, taps reversed, zero history at every
    sequence start), SiLU = x logistic(x) (scipy.special.expit), then divided by
    sqrt(sum over the head of x^2 + eps).  x_q, x_k and w_q, w_k are all distinct, so
    convolving q with w_k or building q from x_k fails; one sequence of head 0 has inputs
    scaled by 1e-3, where sum x^2 is comparable to eps, so eps outside the square root
    (x / (|x| + eps)) or a missing eps fails too."""
    rng = np.random.default_rng(24)
    lengths = [7, 2, 11]
    c = _prep_case(rng, lengths, H=2, dk=6)
    cu = c["cu_seqlens"]
    a0, b0 = cu[2], cu[3]
    for key in ("x_q", "x_k"):
        c[key][a0:b0, 0, :] *= 1e-3
    q, k, _, _, _ = oracle.prep(**c, eps=eps)
    H, dk = c["x_q"].shape[1:]
    for out, x, w in ((q, c["x_q"], c["w_q"]), (k, c["x_k"], c["w_k"])):
        want = np.zeros_like(out)
        for n in range(len(lengths)):
            a, b = cu[n], cu[n + 1]
            for h in range(H):
                for ch in range(dk):
                    pre = scipy.signal.lfilter(w[h * dk + ch][::-1], [1.0], x[a:b, h, ch])
                    want[a:b, h, ch] = pre * scipy.special.expit(pre)
        want = _l2norm_reference(want, eps)
        assert rel(out, want) < RTOL
        # the small-input rows really are in the regime where eps matters
        assert np.min(np.linalg.norm(out[a0:b0, 0], axis=-1)) < 0.999


def test_prep_q_k_pins_reject_planted_mistakes():
    """The q/k pin distinguishes the plausible slips: q convolved with w_k, q built from x_k,
    and eps moved outside the square root.  Each slip is planted in a copy of the pinned
    arithmetic on the CPU; the oracle's q must match the correct form and none of the slips."""
    rng = np.random.default_rng(25)
    lengths = [5, 9]
    c = _prep_case(rng, lengths, H=1, dk=4)
    c["x_q"][:, 0, :] *= np.where(np.arange(c["x_q"].shape[0]) < 5, 1e-3, 1.0)[:, None]
    eps = 1e-6
    q, _, _, _, _ = oracle.prep(**c, eps=eps)
    cu = c["cu_seqlens"]

    def branch(x, w, norm):
        o = np.zeros_like(x)
        for n in range(len(lengths)):
            a, b = cu[n], cu[n + 1]
            for ch in range(x.shape[2]):
                pre = scipy.signal.lfilter(w[ch][::-1], [1.0], x[a:b, 0, ch])
                o[a:b, 0, ch] = pre * scipy.special.expit(pre)
        return norm(o)

    good = lambda o: _l2norm_reference(o, eps)
    eps_outside = lambda o: o / (np.linalg.norm(o, axis=-1, keepdims=True) + eps)
    assert rel(q, branch(c["x_q"], c["w_q"], good)) < RTOL
    for wrong in (branch(c["x_q"], c["w_k"], good), branch(c["x_k"], c["w_q"], good),
                  branch(c["x_q"], c["w_q"], eps_outside)):
        assert rel(q, wrong) > 1e-3


def test_prep_one_hot_taps_identity_and_shift():
    rng = np.random.default_rng(21)
    lengths = [4, 6]
    c = _prep_case(rng, lengths, H=1, dk=3, dv=3)
    cu = c["cu_seqlens"]
    silu = lambda x: x * scipy.special.expit(x)
    c["w_v"] = np.tile([0.0, 0.0, 0.0, 1.0], (3, 1))
    _, _, v, _, _ = oracle.prep(**c)
    assert rel(v, silu(c["x_v"])) < RTOL
    c["w_v"] = np.tile([0.0, 0.0, 1.0, 0.0], (3, 1))
    _, _, v, _, _ = oracle.prep(**c)
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        assert np.all(v[a] == 0.0)  # SiLU(0) = 0 at each sequence start
        assert rel(v[a + 1:b], silu(c["x_v"][a:b - 1])) < RTOL


def test_prep_q_k_are_unit_norm_after_l2norm():
    """L2Norm in eqs. (6)-(7): ||q|| = ||k|| = 1 up to the eps inside the square root."""
    rng = np.random.default_rng(22)
    c = _prep_case(rng, [9, 3])
    q, k, _, _, _ = oracle.prep(**c)
    for x in (q, k):
        n2 = np.sum(x * x, axis=-1)
        # ||x/sqrt(ss+eps)||^2 = ss/(ss+eps) with ss >= 0, so 1 - n2 <= eps/ss
        assert np.all(n2 <= 1.0) and np.all(n2 > 1.0 - 1e-3)
        assert np.median(1.0 - n2) < 1e-5


def test_prep_gates_closed_forms():
    """eq. (9): beta = logistic(logit) (scipy.special.expit).
    eq. (10): alpha = exp(-e^A softplus(u + b)) = (1 + e^{u+b})^(-e^A), and A = 0, u + b = 0
    gives alpha = 1/2 exactly."""
    rng = np.random.default_rng(23)
    c = _prep_case(rng, [5, 5])
    _, _, _, g, beta = oracle.prep(**c)
    assert rel(beta, scipy.special.expit(c["beta_logit"])) < RTOL
    u = c["alpha_logit"] + c["alpha_bias"][None, :]
    alpha_closed = (1.0 + np.exp(u)) ** (-np.exp(c["A_log"])[None, :])
    assert rel(np.exp(g), alpha_closed) < 1e-11
    c["A_log"] = np.zeros(2)
    c["alpha_bias"] = np.zeros(2)
    c["alpha_logit"] = np.zeros_like(c["alpha_logit"])
    _, _, _, g, _ = oracle.prep(**c)
    assert np.max(np.abs(np.exp(g) - 0.5)) < 1e-15
    # large argument: softplus(u) -> u, so g -> -e^A u (no overflow in the stable form)
    c["alpha_logit"] = np.full_like(c["alpha_logit"], 800.0)
    _, _, _, g, _ = oracle.prep(**c)
    assert np.all(np.isfinite(g)) and rel(g, -800.0 * np.ones_like(g)) < 1e-12


# ------------------------------------------------------------ eq. (11)

def test_out_gate_special_cases():
    """sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w):
    w = 0 and z large -> unit RMS (up to eps); z = 0 halves it; positive rescaling of y leaves
    it unchanged (up to eps); w = -1 zeroes the output."""
    rng = np.random.default_rng(30)
    N, H, dv = 7, 3, 16
    y = rng.standard_normal((N, H, dv)) * 3.0
    w0 = np.zeros(dv)
    big = np.full((N, H, dv), 40.0)
    out = oracle.out_gate(y, big, w0, eps=0.0)
    assert rel(np.sqrt(np.mean(out ** 2, axis=-1)), np.ones((N, H))) < 1e-12
    out_half = oracle.out_gate(y, np.zeros_like(y), w0, eps=0.0)
    assert rel(out_half, 0.5 * out) < 1e-12
    assert rel(oracle.out_gate(7.5 * y, big, w0, eps=0.0), out) < 1e-12
    assert np.all(oracle.out_gate(y, big, -np.ones(dv)) == 0.0)
    w = rng.standard_normal(dv) * 0.02
    z = rng.standard_normal((N, H, dv))
    out_w = oracle.out_gate(y, z, w, eps=1e-6)
    base = oracle.out_gate(y, big, w0, eps=1e-6)
    assert rel(out_w, base * scipy.special.expit(z) * (1.0 + w)) < 1e-12


def test_mixer_composes_the_three_stages():
    rng = np.random.default_rng(31)
    c = _prep_case(rng, [6, 4], H=2, dk=4, dv=4)
    N = int(c["cu_seqlens"][-1])
    z = rng.standard_normal((N, 2, 4))
    nw = rng.standard_normal(4) * 0.02
    out, y, S_T = oracle.mixer(z=z, norm_w=nw, **c)
    q, k, v, g, beta = oracle.prep(**c)
    y2, S2 = oracle.recurrence(q, k, v, g, beta, None, c["cu_seqlens"])
    assert np.array_equal(y, y2) and np.array_equal(S_T, S2)
    assert np.array_equal(out, oracle.out_gate(y2, z, nw))


def _in_proj_case(rng, lengths, H, d, D, W=4):
    cu = np.concatenate([[0], np.cumsum(lengths)])
    N = int(cu[-1])
    return dict(x=rng.standard_normal((N, D)), H=H, d=d,
                conv_q=rng.standard_normal((H * d, W)) * 0.5, conv_k=rng.standard_normal((H * d, W)) * 0.5,
                conv_v=rng.standard_normal((H * d, W)) * 0.5, A_log=np.log(rng.uniform(1, 16, H)),
                alpha_bias=rng.standard_normal(H) * 0.5, cu_seqlens=cu)


def test_in_proj_prep_with_one_hot_rows_is_prep_of_the_selected_columns():
    """With every weight row one-hot, W x_t picks columns of x exactly, so the projection step
    reduces to indexing and in_proj_prep must equal prep (pinned above) of those columns.  Each
    block (W_q, W_k, W_v, W_z, W_beta, W_alpha) picks its own random columns, so a block taken
    from the wrong rows, a transposed operand or a projection applied after the conv fails."""
    rng = np.random.default_rng(41)
    H, d, D = 2, 4, 13
    c = _in_proj_case(rng, [5, 1, 9], H, d, D)
    hd = H * d
    sel = rng.integers(0, D, size=4 * hd + 2 * H)
    w = np.zeros((4 * hd + 2 * H, D))
    w[np.arange(w.shape[0]), sel] = 1.0
    q, k, v, g, beta, z = oracle.in_proj_prep(w=w, **c)
    x, N = c["x"], c["x"].shape[0]
    cols = [c["x"][:, sel[j * hd:(j + 1) * hd]].reshape(N, H, d) for j in range(4)]
    ref = oracle.prep(cols[0], cols[1], cols[2], c["conv_q"], c["conv_k"], c["conv_v"],
                      x[:, sel[4 * hd:4 * hd + H]], x[:, sel[4 * hd + H:]], c["A_log"], c["alpha_bias"],
                      cu_seqlens=c["cu_seqlens"])
    for a, b in zip((q, k, v, g, beta), ref):
        assert np.array_equal(a, b)
    assert np.array_equal(z, cols[3])


def test_in_proj_prep_projections_by_explicit_sums():
    """The projections themselves, summed term by term in Python: z_t[c] = sum_j W_z[c, j] x_t[j],
    beta_t = logistic(sum_j W_beta[h, j] x_t[j]) (eq. 9) and
    g_t = -exp(A_h) softplus(sum_j W_alpha[h, j] x_t[j] + b_h) (eq. 10)."""
    rng = np.random.default_rng(42)
    H, d, D = 2, 2, 5
    c = _in_proj_case(rng, [3], H, d, D)
    w = rng.standard_normal((4 * H * d + 2 * H, D)) / math.sqrt(D)
    q, k, v, g, beta, z = oracle.in_proj_prep(w=w, **c)
    x, hd = c["x"], H * d
    for t in range(x.shape[0]):
        for h in range(H):
            for i in range(d):
                zz = sum(w[3 * hd + h * d + i, j] * x[t, j] for j in range(D))
                assert abs(z[t, h, i] - zz) < 1e-12
            lb = sum(w[4 * hd + h, j] * x[t, j] for j in range(D))
            la = sum(w[4 * hd + H + h, j] * x[t, j] for j in range(D)) + c["alpha_bias"][h]
            assert abs(beta[t, h] - 1.0 / (1.0 + math.exp(-lb))) < 1e-12
            sp = math.log1p(math.exp(la)) if la < 30 else la
            assert abs(g[t, h] + math.exp(c["A_log"][h]) * sp) < 1e-12


# IEEE 754 binary16: p = 11, emin = -14; bfloat16: p = 8, emin = -126.  The subnormal spacing
# is 2^(emin - p + 1).
@pytest.mark.parametrize("fmt,bits,emin", [("bf16", 8, -126), ("fp16", 11, -14)])
def test_round_to_format_is_single_round_to_nearest_even(fmt, bits, emin):
    """The 16-bit storage rounding of the mixer (one IEEE round-to-nearest-even from fp64):
    every result has at most `bits` significant bits, lies within half a spacing of x, is the
    nearer neighbour, and exact midpoints go to the even significand.  Checked by integer
    arithmetic on the significand, not by a library conversion."""
    rng = np.random.default_rng(33)
    x = rng.standard_normal(200000) * np.exp(rng.uniform(-6, 6, 200000))
    r = oracle.round_to_format(x, fmt)
    m, e = np.frexp(x)
    step = np.ldexp(1.0, np.maximum(e - bits, emin - bits + 1))  # spacing at |x| (subnormals too)
    k = r / step                                        # r in units of the spacing at |x|
    assert np.all(k == np.round(k))                     # representable: an integer multiple
    assert np.all(np.abs(r - x) <= step / 2)            # nearest (within half a spacing)
    # midpoints: x = (2j + 1) step / 2 for integer j goes to the even multiple of step
    j = np.floor(x / step)
    mid = (j + 0.5) * step
    rm = oracle.round_to_format(mid, fmt)
    # (j + 0.5) step may sit at a binade edge where the spacing differs; keep the interior ones
    inside = ((np.frexp(mid)[1] == e) & (np.frexp(j * step)[1] == e) & (np.frexp((j + 1) * step)[1] == e)
              & (e - bits >= emin - bits + 1))
    want = np.where(j % 2 == 0, j * step, (j + 1) * step)
    assert np.all(rm[inside] == want[inside]) and inside.sum() > 100000
    # just above / below a midpoint: away from / towards j
    up = oracle.round_to_format(mid + step * 2.0 ** -20, fmt)
    dn = oracle.round_to_format(mid - step * 2.0 ** -20, fmt)
    assert np.all(up[inside] == ((j + 1) * step)[inside]) and np.all(dn[inside] == (j * step)[inside])


def test_mixer_inter_dtype_rounds_q_k_v_before_the_recurrence():
    rng = np.random.default_rng(34)
    c = _prep_case(rng, [6, 4], H=2, dk=4, dv=4)
    N = int(c["cu_seqlens"][-1])
    z = rng.standard_normal((N, 2, 4))
    nw = rng.standard_normal(4) * 0.02
    out, y, S_T = oracle.mixer(z=z, norm_w=nw, inter_dtype="bf16", **c)
    q, k, v, g, beta = oracle.prep(**c)
    q, k, v = (oracle.round_to_format(t, "bf16") for t in (q, k, v))
    y2, S2 = oracle.recurrence(q, k, v, g, beta, None, c["cu_seqlens"])
    assert np.array_equal(y, y2) and np.array_equal(S_T, S2)
    assert np.array_equal(out, oracle.out_gate(y2, z, nw))


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(32)
    q, k, v, g, beta, S0 = rand_inputs(rng, 40, 5, 8, 8, nseq=2)
    a = oracle.recurrence(q, k, v, g, beta, S0, num_seqs=2, nthreads=1)
    b = oracle.recurrence(q, k, v, g, beta, S0, num_seqs=2, nthreads=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ----------------------------------------------------------------------------------------------
# Reverse-mode derivative of eqs. (1)-(4): pinned by central finite differences of the forward
# oracle, which fix every partial derivative independently of how the backward is written.
# ----------------------------------------------------------------------------------------------

def _fd_case(lengths, H, dk, dv, seed):
    rng = np.random.default_rng(seed)
    N = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    x = dict(q=rng.standard_normal((N, H, dk)) * 0.5, k=rng.standard_normal((N, H, dk)) * 0.5,
             v=rng.standard_normal((N, H, dv)), g=-rng.uniform(0.05, 0.6, (N, H)), beta=rng.uniform(0.1, 0.9, (N, H)),
             S0=rng.standard_normal((len(lengths), H, dk, dv)) * 0.3)
    w = dict(y=rng.standard_normal((N, H, dv)), S=rng.standard_normal((len(lengths), H, dk, dv)))
    return x, w, cu


def _loss(x, w, cu, scale):
    y, S_T = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], cu, scale=scale)
    return float((w["y"] * y).sum() + (w["S"] * S_T).sum())


@pytest.mark.parametrize("lengths,scale", [([5, 3], 1.0), ([70], 0.7), ([0, 4], 1.0)])
def test_backward_matches_central_differences(lengths, scale):
    """Every input (q, k, v, g, beta, S0): the oracle's gradient of L = <w_y, y> + <w_S, S_T>
    against (L(x + h) - L(x - h)) / 2h, element by element.  The 70-token sequence crosses the
    backward's 64-token recomputation block; the empty sequence contributes only dS0 = w_S."""
    H, dk, dv = 2, 3, 2
    x, w, cu = _fd_case(lengths, H, dk, dv, seed=91 + len(lengths))
    grad = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], w["y"], S0=x["S0"], dS_T=w["S"],
                           cu_seqlens=cu, scale=scale)
    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", S0="dS0")
    h = 1e-6
    for name, gname in names.items():
        arr = x[name]
        fd = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = arr[idx]
            arr[idx] = old + h
            lp = _loss(x, w, cu, scale)
            arr[idx] = old - h
            lm = _loss(x, w, cu, scale)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        err = np.abs(grad[gname] - fd).max() / max(np.abs(fd).max(), 1e-12)
        assert err < 1e-6, (name, err)


def test_backward_of_pure_decay_is_closed_form():
    """beta = 0: S_t = alpha_t S_{t-1}, y_t = scale (prod alpha) S0^T q_t.  With one token,
    dq = scale alpha S0 dy, dS0 = alpha (scale q dy^T + dS_T), dg = alpha <scale q dy^T + dS_T, S0>,
    and v, k receive nothing."""
    rng = np.random.default_rng(93)
    dk, dv, scale = 3, 4, 0.8
    q, k, v = rng.standard_normal((1, 1, dk)), rng.standard_normal((1, 1, dk)), rng.standard_normal((1, 1, dv))
    g, beta = np.array([[-0.4]]), np.zeros((1, 1))
    S0, dy, dST = rng.standard_normal((1, 1, dk, dv)), rng.standard_normal((1, 1, dv)), rng.standard_normal((1, 1, dk, dv))
    grad = oracle.backward(q, k, v, g, beta, dy, S0=S0, dS_T=dST, scale=scale)
    a = np.exp(-0.4)
    G = scale * np.outer(q[0, 0], dy[0, 0]) + dST[0, 0]
    assert np.allclose(grad["dq"][0, 0], scale * a * S0[0, 0] @ dy[0, 0])
    assert np.allclose(grad["dS0"][0, 0], a * G)
    assert np.isclose(grad["dg"][0, 0], a * (G * S0[0, 0]).sum())
    assert np.allclose(grad["dv"], 0) and np.allclose(grad["dk"], 0)
