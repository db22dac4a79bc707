"""fp64 CPU oracle for the Gated DeltaNet token mixer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product library never calls
it, and it shares no code with the CUDA path: the arithmetic lives in
``gdn_oracle.c`` (plain C, fp64, one thread per independent (sequence, head)
unit), which this module compiles with gcc on first use and calls via ctypes.

Every function follows "On the design of Qwen3.8-Next architecture"
(paper-archivist reading of arXiv 2608.30320), section 2.1.1:

* :func:`recurrence`  -- eqs. (1)-(4), token by token ("Gated Delta recurrence").
* :func:`decode_step` -- the same four equations for one token per row,
  against a state updated in place.
* :func:`prep`        -- eqs. (6)-(10) ("GDN parameterisation").
* :func:`in_proj_prep` -- the input projections W_q x, W_k x, W_v x, W_beta x, W_alpha x
  and W_z x of eqs. (6)-(11), then eqs. (6)-(10).
* :func:`out_gate`    -- eq. (11) without the output projection W_o.
* :func:`mixer`       -- prep -> recurrence -> out_gate in fp64 (optionally with q, k, v
  rounded once to a 16-bit storage format between prep and the recurrence,
  :func:`round_to_format`).

The pins that tie these functions to the page (closed form eq. (5), pure decay,
exact retrieval, brute-force products, textbook special cases, a hand-worked
example) are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``liboracle.so`` (gcc, -O2, fp64, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_recurrence.argtypes = [_D, _D, _D, _D, _D, _D, _I64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_double, _D, _D,
                                              ctypes.c_int]
            lib.oracle_prep.argtypes = [_D, _D, _D, _D, _D, _D, ctypes.c_int, _D, _D, _D, _D, _I64,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_double, _D, _D, _D, _D, _D, ctypes.c_int]
            lib.oracle_out_gate.argtypes = [_D, _D, _D, ctypes.c_double, ctypes.c_long, ctypes.c_int,
                                            ctypes.c_int, _D]
            lib.oracle_decode_step.argtypes = [_D, _D, _D, _D, _D, _D, _I64, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_double, _D, ctypes.c_int]
            lib.oracle_backward.argtypes = [_D, _D, _D, _D, _D, _D, _I64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_double, _D, _D, _D, _D, _D, _D, _D, _D,
                                            ctypes.c_int]
            lib.oracle_threads_used.argtypes = [ctypes.c_int, ctypes.c_long]
            lib.oracle_threads_used.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x):
    """Exact upcast to a C-contiguous float64 array (torch tensors of any float dtype accepted)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch  # only to read a caller's tensor; the oracle itself uses no torch arithmetic
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_D)


def _cu(cu_seqlens, n_tokens, num_seqs):
    if cu_seqlens is None:
        assert n_tokens % num_seqs == 0
        L = n_tokens // num_seqs
        cu = np.arange(num_seqs + 1, dtype=np.int64) * L
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    assert cu.ndim == 1 and cu[0] == 0 and np.all(np.diff(cu) >= 0) and cu[-1] <= n_tokens
    return cu


def threads_used(nthreads: int, n_units: int) -> int:
    return _load().oracle_threads_used(nthreads, n_units)


def recurrence(q, k, v, g, beta, S0=None, cu_seqlens=None, num_seqs=1, scale=1.0, nthreads=0):
    """Eqs. (1)-(4) for packed sequences.

    q, k: [N, H, dk]; v: [N, H, dv]; g = log(alpha), beta: [N, H];
    S0: [num_seqs, H, dk, dv] or None (zeros); cu_seqlens: [num_seqs+1] or None
    (equal lengths).  Returns (y [N, H, dv], S_T [num_seqs, H, dk, dv]) in float64.
    """
    q, k, v, g, beta, S0 = (_f64(t) for t in (q, k, v, g, beta, S0))
    N, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        num_seqs = len(cu_seqlens) - 1
    cu = _cu(cu_seqlens, N, num_seqs)
    assert k.shape == (N, H, dk) and v.shape == (N, H, dv) and g.shape == (N, H) and beta.shape == (N, H)
    if S0 is not None:
        assert S0.shape == (num_seqs, H, dk, dv)
    y = np.zeros((N, H, dv))
    S_T = np.zeros((num_seqs, H, dk, dv))
    _load().oracle_recurrence(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                              cu.ctypes.data_as(_I64), num_seqs, H, dk, dv, float(scale),
                              _ptr(y), _ptr(S_T), int(nthreads))
    return y, S_T


def backward(q, k, v, g, beta, dy, S0=None, dS_T=None, cu_seqlens=None, num_seqs=1, scale=1.0, nthreads=0):
    """Reverse-mode gradients through eqs. (1)-(4): for a loss L with dL/dy = dy and
    dL/dS_T = dS_T (None: zero), returns dict(dq, dk, dv, dg, dbeta, dS0) in float64 (dg is
    the gradient with respect to g = log alpha)."""
    q, k, v, g, beta, S0, dy, dS_T = (_f64(t) for t in (q, k, v, g, beta, S0, dy, dS_T))
    N, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        num_seqs = len(cu_seqlens) - 1
    cu = _cu(cu_seqlens, N, num_seqs)
    out = dict(dq=np.zeros((N, H, dk)), dk=np.zeros((N, H, dk)), dv=np.zeros((N, H, dv)), dg=np.zeros((N, H)),
               dbeta=np.zeros((N, H)), dS0=np.zeros((num_seqs, H, dk, dv)))
    _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), cu.ctypes.data_as(_I64),
                            num_seqs, H, dk, dv, float(scale), _ptr(dy), _ptr(dS_T), _ptr(out["dq"]),
                            _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dS0"]),
                            int(nthreads))
    return out


def decode_step(q, k, v, g, beta, state, state_slot=None, scale=1.0, nthreads=0, inplace=False):
    """One token per row: eqs. (1)-(4) against ``state`` [slots, H, dk, dv].

    Returns (y [B, H, dv], new_state) in float64.  The input state is not modified, unless
    ``inplace`` is set and ``state`` is already a C-contiguous float64 array, which is then
    updated and returned (long multi-step checks avoid copying the whole state every step).
    """
    q, k, v, g, beta = (_f64(t) for t in (q, k, v, g, beta))
    if inplace:
        assert isinstance(state, np.ndarray) and state.dtype == np.float64 and state.flags.c_contiguous
        st = state
    else:
        st = _f64(state).copy()
    B, H, dk = q.shape
    dv = v.shape[2]
    slot = None
    if state_slot is not None:
        if hasattr(state_slot, "detach"):
            state_slot = state_slot.detach().cpu().numpy()
        slot = np.ascontiguousarray(state_slot, dtype=np.int64)
        assert slot.shape == (B,) and slot.min() >= 0 and slot.max() < st.shape[0]
    else:
        assert st.shape[0] >= B
    y = np.zeros((B, H, dv))
    _load().oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(st),
                               None if slot is None else slot.ctypes.data_as(_I64),
                               B, H, dk, dv, float(scale), _ptr(y), int(nthreads))
    return y, st


def prep(x_q, x_k, x_v, w_q, w_k, w_v, beta_logit, alpha_logit, A_log, alpha_bias,
         cu_seqlens=None, num_seqs=1, eps=1e-6, nthreads=0):
    """Eqs. (6)-(10).  Returns (q, k, v, g = log alpha, beta) in float64."""
    x_q, x_k, x_v, w_q, w_k, w_v, bl, al, A, ba = (
        _f64(t) for t in (x_q, x_k, x_v, w_q, w_k, w_v, beta_logit, alpha_logit, A_log, alpha_bias))
    N, H, dk = x_q.shape
    dv = x_v.shape[2]
    W = w_q.shape[1]
    assert w_q.shape == (H * dk, W) and w_k.shape == (H * dk, W) and w_v.shape == (H * dv, W)
    if cu_seqlens is not None:
        num_seqs = len(cu_seqlens) - 1
    cu = _cu(cu_seqlens, N, num_seqs)
    q = np.zeros((N, H, dk)); k = np.zeros((N, H, dk)); v = np.zeros((N, H, dv))
    g = np.zeros((N, H)); beta = np.zeros((N, H))
    _load().oracle_prep(_ptr(x_q), _ptr(x_k), _ptr(x_v), _ptr(w_q), _ptr(w_k), _ptr(w_v), W,
                        _ptr(bl), _ptr(al), _ptr(A), _ptr(ba), cu.ctypes.data_as(_I64), num_seqs,
                        H, dk, dv, float(eps), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                        int(nthreads))
    return q, k, v, g, beta


def in_proj_prep(x, w, H, d, conv_q, conv_k, conv_v, A_log, alpha_bias, cu_seqlens=None, num_seqs=1,
                 eps=1e-6, nthreads=0):
    """The mixer's input side from the normalised residual stream x_t: the projections that
    eqs. (6)-(11) apply to x_t, then eqs. (6)-(10).

    x [N, D]; w [4*H*d + 2*H, D] stacks, as rows (out_features x in_features), W_q, W_k, W_v,
    W_z (H*d rows each, row c = h*d + i) and W_beta, W_alpha (H rows each).  conv_* [H*d, W]
    are the ShortConv taps.  The projections are one fp64 matrix product; their outputs go
    to prep() unrounded.  Returns (q, k, v, g, beta, z) in float64, z = W_z x [N, H, d].
    """
    x, w = _f64(x), _f64(w)
    N, D = x.shape
    hd = H * d
    assert w.shape == (4 * hd + 2 * H, D)
    p = x @ w.T                                            # [N, 4*H*d + 2*H]
    xq, xk, xv, z = (p[:, j * hd:(j + 1) * hd].reshape(N, H, d) for j in range(4))
    bl, al = p[:, 4 * hd:4 * hd + H], p[:, 4 * hd + H:]
    q, k, v, g, beta = prep(xq, xk, xv, conv_q, conv_k, conv_v, bl, al, A_log, alpha_bias,
                            cu_seqlens, num_seqs, eps, nthreads)
    return q, k, v, g, beta, z.copy()


# significant bits and smallest exponent step of the 16-bit storage formats
_FORMATS = {"bf16": (8, -133), "fp16": (11, -24)}


def round_to_format(x, fmt):
    """x (float64) rounded once to the nearest value of a 16-bit storage format, ties to the
    even significand (IEEE 754 round-to-nearest-even), returned as float64.  fmt: "bf16"
    (8 significant bits, fp32's exponent range) or "fp16" (11 significant bits, subnormal
    step 2^-24).  Values are assumed inside the format's finite range."""
    bits, min_step = _FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                                    # |x| = m 2^e, 1/2 <= m < 1
    step = np.ldexp(1.0, np.maximum(e - bits, min_step))  # spacing of the format at |x|
    return np.round(x / step) * step                      # np.round: ties to even


def out_gate(y, z, w, eps=1e-6):
    """Eq. (11) without W_o: sigmoid(z) * zero-centred RMSNorm(y), per (token, head) over dv."""
    y, z, w = _f64(y), _f64(z), _f64(w)
    N, H, dv = y.shape
    assert z.shape == y.shape and w.shape == (dv,)
    out = np.zeros_like(y)
    _load().oracle_out_gate(_ptr(y), _ptr(z), _ptr(w), float(eps), N, H, dv, _ptr(out))
    return out


def mixer(x_q, x_k, x_v, w_q, w_k, w_v, beta_logit, alpha_logit, A_log, alpha_bias, z, norm_w,
          cu_seqlens=None, num_seqs=1, S0=None, eps_l2=1e-6, eps_rms=1e-6, nthreads=0, inter_dtype=None):
    """The full post-projection mixer in fp64: eqs. (6)-(10), (1)-(4), (11) without W_o.

    inter_dtype (None, "bf16", "fp16", or torch.bfloat16 / torch.float16): the storage format
    of q, k, v between the input side (6)-(8) and the recurrence.  The pages leave it open;
    a mixer that keeps them in 16-bit memory rounds each value once to the nearest
    representable number (round_to_format).  None keeps fp64.

    Returns (out [N, H, dv], y [N, H, dv], S_T).
    """
    q, k, v, g, beta = prep(x_q, x_k, x_v, w_q, w_k, w_v, beta_logit, alpha_logit, A_log,
                            alpha_bias, cu_seqlens, num_seqs, eps_l2, nthreads)
    if inter_dtype is not None:
        fmt = inter_dtype if isinstance(inter_dtype, str) else {"torch.bfloat16": "bf16",
                                                                 "torch.float16": "fp16"}[str(inter_dtype)]
        q, k, v = (round_to_format(t, fmt) for t in (q, k, v))
    y, S_T = recurrence(q, k, v, g, beta, S0, cu_seqlens, num_seqs, 1.0, nthreads)
    return out_gate(y, z, norm_w, eps_rms), y, S_T
