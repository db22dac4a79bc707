"""Thin ctypes binding of libgdn.so with the C ABI's entry-point names.

Argument marshalling only: every step of the mixer runs in the CUDA kernels behind
``include/gdn.h``.  PyTorch provides device memory and the current stream; output
tensors are allocated here with ``torch.empty`` when the caller passes none.
There is no fallback: if ``libgdn.so`` is missing or no CUDA device is present, the
compute calls raise.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdn.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libgdn_debug.so")  # the bounds-checking build

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT = range(5)
F32, BF16, F16 = 0, 1, 2
_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}

# Every symbol include/gdn.h declares, with its ctypes signature.
_P, _I, _F, _Z, _U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
SIGNATURES = {
    "gdn_version": ([], _I),
    "gdn_status_string": ([_I], ctypes.c_char_p),
    "gdn_last_error_message": ([], ctypes.c_char_p),
    "gdn_check_device_error": ([_P], _I),
    "gdn_set_wait_budget": ([_U64], None),
    "gdn_prep": ([_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I,
                  _P, _P, _P, _P, _P, _P], _I),
    "gdn_bounds_checked": ([], _I),
    "gdn_inproj_prep": ([_P, _P, _I, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P, _P, _P, _P,
                         _P, _P, _P], _I),
    "gdn_chunk_fwd_workspace_size": ([_I, _I, _I, _I, _I, _I], _Z),
    "gdn_chunk_fwd": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _P, _P,
                       _Z, _P], _I),
    "gdn_chunk_fwd_gated": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _F, _I, _P,
                             _P, _P, _Z, _P], _I),
    "gdn_chunk_fwd_noalloc": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _P, _P], _I),
    "gdn_decode_step": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P, _P], _I),
    "gdn_mixer_decode_step": ([_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _F, _F, _P, _P, _P, _I, _I,
                               _I, _I, _I, _F, _I, _I, _P, _P], _I),
    "gdn_out_gate": ([_P, _P, _P, _F, _I, _I, _I, _I, _I, _P, _P], _I),
    "gdn_state_map_apply": ([_P, _P, _P, _P, _I, _I, _I, _P], _I),
    "gdn_chunk_fwd_prep_workspace_size": ([_I, _I, _I, _I, _I, _I], ctypes.c_size_t),
    "gdn_chunk_bwd_workspace_size": ([_I, _I, _I, _I, _I], ctypes.c_size_t),
    "gdn_chunk_bwd": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P,
                       ctypes.c_size_t, _P], _I),
    "gdn_chunk_fwd_prep": ([_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _F, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I,
                            _I, _P, _P, _P, ctypes.c_size_t, _P], _I),
    "gdn_timing_start": ([_I], _I),
    "gdn_timing_stop": ([_I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_I), ctypes.POINTER(ctypes.c_double),
                         ctypes.POINTER(_I)], _I),
}

_lib = None


class GDNError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{status_string(status)}: {msg}")
        self.status = status


def load(path):
    """ctypes.CDLL of a built libgdn with every declared signature bound.  Raises if it is missing."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: run `python -m linear_attention_token_gdn_b200.build`")
    L = ctypes.CDLL(path)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


def lib():
    """The loaded libgdn.so (ctypes.CDLL with argtypes set).  Raises if it was never built."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


@contextlib.contextmanager
def using(L):
    """Route this module's calls through another loaded build (e.g. load(DEBUG_LIB_PATH), the
    bounds-checking one) inside the block.  The module-level handle is swapped, so the switch
    applies to every thread of the process while the block runs."""
    global _lib
    prev = lib()
    _lib = L
    try:
        yield L
    finally:
        _lib = prev


def status_string(s: int) -> str:
    return lib().gdn_status_string(s).decode()


def last_error_message() -> str:
    return lib().gdn_last_error_message().decode()


def _check(status: int):
    if status != GDN_OK:
        raise GDNError(status, last_error_message())


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libgdn takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dt(t):
    try:
        return _DT[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported dtype {t.dtype}") from None


def version() -> int:
    return lib().gdn_version()


def set_wait_budget(cycles: int):
    lib().gdn_set_wait_budget(int(cycles))


def check_device_error(stream=None):
    """Synchronise the stream and raise if a kernel flagged an error since the last check."""
    _check(lib().gdn_check_device_error(_stream(stream)))


def timing_start(max_launches=4096):
    """gdn_timing_start: time every library kernel launch with CUDA events from now on."""
    _check(lib().gdn_timing_start(int(max_launches)))


def timing_stop(cap=64):
    """gdn_timing_stop: {kernel name: (launches, total device ms)} since timing_start."""
    names = (ctypes.c_char_p * cap)()
    launches = (_I * cap)()
    total = (ctypes.c_double * cap)()
    n = _I(0)
    _check(lib().gdn_timing_stop(cap, names, launches, total, ctypes.byref(n)))
    return {names[i].decode(): (launches[i], total[i]) for i in range(min(n.value, cap))}


def workspace_size(N, num_seqs, H, dk, dv, chunk) -> int:
    return int(lib().gdn_chunk_fwd_workspace_size(N, num_seqs, H, dk, dv, chunk))


def prep(x_q, x_k, x_v, w_q, w_k, w_v, beta_logit, alpha_logit, A_log, alpha_bias, cu_seqlens=None,
         num_seqs=1, eps=1e-6, out_dtype=None, out=None, stream=None):
    """gdn_prep: eqs. (6)-(10).  Returns (q, k, v, g, beta)."""
    N, H, dk = x_q.shape
    dv = x_v.shape[2]
    if cu_seqlens is not None:
        num_seqs = cu_seqlens.numel() - 1
    out_dtype = x_q.dtype if out_dtype is None else out_dtype
    if out is None:
        dev = x_q.device
        out = (torch.empty(N, H, dk, device=dev, dtype=out_dtype), torch.empty(N, H, dk, device=dev, dtype=out_dtype),
               torch.empty(N, H, dv, device=dev, dtype=out_dtype), torch.empty(N, H, device=dev),
               torch.empty(N, H, device=dev))
    q, k, v, g, beta = out
    _check(lib().gdn_prep(_ptr(x_q), _ptr(x_k), _ptr(x_v), _ptr(w_q), _ptr(w_k), _ptr(w_v), w_q.shape[1],
                          _ptr(beta_logit), _ptr(alpha_logit), _ptr(A_log), _ptr(alpha_bias), _ptr(cu_seqlens),
                          num_seqs, N, H, dk, dv, float(eps), _dt(x_q), _DT[out_dtype], _ptr(q), _ptr(k),
                          _ptr(v), _ptr(g), _ptr(beta), _stream(stream)))
    return q, k, v, g, beta


def inproj_prep(x, w, H, conv_q, conv_k, conv_v, A_log, alpha_bias, cu_seqlens=None, num_seqs=1, eps=1e-6,
                out_dtype=None, with_z=True, out=None, stream=None):
    """gdn_inproj_prep: the input projections of x [N, D] by the stacked rows
    w = [W_q; W_k; W_v; W_z; W_beta; W_alpha] fused with eqs. (6)-(10).
    Returns (q, k, v, g, beta, z) (z None when with_z is False)."""
    N, D = x.shape
    d = 128
    if cu_seqlens is not None:
        num_seqs = cu_seqlens.numel() - 1
    out_dtype = x.dtype if out_dtype is None else out_dtype
    if out is None:
        dev = x.device
        out = tuple(torch.empty(N, H, d, device=dev, dtype=out_dtype) for _ in range(3)) + (
            torch.empty(N, H, device=dev), torch.empty(N, H, device=dev),
            torch.empty(N, H, d, device=dev, dtype=out_dtype) if with_z else None)
    q, k, v, g, beta, z = out
    _check(lib().gdn_inproj_prep(_ptr(x), _ptr(w), D, _ptr(conv_q), _ptr(conv_k), _ptr(conv_v), conv_q.shape[1],
                                 _ptr(A_log), _ptr(alpha_bias), _ptr(cu_seqlens), num_seqs, N, H, d, d, float(eps),
                                 _dt(x), _DT[out_dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(g), _ptr(beta),
                                 _stream(stream)))
    return q, k, v, g, beta, z


def chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, num_seqs=None, chunk=64, scale=1.0, y_dtype=None,
              final_state=True, y=None, S_T=None, workspace=None, stream=None):
    """gdn_chunk_fwd: prefill over packed sequences.  Returns (y, S_T or None)."""
    N, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        num_seqs = cu_seqlens.numel() - 1
    elif num_seqs is None:
        num_seqs = 1
    y_dtype = q.dtype if y_dtype is None else y_dtype
    if y is None:
        y = torch.empty(N, H, dv, device=q.device, dtype=y_dtype)
    if S_T is None and final_state:
        S_T = torch.empty(num_seqs, H, dk, dv, device=q.device, dtype=torch.float32)
    ws_bytes = workspace_size(N, num_seqs, H, dk, dv, chunk)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    _check(lib().gdn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                               num_seqs, N, H, dk, dv, int(chunk), float(scale), _dt(q), _DT[y.dtype], _ptr(y),
                               _ptr(S_T), _ptr(workspace), 0 if workspace is None else workspace.numel(),
                               _stream(stream)))
    return y, S_T


def chunk_fwd_gated(q, k, v, g, beta, z, norm_w, eps=1e-6, S0=None, cu_seqlens=None, num_seqs=None, scale=1.0,
                    final_state=True, out=None, S_T=None, workspace=None, stream=None):
    """gdn_chunk_fwd_gated: the chunk-64 prefill with eq. (11)'s output gate fused (y is not
    written).  Returns (out [N, H, dv] in z's dtype, S_T or None)."""
    N, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        num_seqs = cu_seqlens.numel() - 1
    elif num_seqs is None:
        num_seqs = 1
    if out is None:
        out = torch.empty(N, H, dv, device=q.device, dtype=z.dtype)
    if S_T is None and final_state:
        S_T = torch.empty(num_seqs, H, dk, dv, device=q.device, dtype=torch.float32)
    ws_bytes = workspace_size(N, num_seqs, H, dk, dv, 64)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    _check(lib().gdn_chunk_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                                     num_seqs, N, H, dk, dv, 64, float(scale), _dt(q), _ptr(z), _ptr(norm_w),
                                     float(eps), _dt(z), _ptr(out), _ptr(S_T), _ptr(workspace),
                                     0 if workspace is None else workspace.numel(), _stream(stream)))
    return out, S_T


def chunk_fwd_noalloc(q, k, v, g, beta, S0=None, cu_seqlens=None, num_seqs=None, chunk=64, scale=1.0,
                      y_dtype=None, final_state=True, y=None, S_T=None, stream=None):
    """gdn_chunk_fwd_noalloc: gdn_chunk_fwd with the library's built-in scratch instead of a
    caller workspace (for callers that cannot allocate device memory).  Returns (y, S_T)."""
    N, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        num_seqs = cu_seqlens.numel() - 1
    elif num_seqs is None:
        num_seqs = 1
    y_dtype = q.dtype if y_dtype is None else y_dtype
    if y is None:
        y = torch.empty(N, H, dv, device=q.device, dtype=y_dtype)
    if S_T is None and final_state:
        S_T = torch.empty(num_seqs, H, dk, dv, device=q.device, dtype=torch.float32)
    _check(lib().gdn_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                                       num_seqs, N, H, dk, dv, int(chunk), float(scale), _dt(q), _DT[y.dtype],
                                       _ptr(y), _ptr(S_T), _stream(stream)))
    return y, S_T


def decode_step(q, k, v, g, beta, state, state_slot=None, scale=1.0, y_dtype=None, y=None, stream=None):
    """gdn_decode_step: one token per row; ``state`` is updated in place.  Returns y."""
    B, H, dk = q.shape
    dv = v.shape[2]
    if y is None:
        y = torch.empty(B, H, dv, device=q.device, dtype=q.dtype if y_dtype is None else y_dtype)
    _check(lib().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(state_slot),
                                 state.shape[0], B, H, dk, dv, float(scale), _dt(q), _DT[y.dtype], _ptr(y),
                                 _stream(stream)))
    return y


def mixer_decode_step(x_q, x_k, x_v, w_q, w_k, w_v, beta_logit, alpha_logit, A_log, alpha_bias, z, norm_w,
                      conv_state, state, state_slot=None, l2_eps=1e-6, rms_eps=1e-6, scale=1.0, out_dtype=None,
                      out=None, stream=None):
    """gdn_mixer_decode_step: one token per row through the whole mixer; ``conv_state``
    [slots, W-1, H, 2 dk + dv] and ``state`` are updated in place.  Returns out [B, H, dv]."""
    B, H, dk = x_q.shape
    dv = x_v.shape[2]
    W = w_q.shape[1]
    if out is None:
        out = torch.empty(B, H, dv, device=x_q.device, dtype=x_q.dtype if out_dtype is None else out_dtype)
    _check(lib().gdn_mixer_decode_step(_ptr(x_q), _ptr(x_k), _ptr(x_v), _ptr(w_q), _ptr(w_k), _ptr(w_v), W,
                                       _ptr(beta_logit), _ptr(alpha_logit), _ptr(A_log), _ptr(alpha_bias), _ptr(z),
                                       _ptr(norm_w), float(l2_eps), float(rms_eps), _ptr(conv_state), _ptr(state),
                                       _ptr(state_slot), state.shape[0], B, H, dk, dv, float(scale), _dt(x_q),
                                       _DT[out.dtype], _ptr(out), _stream(stream)))
    return out


def chunk_fwd_prep(x_q, x_k, x_v, w_q, w_k, w_v, beta_logit, alpha_logit, A_log, alpha_bias, S0=None,
                   cu_seqlens=None, num_seqs=None, l2_eps=1e-6, scale=1.0, qkv_dtype=None, y_dtype=None, y=None,
                   S_T=None, final_state=True, workspace=None, stream=None):
    """gdn_chunk_fwd_prep: prep (eqs. (6)-(10)) fused into the chunked pass.  q, k, v are rounded
    to qkv_dtype (default: the inputs' format) before the recurrence.  Returns (y, S_T or None)."""
    N, H, dk = x_q.shape
    dv = x_v.shape[2]
    W = w_q.shape[-1]
    if cu_seqlens is not None:
        num_seqs = cu_seqlens.numel() - 1
    elif num_seqs is None:
        num_seqs = 1
    qkv_dtype = x_q.dtype if qkv_dtype is None else qkv_dtype
    y_dtype = qkv_dtype if y_dtype is None else y_dtype
    if y is None:
        y = torch.empty(N, H, dv, device=x_q.device, dtype=y_dtype)
    if S_T is None and final_state:
        S_T = torch.empty(num_seqs, H, dk, dv, device=x_q.device)
    if workspace is None:
        nbytes = lib().gdn_chunk_fwd_prep_workspace_size(N, num_seqs, H, dk, dv, 64)
        workspace = torch.empty(max(nbytes, 16), device=x_q.device, dtype=torch.uint8)
    _check(lib().gdn_chunk_fwd_prep(_ptr(x_q), _ptr(x_k), _ptr(x_v), _ptr(w_q), _ptr(w_k), _ptr(w_v), W,
                                    _ptr(beta_logit), _ptr(alpha_logit), _ptr(A_log), _ptr(alpha_bias), float(l2_eps),
                                    _ptr(S0), _ptr(cu_seqlens), num_seqs, N, H, dk, dv, 64, float(scale), _dt(x_q),
                                    _DT[qkv_dtype], _DT[y_dtype], _ptr(y), _ptr(S_T), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))
    return y, S_T


def chunk_bwd(q, k, v, g, beta, dy, S0=None, dS_T=None, cu_seqlens=None, num_seqs=None, scale=1.0, out=None,
              workspace=None, stream=None):
    """gdn_chunk_bwd: gradients through eqs. (1)-(4).  Returns dict(dq, dk, dv, dg, dbeta, dS0),
    fp32 (dg: with respect to g = log alpha)."""
    N, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        num_seqs = cu_seqlens.numel() - 1
    elif num_seqs is None:
        num_seqs = 1
    dev = q.device
    if out is None:
        out = dict(dq=torch.empty(N, H, dk, device=dev), dk=torch.empty(N, H, dk, device=dev),
                   dv=torch.zeros(N, H, dv, device=dev), dg=torch.empty(N, H, device=dev),
                   dbeta=torch.empty(N, H, device=dev), dS0=torch.empty(num_seqs, H, dk, dv, device=dev))
    if workspace is None:
        nbytes = lib().gdn_chunk_bwd_workspace_size(N, num_seqs, H, dk, dv)
        workspace = torch.empty(max(nbytes, 16), device=dev, dtype=torch.uint8)
    _check(lib().gdn_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(cu_seqlens), num_seqs,
                               N, H, dk, dv, float(scale), _dt(q), _ptr(dy), _dt(dy), _ptr(dS_T), _ptr(out["dq"]),
                               _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dS0"]),
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def state_map_apply(M, B, S_in, S_out=None, stream=None):
    """gdn_state_map_apply: S_out = M S_in + B per state row (B may be None: zero).  M is
    [..., dk, dk], B, S_in and S_out [..., dk, dv], fp32.  Returns S_out."""
    dk, dv = S_in.shape[-2], S_in.shape[-1]
    rows = S_in.numel() // (dk * dv)
    if S_out is None:
        S_out = torch.empty_like(S_in)
    _check(lib().gdn_state_map_apply(_ptr(M), _ptr(B) if B is not None else None, _ptr(S_in), _ptr(S_out), rows, dk,
                                     dv, _stream(stream)))
    return S_out


def out_gate(y, z, norm_w, eps=1e-6, out=None, stream=None):
    """gdn_out_gate: eq. (11) without W_o.  Returns out (dtype of z)."""
    N, H, dv = y.shape
    if out is None:
        out = torch.empty(N, H, dv, device=z.device, dtype=z.dtype)
    _check(lib().gdn_out_gate(_ptr(y), _ptr(z), _ptr(norm_w), float(eps), N, H, dv, _dt(y), _dt(z), _ptr(out),
                              _stream(stream)))
    return out
