"""gdn_chunk_fwd_noalloc: the chunked prefill for callers that cannot allocate device
memory (its scratch is a fixed array inside the library's device image).

Collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.  It must pass alone in a fresh process and after the
other tests, so it builds and loads the library itself.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

TOL = 3e-3  # the tensor-core path's bound in the parity tests


def rel_err(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def call_noalloc(L, x, y, S_T):
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    N, H, dk = x["q"].shape
    return L.gdn_chunk_fwd_noalloc(p(x["q"]), p(x["k"]), p(x["v"]), p(x["g"]), p(x["beta"]), p(x["S0"]),
                                   p(x["cu_seqlens"]), x["num_seqs"], N, H, dk, x["dv"], 64, 1.0, gdn.BF16,
                                   gdn.F32, p(y), p(S_T), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device):
    gbuild.build()
    L = gdn.lib()
    # two calls in a row with different inputs: the first fills more of the shared scratch
    # (32 chunks per head) than the second uses (19), so the second finds stale records beyond
    # its own and must not depend on them.  Both entry points run the same deterministic
    # kernels on the same inputs, so their outputs agree bit for bit.
    for seed, lengths in ((41, [1500, 64, 1, 333]), (42, [129, 1000])):
        x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=seed, lengths=lengths, H=4, S0_std=0.1)
        y_ref, S_ref = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"],
                                     chunk=64, y_dtype=torch.float32)
        y = torch.full_like(y_ref, float("nan"))
        S_T = torch.full_like(S_ref, float("nan"))
        st = call_noalloc(L, x, y, S_T)
        assert st == gdn.GDN_OK, gdn.last_error_message()
        gdn.check_device_error()
        assert torch.equal(y, y_ref) and torch.equal(S_T, S_ref)
        assert rel_err(y, y_ref) < TOL


def test_noalloc_rejects_work_beyond_its_scratch(cuda_device):
    L = gdn.lib()
    N, H = 1 << 20, 32  # about 12.6 GB of records
    A = ctypes.c_void_p(0x10000)
    st = L.gdn_chunk_fwd_noalloc(A, A, A, A, A, None, None, 1, N, H, 128, 128, 64, 1.0, gdn.BF16, gdn.BF16, A,
                                 None, None)
    assert st == gdn.GDN_ERR_INVALID_ARG
    assert "scratch" in gdn.last_error_message()


def test_noalloc_answers_unsupported_calls_like_the_workspace_entry_point(cuda_device):
    """A large call the tensor-core path does not take (dk = 64, or fp32 inputs) needs no
    scratch: both entry points return GDN_ERR_UNSUPPORTED, with nothing launched."""
    L = gdn.lib()
    N, H = 1 << 20, 32
    A = ctypes.c_void_p(0x10000)
    for dk, dt in ((64, gdn.BF16), (128, gdn.F32)):
        st = L.gdn_chunk_fwd_noalloc(A, A, A, A, A, None, None, 1, N, H, dk, 128, 64, 1.0, dt, gdn.BF16, A,
                                     None, None)
        st_ws = L.gdn_chunk_fwd(A, A, A, A, A, None, None, 1, N, H, dk, 128, 64, 1.0, dt, gdn.BF16, A,
                                None, None, 0, None)
        assert st == st_ws == gdn.GDN_ERR_UNSUPPORTED
