"""The C-ABI library without a GPU: it loads, exports every symbol include/gdn.h declares,
and rejects bad arguments on the host before enqueuing anything (no device needed)."""
import ctypes
import os
import re

import pytest

from linear_attention_token_gdn_b200 import build as gbuild
from linear_attention_token_gdn_b200 import gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gdn.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported_and_bound(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
        assert n in gdn.SIGNATURES, n
    assert set(gdn.SIGNATURES) == set(names)


def test_status_strings_and_version(L):
    assert gdn.version() >= 100
    assert gdn.status_string(gdn.GDN_OK) == "GDN_OK"
    assert gdn.status_string(gdn.GDN_ERR_TIMEOUT) == "GDN_ERR_TIMEOUT"


A = ctypes.c_void_p(0x10000)      # an aligned fake address: validation never dereferences it
MIS = ctypes.c_void_p(0x10004)    # misaligned


def chunk_call(L, **over):
    a = dict(q=A, k=A, v=A, g=A, beta=A, S0=None, cu=None, num_seqs=2, N=64, H=2, dk=128, dv=128, chunk=64,
             scale=1.0, in_dt=gdn.BF16, y_dt=gdn.BF16, y=A, S_T=None, ws=A, ws_bytes=1 << 30, stream=None)
    a.update(over)
    return L.gdn_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["cu"], a["num_seqs"], a["N"],
                           a["H"], a["dk"], a["dv"], a["chunk"], a["scale"], a["in_dt"], a["y_dt"], a["y"],
                           a["S_T"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("over", [
    dict(q=None), dict(k=MIS), dict(dk=48), dict(dv=256), dict(chunk=-1), dict(N=-1),
    dict(H=0), dict(num_seqs=0), dict(N=63), dict(in_dt=7), dict(y_dt=-1), dict(S0=MIS),
    dict(ws_bytes=0, ws=None),
])
def test_chunk_fwd_rejects_bad_arguments(L, over):
    assert chunk_call(L, **over) == gdn.GDN_ERR_INVALID_ARG
    assert gdn.last_error_message() != ""


@pytest.mark.parametrize("over", [dict(dk=64, dv=64), dict(in_dt=gdn.F32), dict(dk=128, dv=64), dict(chunk=32),
                                  dict(chunk=128)])
def test_chunk_fwd_tensor_core_path_limits(L, over):
    assert chunk_call(L, **over) == gdn.GDN_ERR_UNSUPPORTED


def gated_call(L, **over):
    a = dict(q=A, k=A, v=A, g=A, beta=A, S0=None, cu=None, num_seqs=2, N=64, H=2, dk=128, dv=128, chunk=64,
             scale=1.0, in_dt=gdn.BF16, z=A, w=A, eps=1e-6, io_dt=gdn.BF16, out=A, S_T=None, ws=A,
             ws_bytes=1 << 30, stream=None)
    a.update(over)
    return L.gdn_chunk_fwd_gated(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["cu"], a["num_seqs"],
                                 a["N"], a["H"], a["dk"], a["dv"], a["chunk"], a["scale"], a["in_dt"], a["z"],
                                 a["w"], a["eps"], a["io_dt"], a["out"], a["S_T"], a["ws"], a["ws_bytes"],
                                 a["stream"])


@pytest.mark.parametrize("over", [
    dict(z=None), dict(out=MIS), dict(w=None), dict(eps=-1.0), dict(io_dt=5), dict(N=-1), dict(N=63),
    dict(ws_bytes=0, ws=None), dict(q=None),
])
def test_chunk_fwd_gated_rejects_bad_arguments(L, over):
    assert gated_call(L, **over) == gdn.GDN_ERR_INVALID_ARG
    assert gdn.last_error_message() != ""


@pytest.mark.parametrize("over", [dict(chunk=0), dict(chunk=32), dict(dk=64, dv=64), dict(in_dt=gdn.F32),
                                  dict(io_dt=gdn.F32)])
def test_chunk_fwd_gated_is_tensor_core_only(L, over):
    assert gated_call(L, **over) == gdn.GDN_ERR_UNSUPPORTED


def test_workspace_size_is_zero_without_records(L):
    assert L.gdn_chunk_fwd_workspace_size(8192, 2, 16, 128, 128, 0) == 0     # token recurrence
    assert L.gdn_chunk_fwd_workspace_size(8192, 2, 16, 128, 128, 128) == 0   # not built


def test_workspace_size_covers_every_chunk(L):
    # one 72.5 KB record per (64-token chunk, head); packed sequences add one partial chunk each
    assert L.gdn_chunk_fwd_workspace_size(8192, 2, 16, 128, 128, 64) == (128 + 2) * 16 * 74240
    assert L.gdn_chunk_fwd_workspace_size(100, 3, 4, 128, 128, 64) == (2 + 3) * 4 * 74240
    assert L.gdn_chunk_fwd_workspace_size(8192, 2, 16, 128, 128, 0) == 0


def test_zero_tokens_is_a_no_op(L):
    assert chunk_call(L, N=0, q=None, y=None) == gdn.GDN_OK
    assert gated_call(L, N=0, q=None, z=None, out=None, w=None) == gdn.GDN_OK
    assert L.gdn_decode_step(None, None, None, None, None, None, None, 0, 0, 4, 128, 128, 1.0, 1, 1, None,
                             None) == gdn.GDN_OK
    assert L.gdn_out_gate(None, None, None, 1e-6, 0, 4, 128, 1, 1, None, None) == gdn.GDN_OK


@pytest.mark.parametrize("over", [
    dict(state=None), dict(num_slots=3), dict(dk=8), dict(y=MIS), dict(in_dt=5), dict(slot=MIS),
])
def test_decode_rejects_bad_arguments(L, over):
    a = dict(state=A, slot=None, num_slots=4, B=4, H=2, dk=128, dv=128, in_dt=1, y=A)
    a.update(over)
    st = L.gdn_decode_step(A, A, A, A, A, a["state"], a["slot"], a["num_slots"], a["B"], a["H"], a["dk"], a["dv"],
                           1.0, a["in_dt"], 1, a["y"], None)
    assert st == gdn.GDN_ERR_INVALID_ARG


@pytest.mark.parametrize("over", [dict(W=0), dict(W=9), dict(x_q=None), dict(eps=-1.0), dict(dk=100)])
def test_prep_rejects_bad_arguments(L, over):
    a = dict(W=4, x_q=A, eps=1e-6, dk=128)
    a.update(over)
    st = L.gdn_prep(a["x_q"], A, A, A, A, A, a["W"], A, A, A, A, None, 1, 16, 2, a["dk"], 128, a["eps"], 1, 1,
                    A, A, A, A, A, None)
    assert st == gdn.GDN_ERR_INVALID_ARG


@pytest.mark.parametrize("over", [dict(dv=96), dict(eps=-1.0), dict(out=None), dict(io=3)])
def test_out_gate_rejects_bad_arguments(L, over):
    a = dict(dv=128, eps=1e-6, out=A, io=1)
    a.update(over)
    assert L.gdn_out_gate(A, A, A, a["eps"], 16, 2, a["dv"], 1, a["io"], a["out"], None) == gdn.GDN_ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    import torch
    with pytest.raises(ValueError):
        gdn._ptr(torch.zeros(4))


def test_timing_rejects_bad_use(L):
    assert L.gdn_timing_start(0) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_timing_start(1 << 21) == gdn.GDN_ERR_INVALID_ARG
    # stopping while timing is off is an argument error, with or without a device
    assert L.gdn_timing_stop(0, None, None, None, None) == gdn.GDN_ERR_INVALID_ARG


@pytest.mark.parametrize("over", [dict(W=0), dict(W=9), dict(x_q=None), dict(dk=48), dict(conv=None),
                                  dict(l2=-1.0), dict(num_slots=1), dict(out=MIS)])
def test_mixer_decode_rejects_bad_arguments(L, over):
    a = dict(W=4, x_q=A, dk=128, conv=A, l2=1e-6, num_slots=4, out=A)
    a.update(over)
    st = L.gdn_mixer_decode_step(a["x_q"], A, A, A, A, A, a["W"], A, A, A, A, A, A, a["l2"], 1e-6, a["conv"], A,
                                 None, a["num_slots"], 4, 2, a["dk"], 128, 1.0, 1, 1, a["out"], None)
    assert st == gdn.GDN_ERR_INVALID_ARG


def test_mixer_decode_without_history_needs_no_conv_state(L):
    """conv width 1 keeps no history: a NULL conv_state passes validation (nothing launched
    for zero rows)."""
    assert L.gdn_mixer_decode_step(A, A, A, A, A, A, 1, A, A, A, A, A, A, 1e-6, 1e-6, None, A, None, 4, 0, 2, 128,
                                   128, 1.0, 1, 1, A, None) == gdn.GDN_OK


def test_state_map_apply_validation(L):
    """gdn_state_map_apply: nothing to do for zero rows; bad sizes, misaligned pointers and an
    output overlapping an input are refused before any launch."""
    assert L.gdn_state_map_apply(None, None, None, None, 0, 128, 128, None) == gdn.GDN_OK
    assert L.gdn_state_map_apply(A, None, ctypes.c_void_p(0x20000), ctypes.c_void_p(0x40000), 2, 48, 128,
                                 None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_state_map_apply(A, MIS, ctypes.c_void_p(0x20000), ctypes.c_void_p(0x40000), 2, 128, 128,
                                 None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_state_map_apply(A, None, A, A, 2, 128, 128, None) == gdn.GDN_ERR_INVALID_ARG    # S_out is S_in
    assert L.gdn_state_map_apply(ctypes.c_void_p(0x100000), None, A, ctypes.c_void_p(0x108000), 1, 128, 128,
                                 None) == gdn.GDN_ERR_INVALID_ARG                                   # S_out over M
    assert gdn.last_error_message() != ""


def prep_call(L, **over):
    a = dict(xq=A, W=4, eps=1e-6, N=64, H=2, dk=128, dv=128, chunk=64, in_dt=gdn.BF16, qkv=gdn.F16, y_dt=gdn.BF16,
             ws=A, ws_bytes=1 << 30)
    a.update(over)
    return L.gdn_chunk_fwd_prep(a["xq"], A, A, A, A, A, a["W"], A, A, A, A, a["eps"], None, None, 1, a["N"], a["H"],
                                a["dk"], a["dv"], a["chunk"], 1.0, a["in_dt"], a["qkv"], a["y_dt"], A, None, a["ws"],
                                a["ws_bytes"], None)


@pytest.mark.parametrize("over", [dict(W=0), dict(W=9), dict(eps=-1.0), dict(xq=None), dict(ws=None),
                                  dict(ws_bytes=16), dict(in_dt=9), dict(dk=48)])
def test_chunk_fwd_prep_rejects_bad_arguments(L, over):
    assert prep_call(L, **over) == gdn.GDN_ERR_INVALID_ARG
    assert gdn.last_error_message() != ""


@pytest.mark.parametrize("over", [dict(chunk=0), dict(dk=64, dv=64), dict(in_dt=gdn.F32), dict(qkv=gdn.F32)])
def test_chunk_fwd_prep_is_tensor_core_only(L, over):
    assert prep_call(L, **over) == gdn.GDN_ERR_UNSUPPORTED


def test_chunk_fwd_prep_workspace_is_the_records(L):
    rec = L.gdn_chunk_fwd_workspace_size(8192, 2, 16, 128, 128, 64)
    assert L.gdn_chunk_fwd_prep_workspace_size(8192, 2, 16, 128, 128, 64) == rec


@pytest.mark.parametrize("over", [dict(dk=48), dict(ws=None), dict(ws_bytes=16), dict(dy=None), dict(dS0=None),
                                  dict(in_dt=9)])
def test_chunk_bwd_rejects_bad_arguments(L, over):
    a = dict(dk=128, ws=A, ws_bytes=1 << 30, dy=A, dS0=A, in_dt=gdn.BF16)
    a.update(over)
    st = L.gdn_chunk_bwd(A, A, A, A, A, None, None, 2, 64, 2, a["dk"], 128, 1.0, a["in_dt"], a["dy"], gdn.F32, None,
                         A, A, A, A, A, a["dS0"], a["ws"], a["ws_bytes"], None)
    assert st == gdn.GDN_ERR_INVALID_ARG
    assert gdn.last_error_message() != ""


def test_chunk_bwd_workspace_holds_a_checkpoint_per_eight_tokens(L):
    assert L.gdn_chunk_bwd_workspace_size(8192, 2, 16, 128, 128) == (1024 + 2) * 16 * 128 * 128 * 4
    assert L.gdn_chunk_bwd_workspace_size(0, 2, 16, 128, 128) == 0


@pytest.mark.parametrize("over,status", [
    (dict(D=96), gdn.GDN_ERR_INVALID_ARG), (dict(D=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(W=0), gdn.GDN_ERR_INVALID_ARG), (dict(W=9), gdn.GDN_ERR_INVALID_ARG),
    (dict(x=None), gdn.GDN_ERR_INVALID_ARG), (dict(w=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(eps=-1.0), gdn.GDN_ERR_INVALID_ARG), (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(H=8), gdn.GDN_ERR_UNSUPPORTED), (dict(H=144), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=64), gdn.GDN_ERR_UNSUPPORTED), (dict(io=0), gdn.GDN_ERR_UNSUPPORTED),
])
def test_inproj_prep_rejects_bad_arguments(L, over, status):
    a = dict(D=256, W=4, x=A, w=A, eps=1e-6, q=A, H=16, dk=128, io=1)
    a.update(over)
    st = L.gdn_inproj_prep(a["x"], a["w"], a["D"], A, A, A, a["W"], A, A, None, 1, 16, a["H"], a["dk"], 128,
                           a["eps"], a["io"], 1, a["q"], A, A, None, A, A, None)
    assert st == status


def test_inproj_prep_with_no_tokens_is_a_no_op(L):
    assert L.gdn_inproj_prep(None, None, 256, None, None, None, 4, None, None, None, 1, 0, 16, 128, 128, 1e-6, 1, 1,
                             None, None, None, None, None, None, None) == gdn.GDN_OK


def test_bounds_checking_build_exports_every_symbol_and_says_so(L):
    gbuild.build(debug=True)
    D = gdn.load(gdn.DEBUG_LIB_PATH)
    for n in declared_functions():
        assert hasattr(D, n), n
    assert D.gdn_bounds_checked() == 1 and L.gdn_bounds_checked() == 0
    assert D.gdn_version() == L.gdn_version()
