"""The C ABI without a GPU: the library loads, exports every symbol that
include/vdn.h declares, and rejects bad arguments on the host before it
touches the device."""
import ctypes

import pytest

from frame_wise_delta_b200 import build, vdn


@pytest.fixture(scope="module")
def L():
    build.build()
    return vdn.lib()


def test_exports_every_declared_symbol(L):
    names = vdn.declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert vdn.vdn_version() >= 100
    assert vdn.vdn_status_string(vdn.VDN_OK) == "VDN_OK"
    assert vdn.vdn_status_string(vdn.VDN_ERR_INVALID) == "VDN_ERR_INVALID"
    assert vdn.vdn_status_string(99) == "VDN_ERR_UNKNOWN"


def _call(L, name, *args):
    fn = getattr(L, name)
    return fn(*args)


def _shape(**kw):
    base = dict(B=1, H=2, T=10, U=16, d=16, n_text=8, chunk=5, anchors=0, in_dtype="f32")
    base.update(kw)
    return vdn.make_shape(**base)


def _p(s):
    return ctypes.cast(ctypes.pointer(s), ctypes.c_void_p)


def test_null_shape_is_invalid(L):
    st = L.vdn_frame_grams(None, None, None, None, None, None, None, None)
    assert st == vdn.VDN_ERR_INVALID
    assert "shape" in vdn.vdn_last_error()


@pytest.mark.parametrize("kw,status", [
    (dict(d=48), vdn.VDN_ERR_UNSUPPORTED),
    (dict(chunk=0), vdn.VDN_ERR_INVALID),
    (dict(chunk=17), vdn.VDN_ERR_INVALID),
    (dict(anchors=2), vdn.VDN_ERR_INVALID),
    (dict(T=-1), vdn.VDN_ERR_INVALID),
    (dict(U=-3), vdn.VDN_ERR_INVALID),
])
def test_bad_shapes(L, kw, status):
    s = _shape(**kw)
    assert L.vdn_frame_grams(_p(s), 16, 16, 16, 16, 16, None, None) == status


def test_bad_dtype(L):
    s = _shape()
    s.in_dtype = 7
    assert L.vdn_chunk_readout(_p(s), 16, 16, 16, 16, None, None) == vdn.VDN_ERR_INVALID


def test_dk_dv_mismatch(L):
    s = _shape()
    s.dv = 32
    assert L.vdn_frame_grams(_p(s), 16, 16, 16, 16, 16, None, None) == vdn.VDN_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers(L):
    s = _shape()
    assert L.vdn_frame_grams(_p(s), None, 16, 16, 16, 16, None, None) == vdn.VDN_ERR_INVALID
    assert "K is NULL" in vdn.vdn_last_error()
    assert L.vdn_frame_grams(_p(s), 16, 16, 16, 16, 0x1008, None, None) == vdn.VDN_ERR_INVALID
    assert "Bm is not 16-byte aligned" in vdn.vdn_last_error()
    assert L.vdn_chunk_compose(_p(s), 16, 16, 16, None, 16, 16, None) == vdn.VDN_ERR_INVALID
    assert L.vdn_scan_bidir(_p(s), 16, 16, 16, 16, None, 16, 16, None) == vdn.VDN_ERR_INVALID
    assert "S_T" in vdn.vdn_last_error()


def test_workspace_checks(L):
    s = _shape()
    need = vdn.vdn_forward_workspace_bytes(s)
    assert need > 0 and need % 256 == 0
    args = [_p(s)] + [16] * 9 + [16, 16, 256]  # Q..O, F, G, workspace
    st = L.vdn_forward(*args[:13], need - 1, 16, None, None, None)
    assert st == vdn.VDN_ERR_INVALID and "workspace" in vdn.vdn_last_error()
    st = L.vdn_forward(*args[:12], 0x1010, need, 16, None, None, None)
    assert st == vdn.VDN_ERR_INVALID and "256-byte" in vdn.vdn_last_error()
    assert vdn.vdn_text_state_workspace_bytes(s) == 2 * 2 * 16 * 16 * 4
    # bf16, d = 128: the tensor path also keeps one 64 KB inverse image per (b, h)
    s2 = _shape(d=128, in_dtype="bf16")
    assert vdn.vdn_text_state_workspace_bytes(s2) == 2 * 2 * 128 * 128 * 4 + 2 * 65536


def test_forward_workspace_grows_with_frames(L):
    a = vdn.vdn_forward_workspace_bytes(_shape(T=10))
    b = vdn.vdn_forward_workspace_bytes(_shape(T=20))
    assert b > a
    # zero-size problems are valid and need no device work
    s = _shape(B=0)
    assert L.vdn_frame_grams(_p(s), None, None, None, None, None, None, None) == vdn.VDN_OK
    assert L.vdn_chunk_readout(_p(s), None, None, None, None, None, None) == vdn.VDN_OK


def test_binding_refuses_host_tensors(L):
    import torch
    s = _shape()
    x = torch.zeros(4)
    with pytest.raises(vdn.VdnError):
        vdn.vdn_frame_grams(s, x, x, x, x, x)


def test_pipelined_validation(L):
    s = _shape()  # float32, d = 16: not the tensor path
    need = vdn.vdn_forward_workspace_bytes(s)
    ev = (ctypes.c_void_p * 10)(*([16] * 10))
    evp = ctypes.cast(ev, ctypes.c_void_p)
    args = [_p(s)] + [16] * 11 + [256, need, 16]  # Q..O, F, G, workspace, bytes, info
    assert L.vdn_forward_pipelined(*args, 2, None, evp, None, None) == vdn.VDN_ERR_UNSUPPORTED
    s2 = _shape(d=128, in_dtype="bf16")
    args[0] = _p(s2)
    args[13] = vdn.vdn_forward_workspace_bytes(s2)
    assert L.vdn_forward_pipelined(*args, 0, None, evp, None, None) == vdn.VDN_ERR_INVALID
    assert "groups" in vdn.vdn_last_error()
    assert L.vdn_forward_pipelined(*args, 2, None, None, None, None) == vdn.VDN_ERR_INVALID
    assert "events" in vdn.vdn_last_error()
    ev[9] = None  # 8 + 2 = 10 events, one missing
    assert L.vdn_forward_pipelined(*args, 2, None, evp, None, None) == vdn.VDN_ERR_INVALID
    assert "events[9]" in vdn.vdn_last_error()


def test_beta_per_token_flag_is_checked(L):
    s = _shape()
    s.beta_per_token = 2
    assert L.vdn_frame_grams(_p(s), 16, 16, 16, 16, 16, None, None) == vdn.VDN_ERR_INVALID
    assert "beta_per_token" in vdn.vdn_last_error()
    assert L.vdn_text_state_noalloc(_p(s), 16, 16, 16, 16, 16, None) == vdn.VDN_ERR_INVALID
    assert vdn.shape_for(vdn_synth().WORKLOADS["h3_tb"]).beta_per_token == 1


def vdn_synth():
    from frame_wise_delta_b200 import synth
    return synth


def test_gated_readout_validation(L):
    s = _shape()
    og = vdn.vdn_out_gate(16, 16, 1e-6)
    ogp = ctypes.cast(ctypes.pointer(og), ctypes.c_void_p)
    assert L.vdn_chunk_readout_gated(_p(s), 16, 16, 16, None, 16, None, None) == vdn.VDN_ERR_INVALID
    assert "og is NULL" in vdn.vdn_last_error()
    og.eps = 0.0
    assert L.vdn_chunk_readout_gated(_p(s), 16, 16, 16, ogp, 16, None, None) == vdn.VDN_ERR_INVALID
    assert "eps" in vdn.vdn_last_error()
    og.eps, og.gate = 1e-6, 0x1004
    assert L.vdn_chunk_readout_gated(_p(s), 16, 16, 16, ogp, 16, None, None) == vdn.VDN_ERR_INVALID
    assert "og->gate" in vdn.vdn_last_error()


def _declared_arity():
    """Parameter count of every function include/vdn.h declares."""
    import re
    with open(vdn.HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(vdn_\w+)\s*\(([^)]*)\)\s*;", text):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_signatures_match_the_header(L):
    arity = _declared_arity()
    for name, args in vdn._SIGS.items():
        assert name in arity, name
        assert len(args) == arity[name], (name, len(args), arity[name])
    # every status-returning entry point of the header has a binding signature
    ret_other = {"vdn_status_string", "vdn_last_error", "vdn_version", "vdn_text_state_workspace_bytes",
                 "vdn_forward_workspace_bytes", "vdn_stream_workspace_bytes"}
    assert set(arity) - ret_other == set(vdn._SIGS)


def test_decay_bridge_flag_checks(L):
    s = _shape()
    s.decay_bridge = 2
    assert L.vdn_chunk_readout(_p(s), 16, 16, 16, 16, None, None) == vdn.VDN_ERR_INVALID
    s.decay_bridge = 1
    # the plain readouts have no alpha to bridge with
    assert L.vdn_chunk_readout(_p(s), 16, 16, 16, 16, None, None) == vdn.VDN_ERR_INVALID
    assert "vdn_chunk_readout_bridged" in vdn.vdn_last_error()
    # the bridged readout needs alpha
    assert L.vdn_chunk_readout_bridged(_p(s), 16, 16, 16, None, None, 16, None, None) == vdn.VDN_ERR_INVALID
    s.decay_bridge = 0
    assert L.vdn_chunk_readout_bridged(_p(s), 16, 16, 16, 16, None, 16, None, None) == vdn.VDN_ERR_INVALID


@pytest.mark.parametrize("frame0", [-5, 3, 7])
def test_stream_segment_frame0_checks(L, frame0):
    s = _shape()
    st = L.vdn_stream_segment(_p(s), 16, 16, 16, 16, 16, frame0, 16, 16, 16, 16, 256, 1 << 30, 16, None)
    assert st == vdn.VDN_ERR_INVALID
    assert "frame0" in vdn.vdn_last_error()


def test_stream_segment_rejects_the_decay_bridge(L):
    s = _shape()
    s.decay_bridge = 1
    st = L.vdn_stream_segment(_p(s), 16, 16, 16, 16, 16, 0, 16, 16, 16, 16, 256, 1 << 30, 16, None)
    assert st == vdn.VDN_ERR_UNSUPPORTED


def test_selftest_wait_needs_info(L):
    assert L.vdn_selftest_wait(None, None) == vdn.VDN_ERR_INVALID


@pytest.mark.parametrize("kw", [dict(chunk=0), dict(chunk=17), dict(anchors=2), dict(T=-1)])
def test_noalloc_applies_the_same_shape_rules(L, kw):
    """vdn_text_state_noalloc rejects every shape vdn_text_state rejects, with
    the same status, before it touches the device."""
    s = _shape(**kw)
    a = L.vdn_text_state(_p(s), 16, 16, 16, 16, 16, 1 << 20, 16, None)
    b = L.vdn_text_state_noalloc(_p(s), 16, 16, 16, 16, 16, None)
    assert a == b == vdn.VDN_ERR_INVALID
    for flag in ("decay_bridge", "out_dtype"):
        s = _shape()
        setattr(s, flag, 5)
        assert L.vdn_text_state_noalloc(_p(s), 16, 16, 16, 16, 16, None) == vdn.VDN_ERR_INVALID


def test_bridged_stream_segment_checks(L):
    args = lambda s, frame0: (_p(s), 16, 16, 16, 16, 16, frame0, 16, 16, None, 16, 16, None, 16, 1 << 30, 16, None)
    # needs the decay_bridge flag
    assert L.vdn_stream_segment_bridged(*args(_shape(), 0)) == vdn.VDN_ERR_INVALID
    assert "decay_bridge" in vdn.vdn_last_error()
    s = _shape()
    s.decay_bridge = 1
    assert L.vdn_stream_segment_bridged(*args(s, 3)) == vdn.VDN_ERR_INVALID  # frame0 not a chunk multiple
    assert "frame0" in vdn.vdn_last_error()
    # misaligned carried product
    a = list(args(s, 5))
    a[9] = 18
    assert L.vdn_stream_segment_bridged(*a) == vdn.VDN_ERR_INVALID
    assert "alpha_prev" in vdn.vdn_last_error()
