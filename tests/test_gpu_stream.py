"""GPU parity of the causal streaming call (vdn_stream_segment) against the
fp64 streaming oracle (oracle.stream_segment).

Cases: the tensor-core path (bf16, d = 128, ragged tokens and a ragged last
chunk), the CUDA-core path on bf16 (d = 64) and on float32 (d = 32); a stream
cut into segments against the same stream in one call (the carried states
are the only link, so the outputs must be equal); the first-frame anchor
only at frame0 = 0; the frame0 checks; the full-size H3 stream on sampled
heads. Bounds as for the bidirectional pass: 1e-4 for float32 inputs,
2e-2 for bf16 inputs with a float32 state.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from frame_wise_delta_b200 import synth, vdn
from vdn_testlib import OUT_GUARD, STATE_GUARD, TOL, device_fill, device_inputs, rel, to_dev

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def custom(name, **kw):
    base = dict(name=name, index=70, B=1, H=2, T=12, U=300, d=128, n_text=40, dtype="bf16",
                alpha_lo=0.9, anchors=1)
    base.update(kw)
    return synth.Workload(**base)


TC = custom("stream_tc")
TC_TB = custom("stream_tc_tb", index=71, H=3, T=13, U=200, beta_per_token=True)
BF16_D64 = custom("stream_bf16_d64", index=72, d=64, U=130, T=17)
F32_D32 = custom("stream_f32_d32", index=73, dtype="f32", d=32, U=70, T=13, anchors=0, n_text=5)
CASES = [TC, TC_TB, BF16_D64, F32_D32]


@pytest.fixture(scope="module", autouse=True)
def _build():
    from frame_wise_delta_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _states(w, full, seed):
    """S_prev, S_in per (b, h): the text state, and (for a later segment) a
    seeded perturbation of it so that the two carried states differ."""
    rng = np.random.default_rng(seed)
    ST = np.zeros((w.B, w.H, w.d, w.d))
    for b in range(w.B):
        for h in range(w.H):
            ST[b, h] = oracle.text_state(full["Kx"][b, h], full["Vx"][b, h], full["beta_x"][b, h])
    S_prev = ST + 0.3 * rng.standard_normal(ST.shape)
    S_in = ST + 0.3 * rng.standard_normal(ST.shape)
    return ST, S_prev, S_in


def _segment(w, dev, frame0, S_prev, S_in, T=None, t0=0):
    T = w.T if T is None else T
    s = vdn.make_shape(w.B, w.H, T, w.U, w.d, w.n_text, w.chunk, w.anchors, w.dtype,
                       beta_per_token=w.beta_per_token)
    ws = vdn.workspace(vdn.vdn_stream_workspace_bytes(s))
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    dt = dev["Q"].dtype
    O = torch.full((w.B, w.H, T, w.U, w.d), float("nan"), dtype=dt, device="cuda")
    F = torch.full((w.B, w.H, s.C + 1, w.d, w.d), float("nan"), device="cuda")
    sl = slice(t0, t0 + T)
    part = {k: dev[k][:, :, sl].contiguous() for k in ("Q", "K", "V", "beta", "alpha")}
    vdn.vdn_stream_segment(s, part["Q"], part["K"], part["V"], part["beta"], part["alpha"], frame0,
                           S_prev, S_in, O, F, ws, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    return O, F


def _oracle(w, full, S_prev, S_in, anchor_first, t0=0, T=None):
    T = w.T if T is None else T
    out = {}
    for b in range(w.B):
        for h in range(w.H):
            sl = slice(t0, t0 + T)
            out[(b, h)] = oracle.stream_segment(full["Q"][b, h][sl], full["K"][b, h][sl], full["V"][b, h][sl],
                                                full["beta"][b, h][sl], full["alpha"][b, h][sl], S_prev[b, h],
                                                S_in[b, h], w.chunk, anchor_first)
    return out


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("first", [True, False], ids=["frame0", "later"])
def test_segment_matches_oracle(w, first):
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    ST, S_prev, S_in = _states(w, full, w.seed)
    if first:
        S_prev = S_in = ST
    frame0 = 0 if first else 3 * w.chunk
    O, F = _segment(w, dev, frame0, to_dev(S_prev), to_dev(S_in))
    ref = _oracle(w, full, S_prev, S_in, anchor_first=bool(w.anchors) and first)
    tol = TOL[w.dtype]
    for (b, h), (Or, Fr) in ref.items():
        eo, ef = rel(O[b, h], Or), rel(F[b, h], Fr)
        print(f"{w.name} frame0={frame0} b{b} h{h}: O {eo:.2e} F {ef:.2e}")
        assert eo <= tol and ef <= tol
        # F[0] is S_in as given
        assert torch.equal(F[b, h, 0], to_dev(S_in[b, h]))
    if w.anchors and first:
        assert torch.count_nonzero(O[:, :, 0]) == 0
    assert torch.isfinite(O.float()).all()


@pytest.mark.parametrize("w", [TC, BF16_D64, F32_D32], ids=lambda w: w.name)
def test_segments_equal_one_call(w):
    """Cut at chunk boundaries and carried through (F[C-1], F[C]), the stream
    gives the outputs and states of a single call, element for element."""
    w = dataclasses.replace(w, name=w.name + "_long", T=22)
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    ST, _, _ = _states(w, full, w.seed)
    S = to_dev(ST)
    O, F = _segment(w, dev, 0, S, S)
    Os, Fs = [], [F[:, :, :1]]
    S_prev, S_in = S, S
    for t0, T in ((0, 10), (10, 5), (15, 7)):
        Oi, Fi = _segment(w, dev, t0, S_prev, S_in, T=T, t0=t0)
        Os.append(Oi)
        Fs.append(Fi[:, :, 1:])
        C = Fi.shape[2] - 1
        S_prev, S_in = Fi[:, :, C - 1].contiguous(), Fi[:, :, C].contiguous()
    assert torch.equal(torch.cat(Os, dim=2), O)
    assert torch.equal(torch.cat(Fs, dim=2), F)


def test_stream_class_matches_oracle():
    """vdn.Stream carries the states between equal segments."""
    w = custom("stream_cls", index=74, T=20)
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    ST, _, _ = _states(w, full, w.seed)
    s = vdn.make_shape(w.B, w.H, 10, w.U, w.d, w.n_text, w.chunk, w.anchors, w.dtype)
    st = vdn.Stream(s, to_dev(ST))
    outs = []
    for t0 in (0, 10):
        part = {k: dev[k][:, :, t0:t0 + 10].contiguous() for k in ("Q", "K", "V", "beta", "alpha")}
        outs.append(st(part["Q"], part["K"], part["V"], part["beta"], part["alpha"]).clone())
    torch.cuda.synchronize()
    ref = _oracle(w, full, ST, ST, anchor_first=True)
    O = torch.cat(outs, dim=2)
    for (b, h), (Or, Fr) in ref.items():
        assert rel(O[b, h], Or) <= TOL["bf16"]
        assert rel(st.S_in[b, h], Fr[-1]) <= TOL["bf16"]
        assert rel(st.S_prev[b, h], Fr[-2]) <= TOL["bf16"]


def test_frame0_checks():
    w = F32_D32
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    S = torch.zeros((w.B, w.H, w.d, w.d), device="cuda")
    for frame0 in (-5, 3, 7):
        with pytest.raises(vdn.VdnError):
            _segment(w, dev, frame0, S, S)


def test_empty_segment():
    """T = 0: F[0] = S_in and nothing else is read or written."""
    s = vdn.make_shape(1, 2, 0, 16, 32, 4, 5, 1, "f32")
    ws = vdn.workspace(vdn.vdn_stream_workspace_bytes(s))
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    S_in = torch.randn((1, 2, 32, 32), device="cuda")
    F = torch.full((1, 2, 1, 32, 32), float("nan"), device="cuda")
    vdn.vdn_stream_segment(s, None, None, None, None, None, 0, S_in, S_in, None, F, ws, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    assert torch.equal(F[:, :, 0], S_in)


@pytest.mark.parametrize("pairs", [[(0, 0), (0, 23)]])
def test_full_size_h3_stream(pairs):
    """The H3 clip (102 frames, 1008 tokens, 24 heads) streamed in one call."""
    w = W["h3"]
    sampled = {(b, h): synth.generate_head(w, b, h) for b, h in pairs}
    dev = device_fill(w, sampled, seed=w.seed)
    ST = torch.zeros((w.B, w.H, w.d, w.d), device="cuda")
    for (b, h), inp in sampled.items():
        ST[b, h] = to_dev(oracle.text_state(inp["Kx"], inp["Vx"], inp["beta_x"]))
    O, F = _segment(w, dev, 0, ST, ST)
    assert torch.isfinite(O.float()).all()
    for (b, h), inp in sampled.items():
        S = ST[b, h].double().cpu().numpy()
        Or, Fr = oracle.stream_segment(inp["Q"], inp["K"], inp["V"], inp["beta"], inp["alpha"], S, S, w.chunk,
                                       True)
        eo, ef = rel(O[b, h], Or), rel(F[b, h], Fr)
        print(f"h3 stream b{b} h{h}: O {eo:.2e} F {ef:.2e}")
        assert eo <= TOL["bf16"] and ef <= TOL["bf16"]
        assert ef <= STATE_GUARD and eo <= OUT_GUARD["bf16"], (ef, eo)
    del dev
    torch.cuda.empty_cache()


# ------------------------------------------------ decay bridge in segments
def _bridged_segment(w, dev, frame0, S_prev, S_in, alpha_prev, T=None, t0=0):
    T = w.T if T is None else T
    s = vdn.make_shape(w.B, w.H, T, w.U, w.d, w.n_text, w.chunk, w.anchors, w.dtype,
                       beta_per_token=w.beta_per_token, decay_bridge=True)
    ws = vdn.workspace(vdn.vdn_stream_workspace_bytes(s))
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    dt = dev["Q"].dtype
    O = torch.full((w.B, w.H, T, w.U, w.d), float("nan"), dtype=dt, device="cuda")
    F = torch.full((w.B, w.H, s.C + 1, w.d, w.d), float("nan"), device="cuda")
    tail = torch.full((w.B, w.H, w.d), float("nan"), device="cuda")
    sl = slice(t0, t0 + T)
    part = {k: dev[k][:, :, sl].contiguous() for k in ("Q", "K", "V", "beta", "alpha")}
    vdn.vdn_stream_segment_bridged(s, part["Q"], part["K"], part["V"], part["beta"], part["alpha"], frame0,
                                   S_prev, S_in, alpha_prev, O, F, tail, ws, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    return O, F, tail


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("first", [True, False], ids=["frame0", "later"])
def test_bridged_segment_matches_oracle(w, first):
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    ST, S_prev, S_in = _states(w, full, w.seed + 1)
    rng = np.random.default_rng(w.seed + 2)
    a_prev = rng.uniform(0.5, 1.0, (w.B, w.H, w.d))
    if first:
        S_prev = S_in = ST
        a_prev = np.ones_like(a_prev)
    frame0 = 0 if first else 3 * w.chunk
    anchor_first = bool(w.anchors) and first
    O, F, tail = _bridged_segment(w, dev, frame0, to_dev(S_prev), to_dev(S_in), None if first else to_dev(a_prev))
    tol = TOL[w.dtype]
    for b in range(w.B):
        for h in range(w.H):
            Or, Fr = oracle.stream_segment(full["Q"][b, h], full["K"][b, h], full["V"][b, h], full["beta"][b, h],
                                           full["alpha"][b, h], S_prev[b, h], S_in[b, h], w.chunk, anchor_first,
                                           bridge=True, alpha_prev=a_prev[b, h])
            eo, ef = rel(O[b, h], Or), rel(F[b, h], Fr)
            et = rel(tail[b, h], oracle.stream_bridge_tail(full["alpha"][b, h], w.chunk, anchor_first))
            print(f"{w.name} bridged frame0={frame0} b{b} h{h}: O {eo:.2e} F {ef:.2e} tail {et:.2e}")
            assert eo <= tol and ef <= tol and et <= 1e-6
            assert ef <= STATE_GUARD and eo <= OUT_GUARD[w.dtype]
    assert torch.isfinite(O.float()).all()


@pytest.mark.parametrize("w", [TC, F32_D32], ids=lambda w: w.name)
def test_bridged_segments_equal_one_call(w):
    """A bridged stream cut at chunk boundaries, carrying (F[C-1], F[C]) and
    the last chunk's decay product, gives the outputs of a single call."""
    w = dataclasses.replace(w, name=w.name + "_bridged_long", T=22)
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    ST, _, _ = _states(w, full, w.seed)
    S = to_dev(ST)
    O, F, _ = _bridged_segment(w, dev, 0, S, S, None)
    Os = []
    S_prev, S_in, a_prev = S, S, None
    for t0, T in ((0, 10), (10, 5), (15, 7)):
        Oi, Fi, tail = _bridged_segment(w, dev, t0, S_prev, S_in, a_prev, T=T, t0=t0)
        Os.append(Oi)
        C = Fi.shape[2] - 1
        S_prev, S_in, a_prev = Fi[:, :, C - 1].contiguous(), Fi[:, :, C].contiguous(), tail
    # the segments' chunks run the same kernels on the same inputs, except
    # the bridge factor of each segment's chunk 0, formed from the carried
    # product instead of in one loop: equal to fp32 rounding
    e = rel(torch.cat(Os, dim=2), O.double().cpu().numpy())
    print(f"{w.name}: bridged segments vs one call {e:.2e}")
    assert e <= (1e-6 if w.dtype == "f32" else 4e-3)


def test_stream_class_carries_the_bridge():
    w = dataclasses.replace(TC, name="stream_tc_class_bridged", T=20, anchors=1)
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    ST, _, _ = _states(w, full, w.seed)
    seg = vdn.make_shape(w.B, w.H, 10, w.U, w.d, w.n_text, w.chunk, w.anchors, w.dtype, decay_bridge=True)
    st = vdn.Stream(seg, to_dev(ST))
    outs = []
    for t0 in (0, 10):
        part = {k: dev[k][:, :, t0:t0 + 10].contiguous() for k in ("Q", "K", "V", "beta", "alpha")}
        outs.append(st(part["Q"], part["K"], part["V"], part["beta"], part["alpha"]).clone())
    torch.cuda.synchronize()
    assert int(st.info.item()) == 0
    O = torch.cat(outs, dim=2)
    for b in range(w.B):
        for h in range(w.H):
            Or, _ = oracle.stream_segment(full["Q"][b, h], full["K"][b, h], full["V"][b, h], full["beta"][b, h],
                                          full["alpha"][b, h], ST[b, h], ST[b, h], w.chunk, True, bridge=True)
            e = rel(O[b, h], Or)
            print(f"stream class bridged b{b} h{h}: O {e:.2e}")
            assert e <= OUT_GUARD["bf16"]
