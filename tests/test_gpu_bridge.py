"""GPU parity of the decay-bridge readout ("Method steps" step (5)) against
the fp64 oracle (bridged_readout / vda_head(bridge=True)).

The workloads draw the decay gates from U(0.6, 1) so that the bridge moves
the readout well beyond the tolerance (checked: the plain readout fails the
same bound). Cases: the stage call on the tensor-core and CUDA-core readouts
(with and without the gated epilogue), the fused passes (vdn_forward and its
two-stream form, bit-equal), a full-size H3 sample, and the argument checks.
Bounds: 1e-4 for float32 inputs, 2e-2 for bf16 inputs with a float32 state.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from frame_wise_delta_b200 import synth, vdn
from vdn_testlib import TOL, device_fill, device_inputs, rel, tdtype, to_dev

pytestmark = pytest.mark.gpu
EPS = 1e-6


def custom(name, **kw):
    base = dict(name=name, index=90, B=1, H=2, T=12, U=300, d=128, n_text=40, dtype="bf16", alpha_lo=0.6,
                anchors=1, decay_bridge=True)
    base.update(kw)
    return synth.Workload(**base)


TC = custom("bridge_tc")
TC_TB = custom("bridge_tc_tb", index=91, B=2, H=1, T=23, U=200, beta_per_token=True)
BF16_D64 = custom("bridge_bf16_d64", index=92, d=64, U=130, T=17)
F32_D32 = custom("bridge_f32_d32", index=93, dtype="f32", d=32, U=70, T=13, anchors=0, n_text=5)
CASES = [TC, TC_TB, BF16_D64, F32_D32]


@pytest.fixture(scope="module", autouse=True)
def _build():
    from frame_wise_delta_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _heads(w, full, bridge=True):
    return {(b, h): oracle.vda_head({k: full[k][b, h] for k in full}, w.chunk, w.anchors, bridge=bridge)
            for b in range(w.B) for h in range(w.H)}


def _stack(w, ref, key):
    return np.stack([np.stack([ref[(b, h)][key] for h in range(w.H)]) for b in range(w.B)])


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("gated", [False, True], ids=["plain", "gated"])
def test_readout_bridged_stage(w, gated):
    full = synth.generate_all(w)
    ref = _heads(w, full)
    plain = _heads(w, full, bridge=False)
    s = vdn.shape_for(w)
    O = torch.full((w.B, w.H, w.T, w.U, w.d), float("nan"), dtype=tdtype(w), device="cuda")
    og, want = None, {k: r["O"] for k, r in ref.items()}
    if gated:
        rng = np.random.default_rng(100 + w.index)
        g = (2.0 * rng.standard_normal((w.B, w.H, w.T, w.U, w.d))).astype(np.float32)
        if w.dtype == "bf16":
            g = synth.round_bf16(g)
        nw = rng.uniform(0.5, 1.5, (w.H, w.d)).astype(np.float32)
        gd, nwd = to_dev(g, tdtype(w)), to_dev(nw)
        og = vdn.out_gate(gd, nwd, EPS)
        want = {(b, h): oracle.gated_rmsnorm(ref[(b, h)]["O"], nw[h], g[b, h], EPS) for (b, h) in ref}
    vdn.vdn_chunk_readout_bridged(s, to_dev(full["Q"], tdtype(w)), to_dev(_stack(w, ref, "F")),
                                  to_dev(_stack(w, ref, "G")), to_dev(full["alpha"]), og, O)
    torch.cuda.synchronize()
    assert not torch.isnan(O.float()).any()
    tol = TOL[w.dtype] if not gated else (3e-3 if w.dtype == "bf16" else 1e-5)
    for (b, h), y in want.items():
        e = rel(O[b, h], y)
        print(f"{w.name} {'gated' if gated else 'plain'} b{b} h{h}: {e:.2e}")
        assert e <= tol, e
        if not gated:
            # the bridge matters at this bound: the readout without it is far off
            assert rel(plain[(b, h)]["O"], y) > 10 * tol


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_forward_bridged(w):
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    args = (dev["Q"], dev["K"], dev["V"], dev["beta"], dev["alpha"], dev["Kx"], dev["Vx"], dev["beta_x"])
    fw = vdn.Forward(vdn.shape_for(w))
    fw(*args)
    torch.cuda.synchronize()
    assert int(fw.info.item()) == 0
    ref = _heads(w, full)
    tol = TOL[w.dtype]
    for (b, h), r in ref.items():
        eo, ef, eg = rel(fw.O[b, h], r["O"]), rel(fw.F[b, h], r["F"]), rel(fw.G[b, h], r["G"])
        print(f"{w.name} b{b} h{h}: O {eo:.2e} F {ef:.2e} G {eg:.2e}")
        assert eo <= tol and ef <= tol and eg <= tol
    if w.dtype == "bf16" and w.d == 128:
        pw = vdn.PipelinedForward(vdn.shape_for(w), groups=2)
        pw(*args)
        torch.cuda.synchronize()
        assert int(pw.info.item()) == 0
        assert torch.equal(pw.O, fw.O)


def test_full_size_h3_bridged():
    w = dataclasses.replace(synth.WORKLOADS["h3"], name="h3_bridge", decay_bridge=True)
    pairs = [(0, 5), (0, 17)]
    sampled = {(b, h): synth.generate_head(w, b, h) for b, h in pairs}
    dev = device_fill(w, sampled, seed=w.seed)
    fw = vdn.Forward(vdn.shape_for(w))
    fw(dev["Q"], dev["K"], dev["V"], dev["beta"], dev["alpha"], dev["Kx"], dev["Vx"], dev["beta_x"])
    torch.cuda.synchronize()
    assert int(fw.info.item()) == 0
    assert torch.isfinite(fw.O.float()).all()
    for (b, h), inp in sampled.items():
        r = oracle.vda_head(inp, w.chunk, w.anchors, bridge=True)
        eo = rel(fw.O[b, h], r["O"])
        print(f"h3 bridge b{b} h{h}: O {eo:.2e}")
        assert eo <= TOL["bf16"]
    del dev, fw
    torch.cuda.empty_cache()


def test_argument_checks():
    w = F32_D32
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    s = vdn.shape_for(w)
    z = torch.zeros((w.B, w.H, w.C + 1, w.d, w.d), device="cuda")
    O = torch.empty((w.B, w.H, w.T, w.U, w.d), device="cuda")
    with pytest.raises(vdn.VdnError):  # the plain stage call has no alpha
        vdn.vdn_chunk_readout(s, dev["Q"], z, z, O)
    with pytest.raises(vdn.VdnError):
        vdn.vdn_chunk_readout_bridged(s, dev["Q"], z, z, None, None, O)
    s0 = vdn.shape_for(dataclasses.replace(w, decay_bridge=False))
    with pytest.raises(vdn.VdnError):  # bridged call without the flag
        vdn.vdn_chunk_readout_bridged(s0, dev["Q"], z, z, dev["alpha"], None, O)
    # a stream segment cannot bridge into the previous segment
    ws = vdn.workspace(vdn.vdn_stream_workspace_bytes(s))
    S = torch.zeros((w.B, w.H, w.d, w.d), device="cuda")
    F = torch.empty((w.B, w.H, w.C + 1, w.d, w.d), device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(vdn.VdnError) as e:
        vdn.vdn_stream_segment(s, dev["Q"], dev["K"], dev["V"], dev["beta"], dev["alpha"], 0, S, S, O, F, ws, info)
    assert e.value.status == vdn.VDN_ERR_UNSUPPORTED


@pytest.mark.parametrize("T", [1, 2, 4, 6, 11])
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (32, "f32")], ids=["tc", "f32"])
def test_short_clips(T, d, dtype):
    """Clips of one to three chunks, where every window reaches both ends
    (and with T = 1, 2 every frame is an anchor)."""
    w = custom(f"bridge_T{T}_{dtype}", index=94, T=T, d=d, dtype=dtype, U=70, n_text=7)
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    fw = vdn.Forward(vdn.shape_for(w))
    fw(dev["Q"], dev["K"], dev["V"], dev["beta"], dev["alpha"], dev["Kx"], dev["Vx"], dev["beta_x"])
    torch.cuda.synchronize()
    assert int(fw.info.item()) == 0
    for (b, h), r in _heads(w, full).items():
        eo = rel(fw.O[b, h], r["O"])
        print(f"T={T} {dtype} b{b} h{h}: O {eo:.2e}")
        assert eo <= TOL[dtype]
        if T <= 2:
            assert torch.count_nonzero(fw.O[b, h]) == 0
