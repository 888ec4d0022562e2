"""vdn_text_state_noalloc against vdn_text_state and the fp64 oracle.

The no-allocation entry point serves callers that cannot give the library a
device workspace (a fixed memory plan, or a loop that must not call
cudaMalloc); it keeps its scratch in a fixed device array instead. It must
give the same text state as the workspace version, call after call, although
every call reuses (and leaves behind) the same scratch; and since it factors
on another route than the workspace version (the CUDA-core factor kernel),
its result is also held to the oracle's text state directly. This file is
collected last so that a run stopping at the first failure has run every
other test.
"""
import pytest
import torch

import oracle
from frame_wise_delta_b200 import synth, vdn
from vdn_testlib import device_inputs, rel

pytestmark = pytest.mark.gpu

# two different problems in a row: the second call must not see the first
# call's scratch (bf16 d=128 uses the tensor-core Gram, f32 d=64 the CUDA-core one)
CASES = [
    synth.Workload("noalloc_a", 60, B=2, H=12, T=1, U=1, d=128, n_text=512, dtype="bf16", alpha_lo=0.95, anchors=0),
    synth.Workload("noalloc_b", 61, B=1, H=3, T=1, U=1, d=128, n_text=77, dtype="bf16", alpha_lo=0.95, anchors=0),
    synth.Workload("noalloc_c", 62, B=1, H=5, T=1, U=1, d=64, n_text=40, dtype="f32", alpha_lo=0.95, anchors=0),
]


def _with_workspace(w, dev):
    s = vdn.shape_for(w)
    out = torch.empty((w.B, w.H, w.d, w.d), device="cuda")
    ws = vdn.workspace(vdn.vdn_text_state_workspace_bytes(s))
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_text_state(s, dev["Kx"], dev["Vx"], dev["beta_x"], out, ws, info)
    return out, info


def _no_alloc(w, dev):
    s = vdn.shape_for(w)
    out = torch.full((w.B, w.H, w.d, w.d), float("nan"), device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    vdn.vdn_text_state_noalloc(s, dev["Kx"], dev["Vx"], dev["beta_x"], out, info)
    return out, info


def test_no_alloc_text_state_matches_workspace_version():
    torch.cuda.set_device(0)
    for round_ in range(2):
        for w in CASES:
            dev = device_inputs(w, synth.generate_all(w))
            ref, info_ref = _with_workspace(w, dev)
            got, info = _no_alloc(w, dev)
            torch.cuda.synchronize()
            assert int(info.item()) == 0 and int(info_ref.item()) == 0
            assert torch.isfinite(got).all()
            e = rel(got, ref.double().cpu().numpy())
            assert e <= 1e-5, (round_, w.name, e)


def test_no_alloc_text_state_matches_the_oracle():
    """Each case twice in a row, against the fp64 text state of the same
    (bf16-rounded where the case is bf16) inputs: the route's only error is
    its float32 arithmetic."""
    torch.cuda.set_device(0)
    for round_ in range(2):
        for w in CASES:
            full = synth.generate_all(w)
            dev = device_inputs(w, full)
            got, info = _no_alloc(w, dev)
            torch.cuda.synchronize()
            assert int(info.item()) == 0
            for b in range(w.B):
                for h in range(w.H):
                    ref = oracle.text_state(full["Kx"][b, h], full["Vx"][b, h], full["beta_x"][b, h])
                    e = rel(got[b, h], ref)
                    assert e <= 1e-5, (round_, w.name, b, h, e)


def test_no_alloc_rejects_sizes_beyond_its_scratch():
    w = synth.Workload("noalloc_big", 63, B=1, H=33, T=1, U=1, d=128, n_text=8, dtype="bf16",
                       alpha_lo=0.95, anchors=0)
    s = vdn.shape_for(w)
    with pytest.raises(vdn.VdnError) as e:
        vdn.vdn_text_state_noalloc(s, None, None, None, None, None)
    assert e.value.status == vdn.VDN_ERR_UNSUPPORTED
    assert "scratch" in str(e.value)
