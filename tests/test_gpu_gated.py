"""GPU parity of the readout epilogue of step (5) (RMSNorm over each token's
channels, then a sigmoid gate) against the fp64 oracle: the stage call on the
CUDA-core and tensor-core readouts, the fused passes (vdn_forward and its
two-stream form, bit-equal to each other), and a full-size H3 sample.
Bounds: 1e-4 for float32 outputs, 2e-2 for bf16 ones (the output rounding
alone is ~2^-9 / sqrt(3))."""
import numpy as np
import pytest
import torch

import oracle
from frame_wise_delta_b200 import synth, vdn
from test_gpu_parity import SMALL_CASES, TC_SMALL, custom
from vdn_testlib import TOL, device_fill, device_inputs, oracle_heads, rel, tdtype, to_dev

pytestmark = pytest.mark.gpu
EPS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _build():
    from frame_wise_delta_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _gate_inputs(w, seed):
    """Gate logits ~ N(0, 2^2) (rounded to the input dtype) and RMSNorm weights
    ~ U(0.5, 1.5) per head and channel."""
    rng = np.random.default_rng(seed)
    g = (2.0 * rng.standard_normal((w.B, w.H, w.T, w.U, w.d))).astype(np.float32)
    if w.dtype == "bf16":
        g = synth.round_bf16(g)
    nw = rng.uniform(0.5, 1.5, (w.H, w.d)).astype(np.float32)
    return g, nw


def _expected(w, ref, g, nw, b, h):
    return oracle.gated_rmsnorm(ref[(b, h)]["O"], nw[h], g[b, h], EPS)


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_chunk_readout_gated(w):
    full = synth.generate_all(w)
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    ref = oracle_heads(w, full, pairs)
    Fr = np.stack([np.stack([ref[(b, h)]["F"] for h in range(w.H)]) for b in range(w.B)])
    Gr = np.stack([np.stack([ref[(b, h)]["G"] for h in range(w.H)]) for b in range(w.B)])
    g, nw = _gate_inputs(w, 70 + w.index)
    gd, nwd = to_dev(g, tdtype(w)), to_dev(nw)
    s = vdn.shape_for(w)
    Y = torch.full((w.B, w.H, w.T, w.U, w.d), float("nan"), dtype=tdtype(w), device="cuda")
    og = vdn.out_gate(gd, nwd, EPS)
    vdn.vdn_chunk_readout_gated(s, to_dev(full["Q"], tdtype(w)), to_dev(Fr), to_dev(Gr), og, Y)
    torch.cuda.synchronize()
    assert not torch.isnan(Y.float()).any()
    for b, h in pairs:
        e = rel(Y[b, h], _expected(w, ref, g, nw, b, h))
        print(f"{w.name} b{b} h{h}: Y {e:.2e}")
        assert e <= (3e-3 if w.dtype == "bf16" else 1e-5), (b, h, e)


@pytest.mark.parametrize("w", [synth.WORKLOADS["small"], TC_SMALL,
                               custom("tc_gated5", index=58, H=5, T=17, U=190)], ids=lambda w: w.name)
def test_forward_gated(w):
    full = synth.generate_all(w)
    dev = device_inputs(w, full)
    g, nw = _gate_inputs(w, 80 + w.index)
    gd, nwd = to_dev(g, tdtype(w)), to_dev(nw)
    og = vdn.out_gate(gd, nwd, EPS)
    args = (dev["Q"], dev["K"], dev["V"], dev["beta"], dev["alpha"], dev["Kx"], dev["Vx"], dev["beta_x"])
    fw = vdn.Forward(vdn.shape_for(w))
    fw(*args, og=og)
    torch.cuda.synchronize()
    assert int(fw.info.item()) == 0
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    ref = oracle_heads(w, full, pairs)
    for b, h in pairs:
        e = rel(fw.O[b, h], _expected(w, ref, g, nw, b, h))
        print(f"{w.name} b{b} h{h}: Y {e:.2e}")
        assert e <= TOL[w.dtype]
    if w.dtype == "bf16" and w.d == 128:
        pf = vdn.PipelinedForward(vdn.shape_for(w), groups=2)
        pf(*args, og=og)
        torch.cuda.synchronize()
        assert torch.equal(pf.O, fw.O)


def test_full_size_gated_sample():
    w = synth.WORKLOADS["h3"]
    pairs = [(0, 3), (0, 20)]
    sampled = {(b, h): synth.generate_head(w, b, h) for b, h in pairs}
    dev = device_fill(w, sampled, seed=w.seed)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99)
    gd = (2.0 * torch.randn((w.B, w.H, w.T, w.U, w.d), generator=gen, device="cuda")).to(torch.bfloat16)
    nwd = torch.rand((w.H, w.d), generator=gen, device="cuda") + 0.5
    fw = vdn.PipelinedForward(vdn.shape_for(w), groups=1)
    fw(dev["Q"], dev["K"], dev["V"], dev["beta"], dev["alpha"], dev["Kx"], dev["Vx"], dev["beta_x"],
       og=vdn.out_gate(gd, nwd, EPS))
    torch.cuda.synchronize()
    assert int(fw.info.item()) == 0
    for (b, h), inp in sampled.items():
        r = oracle.vda_head(inp, w.chunk, w.anchors)
        y = oracle.gated_rmsnorm(r["O"], nwd[h].double().cpu().numpy(), gd[b, h].double().cpu().numpy(), EPS)
        e = rel(fw.O[b, h], y)
        print(f"h3 gated b{b} h{h}: Y {e:.2e}")
        assert e <= TOL["bf16"]
    del dev, fw, gd
    torch.cuda.empty_cache()
