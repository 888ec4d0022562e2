"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Every stage is fed inputs computed by the oracle (never by the CUDA path) and
compared element by element (rel-Frobenius per (b, h)); the fused call is
compared end to end, on every config, at full size on sampled heads.
Bounds: 1e-4 for float32 inputs, 2e-2 for bf16 inputs with a float32 state.
"""
import numpy as np
import pytest
import torch

import oracle
from frame_wise_delta_b200 import synth, vdn
from vdn_testlib import OUT_GUARD, TOL, state_guard, device_fill, device_inputs, oracle_heads, rel, run_forward, tdtype, to_dev

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def custom(name, **kw):
    base = dict(name=name, index=40, B=1, H=2, T=12, U=300, d=128, n_text=40, dtype="bf16",
                alpha_lo=0.9, anchors=1)
    base.update(kw)
    return synth.Workload(**base)


# bf16, d = 128 (tensor-core kernels), ragged tokens (300 = 4*64 + 44 = 2*128 + 44)
# and a ragged last chunk (12 = 5 + 5 + 2).
TC_SMALL = custom("tc_small")
# several chunk boundaries outside every window, near-duplicate keys
TC_DUP = custom("tc_dup", index=41, B=2, H=1, T=23, U=200, n_text=17, near_dup=True)
# bf16 inputs on the CUDA-core path (d = 64)
BF16_D64 = custom("bf16_d64", index=42, d=64, U=130, T=17)
# float32 with d = 32, no anchors, ragged chunk
F32_D32 = custom("f32_d32", index=43, dtype="f32", d=32, U=70, T=13, anchors=0, n_text=5)

# per-token write gates beta_{t,u}: the tensor-core Gram (scaled K tiles), the
# CUDA-core Gram on bf16 and on float32 inputs
TC_TB = custom("tc_tb", index=56, B=1, H=3, T=13, U=200, n_text=40, beta_per_token=True)
BF16_D64_TB = custom("bf16_d64_tb", index=57, d=64, U=130, T=11, beta_per_token=True)

SMALL_CASES = [W["tiny"], W["small"], TC_SMALL, TC_DUP, BF16_D64, F32_D32, W["small_tb"], TC_TB, BF16_D64_TB]


def _full(w):
    return synth.generate_all(w)


@pytest.fixture(scope="module", autouse=True)
def _build():
    from frame_wise_delta_b200 import build
    build.build()
    assert torch.cuda.is_available()


# ------------------------------------------------------------- end to end
@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_forward_matches_oracle(w):
    full = _full(w)
    dev = device_inputs(w, full)
    fw = run_forward(w, dev)
    assert int(fw.info.item()) == 0
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    ref = oracle_heads(w, full, pairs)
    tol = TOL[w.dtype]
    for (b, h), r in ref.items():
        eo, ef, eg = rel(fw.O[b, h], r["O"]), rel(fw.F[b, h], r["F"]), rel(fw.G[b, h], r["G"])
        print(f"{w.name} b{b} h{h}: O {eo:.2e} F {ef:.2e} G {eg:.2e}")
        assert eo <= tol and ef <= tol and eg <= tol
        assert ef <= state_guard(w) and eg <= state_guard(w) and eo <= OUT_GUARD[w.dtype], (ef, eg, eo)


# ------------------------------------------------------------- per stage
def _stats_ref(w, full):
    A = np.zeros((w.B, w.H, w.T, w.d, w.d))
    B = np.zeros_like(A)
    for b in range(w.B):
        for h in range(w.H):
            for t in range(w.T):
                A[b, h, t], B[b, h, t] = oracle.frame_stats(full["K"][b, h, t], full["V"][b, h, t],
                                                            full["beta"][b, h, t])
    return A, B


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_frame_grams(w):
    full = _full(w)
    dev = device_inputs(w, full)
    s = vdn.shape_for(w)
    A = torch.empty((w.B, w.H, w.T, w.d, w.d), device="cuda")
    Bm = torch.empty_like(A)
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_frame_grams(s, dev["K"], dev["V"], dev["beta"], A, Bm, info)
    torch.cuda.synchronize()
    Ar, Br = _stats_ref(w, full)
    assert int(info.item()) == 0
    # products of bf16 values are exact in fp32; only the fp32 sums round
    assert rel(A, Ar) <= 1e-5 and rel(Bm, Br) <= 1e-5, (rel(A, Ar), rel(Bm, Br))


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_frame_factor(w):
    full = _full(w)
    Ar, Br = _stats_ref(w, full)
    s = vdn.shape_for(w)
    M = torch.empty((w.B, w.H, w.T, w.d, w.d), device="cuda")
    J = torch.empty_like(M)
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    vdn.vdn_frame_factor(s, to_dev(Ar), to_dev(Br), to_dev(full["alpha"]), M, J, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    Mr = np.zeros_like(Ar)
    Jr = np.zeros_like(Br)
    for b in range(w.B):
        for h in range(w.H):
            for t in range(w.T):
                Mr[b, h, t], Jr[b, h, t] = oracle.transition(Ar[b, h, t], Br[b, h, t], full["alpha"][b, h, t],
                                                             oracle.is_anchor(t, w.T, w.anchors))
    assert rel(M, Mr) <= 1e-5 and rel(J, Jr) <= 1e-5, (rel(M, Mr), rel(J, Jr))


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_frame_invert(w):
    full = _full(w)
    Ar, _ = _stats_ref(w, full)
    s = vdn.shape_for(w)
    W = torch.empty((w.B, w.H, w.T, w.d, w.d), device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    vdn.vdn_frame_invert(s, to_dev(Ar), W, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    ref = np.linalg.inv(np.eye(w.d) + Ar)
    # the tensor-core blocked sweep (bf16 shapes, d = 128) multiplies hi/lo
    # bf16 splits (each operand exact to ~2^-17): 1e-4, the fp32 bound; the
    # fp32 sweep: 1e-5. Its two triangles come from separate products (the
    # column block G_iK G_KK^{-1} and the pivot rows G_KK^{-1} G_Kj), so
    # symmetry holds to the inverse's own accuracy, not exactly.
    tc = w.dtype == "bf16" and w.d == 128
    e = rel(W, ref)
    Wc = W.double().cpu().numpy()
    asym = rel(np.swapaxes(Wc, -1, -2), Wc)
    print(f"{w.name}: invert rel {e:.2e} asym {asym:.2e}")
    assert e <= (1e-4 if tc else 1e-5), e
    if tc:
        assert asym <= 1e-4, asym
    else:
        assert np.allclose(Wc, np.swapaxes(Wc, -1, -2), rtol=0, atol=1e-6)


def _maps_ref(w, full):
    C = w.C
    out = [np.zeros((w.B, w.H, C, w.d, w.d)) for _ in range(4)]
    for b in range(w.B):
        for h in range(w.H):
            maps = oracle.chunk_maps(full["K"][b, h], full["V"][b, h], full["beta"][b, h], full["alpha"][b, h],
                                     w.chunk, w.anchors)
            for o, m in zip(out, maps):
                o[b, h] = m
    return out


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_chunk_compose(w):
    full = _full(w)
    Ar, Br = _stats_ref(w, full)
    Mt = np.zeros_like(Ar)
    Jt = np.zeros_like(Br)
    for b in range(w.B):
        for h in range(w.H):
            for t in range(w.T):
                Mt[b, h, t], Jt[b, h, t] = oracle.transition(Ar[b, h, t], Br[b, h, t], full["alpha"][b, h, t],
                                                             oracle.is_anchor(t, w.T, w.anchors))
    s = vdn.shape_for(w)
    outs = [torch.empty((w.B, w.H, w.C, w.d, w.d), device="cuda") for _ in range(4)]
    vdn.vdn_chunk_compose(s, to_dev(Mt), to_dev(Jt), *outs)
    torch.cuda.synchronize()
    for got, ref, name in zip(outs, _maps_ref(w, full), ("Mf", "Jf", "Mb", "Jb")):
        assert rel(got, ref) <= 1e-5, (name, rel(got, ref))


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_scans(w):
    full = _full(w)
    Mf, Jf, Mb, Jb = _maps_ref(w, full)
    ST = np.zeros((w.B, w.H, w.d, w.d))
    Fr = np.zeros((w.B, w.H, w.C + 1, w.d, w.d))
    Gr = np.zeros_like(Fr)
    for b in range(w.B):
        for h in range(w.H):
            ST[b, h] = oracle.text_state(full["Kx"][b, h], full["Vx"][b, h], full["beta_x"][b, h])
            Fr[b, h], Gr[b, h] = oracle.scan_states(full["K"][b, h], full["V"][b, h], full["beta"][b, h],
                                                    full["alpha"][b, h], ST[b, h], w.chunk, w.anchors)
    s = vdn.shape_for(w)
    d = {k: to_dev(v) for k, v in dict(Mf=Mf, Jf=Jf, Mb=Mb, Jb=Jb, ST=ST).items()}
    F = torch.empty((w.B, w.H, w.C + 1, w.d, w.d), device="cuda")
    G = torch.empty_like(F)
    vdn.vdn_scan_bidir(s, d["Mf"], d["Jf"], d["Mb"], d["Jb"], d["ST"], F, G)
    F2 = torch.empty_like(F)
    G2 = torch.empty_like(F)
    vdn.vdn_scan_fwd(s, d["Mf"], d["Jf"], d["ST"], F2)
    vdn.vdn_scan_bwd(s, d["Mb"], d["Jb"], d["ST"], G2)
    torch.cuda.synchronize()
    assert rel(F, Fr) <= 1e-5 and rel(G, Gr) <= 1e-5, (rel(F, Fr), rel(G, Gr))
    assert torch.equal(F, F2) and torch.equal(G, G2)


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_chunk_readout(w):
    full = _full(w)
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    ref = oracle_heads(w, full, pairs)
    Fr = np.stack([np.stack([ref[(b, h)]["F"] for h in range(w.H)]) for b in range(w.B)])
    Gr = np.stack([np.stack([ref[(b, h)]["G"] for h in range(w.H)]) for b in range(w.B)])
    s = vdn.shape_for(w)
    O = torch.full((w.B, w.H, w.T, w.U, w.d), float("nan"), dtype=tdtype(w), device="cuda")
    vdn.vdn_chunk_readout(s, to_dev(full["Q"], tdtype(w)), to_dev(Fr), to_dev(Gr), O)
    torch.cuda.synchronize()
    assert not torch.isnan(O.float()).any()
    for (b, h), r in ref.items():
        e = rel(O[b, h], r["O"])
        # bf16 output rounding alone is ~2^-9 / sqrt(3) relative
        assert e <= (3e-3 if w.dtype == "bf16" else 1e-5), (b, h, e)


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_text_state(w):
    full = _full(w)
    dev = device_inputs(w, full)
    s = vdn.shape_for(w)
    ST = torch.empty((w.B, w.H, w.d, w.d), device="cuda")
    ws = vdn.workspace(vdn.vdn_text_state_workspace_bytes(s))
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_text_state(s, dev["Kx"], dev["Vx"], dev["beta_x"], ST, ws, info)
    torch.cuda.synchronize()
    for b in range(w.B):
        for h in range(w.H):
            r = oracle.text_state(full["Kx"][b, h], full["Vx"][b, h], full["beta_x"][b, h])
            assert rel(ST[b, h], r) <= 1e-5


# ----------------------------------------------------------- edge cases
@pytest.mark.parametrize("kw", [
    dict(T=0), dict(U=0), dict(n_text=0), dict(B=0), dict(T=1), dict(T=3, U=1),
    dict(T=5, chunk=5), dict(T=11, chunk=1), dict(T=9, chunk=16),
], ids=lambda kw: "-".join(f"{k}{v}" for k, v in kw.items()))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_edge_shapes(kw, dtype):
    d = 128 if dtype == "bf16" else 16
    w = custom("edge", index=44, dtype=dtype, d=d, U=kw.get("U", 33), T=kw.get("T", 7),
               B=kw.get("B", 1), H=2, n_text=kw.get("n_text", 6), chunk=kw.get("chunk", 5))
    full = _full(w)
    s = vdn.shape_for(w)
    dev = device_inputs(w, full)
    fw = vdn.Forward(s)
    fw(dev["Q"], dev["K"], dev["V"], dev["beta"], dev["alpha"], dev["Kx"], dev["Vx"], dev["beta_x"])
    torch.cuda.synchronize()
    assert int(fw.info.item()) == 0
    for b in range(w.B):
        for h in range(w.H):
            inp = {k: full[k][b, h] for k in full}
            r = oracle.vda_head(inp, w.chunk, w.anchors)
            assert rel(fw.F[b, h], r["F"]) <= TOL[dtype] / 10
            assert rel(fw.G[b, h], r["G"]) <= TOL[dtype] / 10
            if w.T * w.U > 0:
                assert rel(fw.O[b, h], r["O"]) <= TOL[dtype]


def test_no_frame_outside_window_reads_text_state():
    # two chunks: every window covers the clip, so O = S^T q exactly as in the oracle pin
    w = custom("two_chunks", index=45, T=10, anchors=0)
    full = _full(w)
    dev = device_inputs(w, full)
    fw = run_forward(w, dev)
    for h in range(w.H):
        ST = oracle.text_state(full["Kx"][0, h], full["Vx"][0, h], 1.0)
        ref = np.einsum("tuk,vk->tuv", full["Q"][0, h].astype(np.float64), ST)
        assert rel(fw.O[0, h], ref) <= 3e-3


@pytest.mark.parametrize("d", [16, 128])
def test_nonpositive_pivot_is_reported_by_invert(d):
    w = custom("poison_inv", index=47, dtype="f32", d=d, T=9, anchors=0)
    full = _full(w)
    Ar, _ = _stats_ref(w, full)
    Ar[0, 1, 4, 2, 2] = -7.0      # (b=0, h=1, t=4): linear index 13
    Ar[0, 1, 7, 5, 5] = np.inf    # (0, 1, 7): 16
    s = vdn.shape_for(w)
    W = torch.empty((w.B, w.H, w.T, w.d, w.d), device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_frame_invert(s, to_dev(Ar), W, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 1 + 13


def test_nonpositive_pivot_is_reported_by_block_invert():
    # bf16, d = 128: the tensor-core blocked sweep takes the four 32 x 32
    # pivot blocks in turn (each as the Schur complement left by the ones
    # before); a poisoned trailing diagonal makes the last block indefinite, a
    # poisoned leading one the first
    w = custom("poison_tc", index=48, T=9, anchors=0)
    full = _full(w)
    Ar, _ = _stats_ref(w, full)
    Ar[0, 1, 2, 100, 100] = -60.0   # (b=0, h=1, t=2): linear index 11, S fails
    Ar[0, 1, 6, 3, 3] = -9.0        # (0, 1, 6): 15, P fails
    s = vdn.shape_for(w)
    W = torch.empty((w.B, w.H, w.T, w.d, w.d), device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_frame_invert(s, to_dev(Ar), W, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 1 + 11
    Ar[0, 1, 2, 100, 100] = 0.0
    vdn.vdn_frame_invert(s, to_dev(Ar), W, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 1 + 15
    # the frames that were not poisoned are still exact
    ref = np.linalg.inv(np.eye(w.d) + Ar[0, 0])
    assert rel(W[0, 0], ref) <= 1e-4


@pytest.mark.parametrize("w", [TC_SMALL, TC_TB], ids=lambda w: w.name)
def test_fused_pass_reports_an_indefinite_frame(w):
    # a negative write gate makes I + A_t indefinite for one frame: the fused
    # tensor-core pass sweeps its leading block (in the Gram kernel's sweep
    # pairs, or the separate Schur step with per-token gates) and then its
    # Schur complement, and reports that frame in *info (frame index + 1)
    full = _full(w)
    b, h, t = w.B - 1, w.H - 1, 4
    full["beta"] = np.array(full["beta"], copy=True)
    full["beta"][b, h, t] = -2.0
    dev = device_inputs(w, full)
    fw = run_forward(w, dev)
    assert int(fw.info.item()) == 1 + (b * w.H + h) * w.T + t
    # the same inputs with the gate restored pass
    full["beta"][b, h, t] = 0.5
    fw = run_forward(w, device_inputs(w, full))
    assert int(fw.info.item()) == 0


def test_nonpositive_pivot_is_reported():
    w = custom("poison", index=46, dtype="f32", d=16, T=9, anchors=0)
    full = _full(w)
    Ar, Br = _stats_ref(w, full)
    Ar[0, 1, 6, 3, 3] = np.nan     # frame (b=0, h=1, t=6): linear index 15
    Ar[0, 1, 8, 0, 0] = -5.0       # (0, 1, 8): 17, non-positive pivot
    s = vdn.shape_for(w)
    M = torch.empty((w.B, w.H, w.T, w.d, w.d), device="cuda")
    J = torch.empty_like(M)
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_frame_factor(s, to_dev(Ar), to_dev(Br), to_dev(full["alpha"]), M, J, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 1 + 15


# ------------------------------------------------------------ full size
FULL = [("h3", [(0, 0), (0, 23)]), ("long", [(0, 5)]), ("batched", [(0, 0), (3, 17)]),
        ("h3_tb", [(0, 7)])]


@pytest.mark.parametrize("name,pairs", FULL, ids=[f[0] for f in FULL])
def test_full_size_sampled_heads(name, pairs):
    w = W[name]
    sampled = {(b, h): synth.generate_head(w, b, h) for b, h in pairs}
    dev = device_fill(w, sampled, seed=w.seed)
    fw = run_forward(w, dev)
    assert int(fw.info.item()) == 0
    assert torch.isfinite(fw.O.float()).all()
    for (b, h), inp in sampled.items():
        r = oracle.vda_head(inp, w.chunk, w.anchors)
        eo, ef, eg = rel(fw.O[b, h], r["O"]), rel(fw.F[b, h], r["F"]), rel(fw.G[b, h], r["G"])
        print(f"{name} b{b} h{h}: O {eo:.2e} F {ef:.2e} G {eg:.2e}")
        assert eo <= TOL["bf16"] and ef <= TOL["bf16"] and eg <= TOL["bf16"]
        assert ef <= state_guard(w) and eg <= state_guard(w) and eo <= OUT_GUARD["bf16"], (ef, eg, eo)
    del dev, fw
    torch.cuda.empty_cache()
