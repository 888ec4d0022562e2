"""Helpers shared by the GPU parity tests: device copies of seeded inputs,
the fp64 oracle run on the same inputs, and the rel-Frobenius check."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from frame_wise_delta_b200 import synth
from frame_wise_delta_b200 import vdn

# Tolerances on rel-Frobenius error per (b, h): float32 inputs 1e-4, bf16
# inputs with a float32 state 2e-2 (the acceptance bounds of this path).
TOL = {"f32": 1e-4, "bf16": 2e-2}
# Regression guards, tighter than those bounds. Both sides read the same
# (bf16-rounded) inputs and both carry the state in (at least) fp32, so the
# boundary states hold only the fp32 arithmetic's error (~1e-5 and below);
# the bf16 output adds its own rounding (2^-9 relative per element). A state
# accuracy regression that the acceptance bound would let through fails these.
STATE_GUARD = 1e-4
OUT_GUARD = {"f32": 1e-4, "bf16": 3e-3}


def state_guard(w) -> float:
    """The state guard of a workload. Near-duplicate keys (cosine 0.99) make
    cond(I + A_t) ~ 1e2-2e2, which magnifies rounding in the per-frame
    inverse: the Schur complement S = R - Q^T P^{-1} Q is much smaller than R
    there, so it is formed in fp32 on the CUDA cores, and an inverse computed
    exactly in fp32 is already off by ~3e-5 relative. The boundary states
    then sit ~1.1e-4 from the oracle (measured on the batched workload; ~3e-3
    when the products forming S took bf16 hi/lo splits on the tensor cores),
    and the guard is 5e-4; the well-conditioned workloads keep 1e-4."""
    return 5e-4 if getattr(w, "near_dup", False) else STATE_GUARD


def tdtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype)


def device_inputs(w: synth.Workload, full: dict) -> dict:
    """Move [B, H, ...] host arrays to the device (Q/K/V/Kx/Vx in the workload dtype)."""
    dt = tdtype(w)
    out = {}
    for k in ("Q", "K", "V", "Kx", "Vx"):
        out[k] = to_dev(full[k], dt)
    for k in ("beta", "alpha", "beta_x"):
        out[k] = to_dev(full[k])
    return out


def oracle_heads(w: synth.Workload, full: dict, pairs) -> dict:
    """Run the oracle on the given (b, h) pairs of host arrays."""
    res = {}
    for b, h in pairs:
        inp = {k: full[k][b, h] for k in full}
        res[(b, h)] = oracle.vda_head(inp, w.chunk, w.anchors)
    return res


def rel(x, ref) -> float:
    if isinstance(x, torch.Tensor):
        x = x.detach().float().cpu().numpy()
    return oracle.rel_frobenius(x, ref)


def run_forward(w: synth.Workload, dev: dict):
    s = vdn.shape_for(w)
    fw = vdn.Forward(s)
    fw(dev["Q"], dev["K"], dev["V"], dev["beta"], dev["alpha"], dev["Kx"], dev["Vx"], dev["beta_x"])
    torch.cuda.synchronize()
    return fw


def device_fill(w: synth.Workload, sampled: dict, seed: int) -> dict:
    """Full-size device inputs: the sampled (b, h) pairs hold the exact seeded
    values from synth; every other pair is filled on the device from a seeded
    torch generator (heads are independent, so only the sampled pairs are
    compared with the oracle)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    dt = tdtype(w)
    B, H, T, U, d = w.B, w.H, w.T, w.U, w.d
    dev = {}
    for k, shp in (("Q", (B, H, T, U, d)), ("K", (B, H, T, U, d)), ("V", (B, H, T, U, d)),
                   ("Kx", (B, H, w.n_text, d)), ("Vx", (B, H, w.n_text, d))):
        t = torch.empty(shp, dtype=dt, device="cuda")
        for b in range(B):
            x = torch.randn(shp[1:], generator=g, device="cuda", dtype=torch.float32)
            if k in ("K", "Kx"):
                x = x / x.norm(dim=-1, keepdim=True)
            t[b].copy_(x.to(dt))
            del x
        dev[k] = t
    tb = w.beta_per_token
    dev["beta"] = torch.rand((B, H, T, U) if tb else (B, H, T), generator=g, device="cuda") * 0.9 + 0.1
    dev["alpha"] = torch.rand((B, H, T, d), generator=g, device="cuda") * (1 - w.alpha_lo) + w.alpha_lo
    dev["beta_x"] = (torch.rand((B, H, w.n_text), generator=g, device="cuda") * 0.9 + 0.1 if tb
                     else torch.ones((B, H), device="cuda"))
    for (b, h), inp in sampled.items():
        for k in ("Q", "K", "V", "Kx", "Vx"):
            dev[k][b, h].copy_(to_dev(inp[k], dt))
        for k in ("beta", "alpha"):
            dev[k][b, h].copy_(to_dev(inp[k]))
        if tb:
            dev["beta_x"][b, h].copy_(to_dev(inp["beta_x"]))
        else:
            dev["beta_x"][b, h] = float(inp["beta_x"])
    return dev
