"""Seeded synthetic inputs for the frame-wise delta-rule memory (VDA).

This module only draws random inputs. It holds none of the method's
arithmetic, so both the CUDA path and the fp64 oracle can use it without
sharing any of the computation they are compared on.

Every tensor of one (b, h) pair is drawn from its own numpy PCG64 stream,
keyed by (seed, b, h, tensor id). Any single head can therefore be
regenerated exactly without drawing the others, which is how the tests
compare sampled heads of the large workloads.

Workload shapes follow the paper "Video DeltaNet: A Video-Native Hybrid
Attention for Livestream Video Generation" (section "VAE latent frames and
temporal chunks": a 102-frame 48x84 latent, 5-frame chunks, 15-frame
windows; section "Method steps", step (2): L2-normalised keys, a write gate
beta and a channel-wise decay alpha).
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

BASE_SEED = 20260917

# tensor ids used to key the per-(b, h) random streams
_TID = {"Q": 0, "K": 1, "V": 2, "Kx": 3, "Vx": 4, "beta": 5, "alpha": 6, "proto": 7, "beta_x": 8}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic VDA workload.

    B, H: batch and heads. T: latent frames. U: spatial tokens per frame.
    d: key and value width (d_k = d_v = d). n_text: text tokens.
    dtype: "f32" or "bf16" storage of Q/K/V and the text keys/values.
    alpha_lo: decay drawn from U(alpha_lo, 1) per channel and frame.
    anchors: 1 when the first and last frames are softmax anchors that the
    linear branch skips.
    near_dup: keys of a frame cluster around a few prototypes (cosine 0.99).
    beta_per_token: one write gate per token, beta [T, U] and beta_x
    [n_text] ~ U(beta_lo, 1); otherwise beta [T] per frame and beta_x = 1.
    decay_bridge: the readout goes through the decay bridge (changes no
    input; carried so that a workload names the whole computation).
    """

    name: str
    index: int
    B: int
    H: int
    T: int
    U: int
    d: int
    n_text: int
    dtype: str
    alpha_lo: float
    anchors: int
    near_dup: bool = False
    chunk: int = 5
    beta_lo: float = 0.1
    beta_per_token: bool = False
    decay_bridge: bool = False

    @property
    def seed(self) -> int:
        return BASE_SEED + self.index

    @property
    def C(self) -> int:
        return -(-self.T // self.chunk)

    @property
    def frames(self) -> int:
        return self.B * self.T

    @property
    def tokens(self) -> int:
        return self.B * self.T * self.U


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 0, B=1, H=1, T=10, U=16, d=16, n_text=8, dtype="f32",
                 alpha_lo=0.9, anchors=0),
        Workload("small", 1, B=1, H=4, T=20, U=256, d=64, n_text=64, dtype="f32",
                 alpha_lo=0.9, anchors=1),
        Workload("h3", 2, B=1, H=24, T=102, U=1008, d=128, n_text=512, dtype="bf16",
                 alpha_lo=0.95, anchors=1),
        Workload("long", 3, B=1, H=24, T=400, U=1008, d=128, n_text=512, dtype="bf16",
                 alpha_lo=0.95, anchors=1),
        Workload("batched", 4, B=4, H=24, T=102, U=1920, d=128, n_text=256, dtype="bf16",
                 alpha_lo=0.95, anchors=1, near_dup=True),
        # per-token write gates beta_{t,u} ("Core method" objective)
        Workload("small_tb", 5, B=1, H=4, T=20, U=256, d=64, n_text=64, dtype="f32",
                 alpha_lo=0.9, anchors=1, beta_per_token=True),
        Workload("h3_tb", 6, B=1, H=24, T=102, U=1008, d=128, n_text=512, dtype="bf16",
                 alpha_lo=0.95, anchors=1, beta_per_token=True),
    ]
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _rng(w: Workload, b: int, h: int, tensor: str) -> np.random.Generator:
    return np.random.default_rng([w.seed, b, h, _TID[tensor]])


def _unit_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-30)).astype(np.float32)


def _store(w: Workload, x: np.ndarray) -> np.ndarray:
    return round_bf16(x) if w.dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def _keys(w: Workload, b: int, h: int, rows: tuple) -> np.ndarray:
    g = _rng(w, b, h, "K").standard_normal(rows + (w.d,), dtype=np.float32)
    if not w.near_dup:
        return _unit_rows(g)
    # Near-duplicate keys: per frame, P unit prototypes; each key is a prototype
    # plus isotropic noise of scale sigma, renormalised, so that its expected
    # cosine to the prototype is 0.99.
    P = 8
    pr = _rng(w, b, h, "proto")
    protos = _unit_rows(pr.standard_normal((rows[0], P, w.d), dtype=np.float32))
    pick = pr.integers(0, P, size=rows)
    sigma = np.float32(np.sqrt((1.0 / 0.99 ** 2 - 1.0) / w.d))
    base = np.take_along_axis(protos, pick[..., None], axis=1)
    return _unit_rows(base + sigma * g)


ALL_PARTS = ("Q", "K", "V", "Kx", "Vx", "beta", "alpha", "beta_x")


def generate_head(w: Workload, b: int, h: int, parts=ALL_PARTS) -> dict:
    """Inputs of one (b, h) pair as float32 numpy arrays.

    Q, K, V: [T, U, d]; Kx, Vx: [n_text, d]; beta: [T]; alpha: [T, d];
    beta_x: float. For bf16 workloads Q/K/V/Kx/Vx hold bf16-representable
    values (rounded to nearest even), which both sides read. `parts` selects
    a subset; every tensor has its own stream, so a subset is drawn exactly as
    it is in the full set.
    """
    T, U, d = w.T, w.U, w.d
    make = {
        "Q": lambda: _store(w, _rng(w, b, h, "Q").standard_normal((T, U, d), dtype=np.float32)),
        "K": lambda: _store(w, _keys(w, b, h, (T, U))),
        "V": lambda: _store(w, _rng(w, b, h, "V").standard_normal((T, U, d), dtype=np.float32)),
        "Kx": lambda: _store(w, _unit_rows(_rng(w, b, h, "Kx").standard_normal((w.n_text, d), dtype=np.float32))),
        "Vx": lambda: _store(w, _rng(w, b, h, "Vx").standard_normal((w.n_text, d), dtype=np.float32)),
        "beta": lambda: _rng(w, b, h, "beta").uniform(
            w.beta_lo, 1.0, size=(T, U) if w.beta_per_token else T).astype(np.float32),
        "alpha": lambda: _rng(w, b, h, "alpha").uniform(w.alpha_lo, 1.0, size=(T, d)).astype(np.float32),
        # per-token gates also gate the text tokens; otherwise beta_x = 1
        "beta_x": lambda: (_rng(w, b, h, "beta_x").uniform(w.beta_lo, 1.0, size=w.n_text).astype(np.float32)
                           if w.beta_per_token else np.float32(1.0)),
    }
    return {k: make[k]() for k in parts}


def generate_pairs(w: Workload, pairs, threads: int = 8) -> dict:
    """Inputs of the given (b, h) pairs stacked as [1, len(pairs), ...] float32
    arrays: a contiguous share of the pairs laid out as one batch of that many
    heads, each pair drawn exactly as in the full set."""
    n = len(pairs)
    out = {
        "Q": np.empty((1, n, w.T, w.U, w.d), np.float32),
        "K": np.empty((1, n, w.T, w.U, w.d), np.float32),
        "V": np.empty((1, n, w.T, w.U, w.d), np.float32),
        "Kx": np.empty((1, n, w.n_text, w.d), np.float32),
        "Vx": np.empty((1, n, w.n_text, w.d), np.float32),
        "beta": np.empty((1, n, w.T, w.U) if w.beta_per_token else (1, n, w.T), np.float32),
        "alpha": np.empty((1, n, w.T, w.d), np.float32),
        "beta_x": np.empty((1, n, w.n_text) if w.beta_per_token else (1, n), np.float32),
    }

    def fill(i):
        b, h = pairs[i]
        for k, v in generate_head(w, b, h).items():
            out[k][0, i] = v

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, range(n)))
    return out


def generate_all(w: Workload, threads: int = 8) -> dict:
    """Full [B, H, ...] float32 arrays for every input of a workload."""
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    flat = generate_pairs(w, pairs, threads)
    return {k: v.reshape((w.B, w.H) + v.shape[2:]) for k, v in flat.items()}
