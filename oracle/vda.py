"""fp64 CPU oracle of the bidirectional frame-wise delta-rule memory (VDA).

TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's
CPU-baseline leg call it; the product path never does. It shares no code
with the CUDA library: it is plain numpy in float64, written from the
definitions of the paper "Video DeltaNet: A Video-Native Hybrid Attention for
Livestream Video Generation" (summary page), section by section:

* "Core method": the frame-level objective
      S_t = argmin_S 1/2 ||S - Sbar_t||_F^2 + sum_u beta_{t,u}/2 ||S k_{t,u} - v_{t,u}||^2
  with Sbar_t = S_{t-1} Diag(alpha_t) (section "Prerequisites / Delta rule"),
  whose closed form is S_t = (Sbar_t + B_t)(I + A_t)^{-1}.
* "Method steps", step (3): A_t = K_t^T Diag(beta_t) K_t,
  B_t = V_t^T Diag(beta_t) K_t; transition M_t = Diag(alpha_t)(I + A_t)^{-1}
  and injection J_t = B_t (I + A_t)^{-1}.
* "Core method" and step (4): a forward and a backward scan, both started
  from half of the text state S^T; each query chunk reads the forward state
  just before its 15-frame window and the backward state just after it, and
  the two readouts are summed.

Readings taken where the page leaves a step open (each is listed with its
reason in the design notes of this repository):
* beta is one scalar per frame (a per-token vector is also accepted here);
* the backward scan applies each frame's own (alpha_t, A_t, B_t) in reverse
  frame order;
* S^T is one VDA update from S = 0 over the text tokens (beta_x, no decay);
* both scans start from S^T / 2;
* chunk c's window is chunks c-1..c+1 (clipped), so its readout state is
  R_c = F[max(c-1, 0)] + G[min(c+2, C)], where F[j] is the forward state
  after chunks 0..j-1 and G[j] the backward state after chunks C-1..j;
* with anchors on, the first and last frames neither write nor read;
* a ragged last chunk holds T mod 5 frames.

The oracle never composes chunk maps for the scan: it steps frame by frame
with a linear solve, so the CUDA path's chunk composition is checked against
the definition rather than against a restatement of itself.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def num_chunks(T: int, chunk: int) -> int:
    """C = ceil(T / chunk); the last chunk may be partial."""
    return -(-T // chunk)


def is_anchor(t: int, T: int, anchors: int) -> bool:
    """First/last frames are softmax anchors that the linear branch drops."""
    return bool(anchors) and (t == 0 or t == T - 1)


def frame_stats(K_t, V_t, beta_t):
    """Frame statistics of "Method steps" step (3).

    K_t: [U, d_k] keys (rows k_{t,u}); V_t: [U, d_v] values; beta_t: a scalar
    write gate for the frame or a [U] vector of per-token gates.
    Returns A_t = K^T Diag(beta) K  [d_k, d_k] and B_t = V^T Diag(beta) K  [d_v, d_k].
    """
    K = _f64(K_t)
    V = _f64(V_t)
    b = _f64(beta_t)
    if b.ndim == 0:
        Kb = K * b
    else:
        Kb = K * b[:, None]
    A = K.T @ Kb
    B = V.T @ Kb
    return A, B


def frame_update(S_prev, alpha_t, A_t, B_t):
    """One frame of VDA ("Core method"): S_t = (S_{t-1} Diag(alpha_t) + B_t)(I + A_t)^{-1}.

    Computed as the solution of S_t (I + A_t) = Sbar_t + B_t, the normal
    equations of the frame objective, with a dense LU solve (no inverse).
    """
    S_prev = _f64(S_prev)
    A_t = _f64(A_t)
    B_t = _f64(B_t)
    d_k = A_t.shape[0]
    S_bar = S_prev * _f64(alpha_t)[None, :]
    G = np.eye(d_k) + A_t
    R = S_bar + B_t
    # S G = R  <=>  G^T S^T = R^T
    return np.linalg.solve(G.T, R.T).T


def text_state(Kx, Vx, beta_x=1.0):
    """Text state S^T (reading of "Core method" / step (4)): one VDA update
    from the zero state over all text tokens, with gate beta_x and no decay."""
    A, B = frame_stats(Kx, Vx, beta_x)
    d_v, d_k = B.shape
    return frame_update(np.zeros((d_v, d_k)), np.ones(d_k), A, B)


def transition(A_t, B_t, alpha_t, anchor: bool = False):
    """Per-frame affine map of step (3): M_t = Diag(alpha_t)(I + A_t)^{-1},
    J_t = B_t (I + A_t)^{-1}, so that S_t = S_{t-1} M_t + J_t.
    Anchor frames are identity maps (M = I, J = 0)."""
    A_t = _f64(A_t)
    B_t = _f64(B_t)
    d_k = A_t.shape[0]
    if anchor:
        return np.eye(d_k), np.zeros_like(B_t)
    W = np.linalg.inv(np.eye(d_k) + A_t)
    return _f64(alpha_t)[:, None] * W, B_t @ W


def scan_states(K, V, beta, alpha, S_T, chunk: int = 5, anchors: int = 0):
    """Forward and backward frame-by-frame scans ("Core method"; step (4)).

    K, V: [T, U, d]; beta: [T] (or [T, U]); alpha: [T, d_k]; S_T: [d_v, d_k].
    Returns F, G of shape [C+1, d_v, d_k]:
      F[0] = S_T / 2 and F[j] = forward state after the frames of chunks 0..j-1;
      G[C] = S_T / 2 and G[j] = backward state after the frames of chunks C-1..j.
    """
    T = K.shape[0]
    C = num_chunks(T, chunk)
    stats = [frame_stats(K[t], V[t], beta[t]) for t in range(T)]
    S_half = 0.5 * _f64(S_T)
    F = np.empty((C + 1,) + S_half.shape)
    G = np.empty((C + 1,) + S_half.shape)

    S = S_half.copy()
    F[0] = S
    for t in range(T):
        if not is_anchor(t, T, anchors):
            S = frame_update(S, alpha[t], *stats[t])
        if (t + 1) % chunk == 0 or t == T - 1:
            F[num_chunks(t + 1, chunk)] = S

    S = S_half.copy()
    G[C] = S
    for t in range(T - 1, -1, -1):
        if not is_anchor(t, T, anchors):
            S = frame_update(S, alpha[t], *stats[t])
        if t % chunk == 0:
            G[t // chunk] = S
    return F, G


def readout_state(F, G, c: int):
    """State read by query chunk c: the forward state just before its window
    (chunks c-1..c+1) plus the backward state just after it."""
    C = F.shape[0] - 1
    return _f64(F[max(c - 1, 0)]) + _f64(G[min(c + 2, C)])


def chunk_readout(Q, F, G, chunk: int = 5, anchors: int = 0):
    """Linear-branch readout o_{t,u} = R_c q_{t,u} for every non-anchor frame
    t of chunk c (anchor rows read nothing). Q: [T, U, d_k] -> O: [T, U, d_v]."""
    Q = _f64(Q)
    T, U, _ = Q.shape
    d_v = F.shape[1]
    O = np.zeros((T, U, d_v))
    for t in range(T):
        if is_anchor(t, T, anchors):
            continue
        R = readout_state(F, G, t // chunk)
        O[t] = Q[t] @ R.T
    return O


def bridge_factors(alpha, t: int, chunk: int = 5, anchors: int = 0):
    """Decay bridge of "Method steps" step (5) for query frame t.

    Reading: the forward state read by chunk c = t // chunk holds the frames
    before its window (chunks c-1..c+1, clipped), i.e. frames < f0 with
    f0 = chunk * max(c - 1, 0); the window's frames write through the softmax
    branch, not the memory, but their decay still acts, so the state is
    carried to frame t through Diag(alpha_r) for r = f0..t. The backward state
    holds the frames after the window, > f1 = min(chunk * (c + 2), T) - 1, and
    is carried down to t through r = f1..t. An anchor frame's transition is
    the identity, so its alpha counts as 1.
    alpha: [T, d_k]. Returns (pf, pb), each [d_k].
    """
    alpha = _f64(alpha)
    T, d_k = alpha.shape
    c = t // chunk
    f0 = chunk * max(c - 1, 0)
    f1 = min(chunk * (c + 2), T) - 1
    pf = np.ones(d_k)
    for r in range(f0, t + 1):
        if not is_anchor(r, T, anchors):
            pf = pf * alpha[r]
    pb = np.ones(d_k)
    for r in range(t, f1 + 1):
        if not is_anchor(r, T, anchors):
            pb = pb * alpha[r]
    return pf, pb


def bridged_readout(Q, F, G, alpha, chunk: int = 5, anchors: int = 0):
    """Linear-branch readout with the decay bridge (step (5)):
    o_{t,u} = R_t q_{t,u} with R_t = F_{max(c-1,0)} Diag(pf_t) + G_{min(c+2,C)} Diag(pb_t)
    (bridge_factors); anchor rows read nothing. With every alpha = 1 this is
    chunk_readout. Q: [T, U, d_k], alpha: [T, d_k] -> O: [T, U, d_v]."""
    Q = _f64(Q)
    T, U, _ = Q.shape
    C = F.shape[0] - 1
    d_v = F.shape[1]
    O = np.zeros((T, U, d_v))
    for t in range(T):
        if is_anchor(t, T, anchors):
            continue
        c = t // chunk
        pf, pb = bridge_factors(alpha, t, chunk, anchors)
        R = _f64(F[max(c - 1, 0)]) * pf[None, :] + _f64(G[min(c + 2, C)]) * pb[None, :]
        O[t] = Q[t] @ R.T
    return O


def gated_rmsnorm(O, weight, gate, eps: float = 1e-6):
    """Readout epilogue of "Method steps" step (5): RMSNorm of every token's
    readout over its d_v channels, then a sigmoid gate, channel by channel:
        y = o / sqrt(mean_i o_i^2 + eps) * weight * sigmoid(gate).
    O, gate: [..., d_v]; weight: [d_v] (one RMSNorm weight vector per head).
    """
    O = _f64(O)
    g = _f64(gate)
    rms = np.sqrt(np.mean(O * O, axis=-1, keepdims=True) + eps)
    return O / rms * _f64(weight) * (1.0 / (1.0 + np.exp(-g)))


def chunk_maps(K, V, beta, alpha, chunk: int = 5, anchors: int = 0):
    """Affine map S -> S M_c + J_c that each chunk's frames apply, per direction.

    Found by running the oracle's own frame update over the chunk's frames:
    J_c is the result from the zero state, M_c the result from the identity
    with the injections switched off (the update is linear in (S, B_t)).
    Returns Mf, Jf, Mb, Jb of shape [C, d, d] (forward and backward order).
    """
    T = K.shape[0]
    d_k = K.shape[2]
    d_v = V.shape[2]
    C = num_chunks(T, chunk)
    Mf = np.empty((C, d_k, d_k))
    Jf = np.empty((C, d_v, d_k))
    Mb = np.empty((C, d_k, d_k))
    Jb = np.empty((C, d_v, d_k))
    for c in range(C):
        frames = list(range(c * chunk, min((c + 1) * chunk, T)))
        for order, Mo, Jo in ((frames, Mf, Jf), (frames[::-1], Mb, Jb)):
            Sm = np.eye(d_k)
            Sj = np.zeros((d_v, d_k))
            for t in order:
                if is_anchor(t, T, anchors):
                    continue
                A, B = frame_stats(K[t], V[t], beta[t])
                Sm = frame_update(Sm, alpha[t], A, np.zeros((d_k, d_k)))
                Sj = frame_update(Sj, alpha[t], A, B)
            Mo[c] = Sm
            Jo[c] = Sj
    return Mf, Jf, Mb, Jb


def vda_head(inp: dict, chunk: int = 5, anchors: int = 0, bridge: bool = False) -> dict:
    """The whole linear branch for one (batch, head) pair.

    inp holds Q, K, V [T, U, d], Kx, Vx [n_text, d], beta [T], alpha [T, d]
    and beta_x; with gate [T, U, d] and norm_w [d] also the gated RMSNorm
    output Y. bridge: read through the decay bridge (bridged_readout).
    Returns S_T, F, G, O (and Y), all float64.
    """
    S_T = text_state(inp["Kx"], inp["Vx"], inp.get("beta_x", 1.0))
    F, G = scan_states(inp["K"], inp["V"], inp["beta"], inp["alpha"], S_T, chunk, anchors)
    if bridge:
        O = bridged_readout(inp["Q"], F, G, inp["alpha"], chunk, anchors)
    else:
        O = chunk_readout(inp["Q"], F, G, chunk, anchors)
    out = {"S_T": S_T, "F": F, "G": G, "O": O}
    if "gate" in inp:  # gated RMSNorm epilogue (step (5))
        out["Y"] = gated_rmsnorm(O, inp["norm_w"], inp["gate"], inp.get("eps", 1e-6))
    return out


def stream_segment(Q, K, V, beta, alpha, S_prev, S_in, chunk: int = 5, anchor_first: bool = False,
                   bridge: bool = False, alpha_prev=None):
    """One segment of a live stream read through the forward memory only.

    Reading of the page's livestream framing ("Future directions": continuous
    generation with streaming systems): the frames after the segment do not
    exist yet, so only the forward scan runs, carried from segment to segment;
    each chunk c reads the forward state before the chunk ahead of it,
    R_c = F_{max(c-1,0)} of the whole stream, with no backward term.
    The segment starts on a chunk boundary; S_prev and S_in are the stream's
    forward states before chunks c0 - 1 and c0 (for the first segment both are
    the text state, counted once by the single scan); anchor_first makes the
    segment's first frame an anchor (the stream's frame 0).

    bridge: read through the decay bridge of "Method steps" step (5), forward
    half (the reading of bridge_factors): frame t of chunk c reads the state
    before its window carried through the decay of the window's frames up to
    t, R_t = F_{c-1} Diag(prod_{r=f0..t} alpha_r) with f0 the first frame of
    chunk c - 1. For the segment's chunk 0 the window starts in the previous
    segment's last chunk, whose decay product alpha_prev ([d_k], see
    stream_bridge_tail; ones, or None, for the stream's first segment) joins
    the product: R_t = S_prev Diag(alpha_prev * prod_{r=0..t} alpha_r). An
    anchor frame's alpha counts as 1.

    Q, K, V: [T, U, d]; beta: [T] (or [T, U]); alpha: [T, d_k].
    Returns O [T, U, d_v] and F [C+1, d_v, d_k] with F[0] = S_in and F[j] the
    state after the segment's chunks 0..j-1 (frame by frame, no chunk maps).
    """
    Q = _f64(Q)
    alpha = _f64(alpha)
    T = K.shape[0]
    C = num_chunks(T, chunk)
    S = _f64(S_in).copy()
    F = np.empty((C + 1,) + S.shape)
    F[0] = S
    for t in range(T):
        if not (anchor_first and t == 0):
            S = frame_update(S, alpha[t], *frame_stats(K[t], V[t], beta[t]))
        if (t + 1) % chunk == 0 or t == T - 1:
            F[num_chunks(t + 1, chunk)] = S
    d_k = S.shape[1]
    O = np.zeros((T,) + Q.shape[1:2] + (S.shape[0],))
    for t in range(T):
        if anchor_first and t == 0:
            continue
        c = t // chunk
        R = _f64(S_prev) if c == 0 else F[c - 1]
        if bridge:
            p = np.ones(d_k) if (c > 0 or alpha_prev is None) else _f64(alpha_prev).copy()
            for r in range(chunk * max(c - 1, 0), t + 1):
                if not (anchor_first and r == 0):
                    p = p * alpha[r]
            R = R * p[None, :]
        O[t] = Q[t] @ R.T
    return O, F


def stream_bridge_tail(alpha, chunk: int = 5, anchor_first: bool = False):
    """Decay product over a segment's last chunk (the frames a next segment's
    first chunk finds at the start of its window): prod alpha_r over
    r = chunk * (C - 1) .. T - 1, an anchor frame counting as 1. [d_k]."""
    alpha = _f64(alpha)
    T, d_k = alpha.shape
    p = np.ones(d_k)
    for r in range(chunk * (num_chunks(T, chunk) - 1), T):
        if not (anchor_first and r == 0):
            p = p * alpha[r]
    return p


def rel_frobenius(x, ref) -> float:
    """||x - ref||_F / ||ref||_F (0 when both are zero)."""
    x = _f64(x)
    ref = _f64(ref)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    if den == 0.0:
        # a zero reference: equal arrays agree exactly, any other differs
        # without bound (tested element by element, so a tiny difference whose
        # square underflows still counts)
        return 0.0 if not np.any(x != ref) else math.inf
    return float(num / den)
