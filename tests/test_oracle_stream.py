"""Pins of the streaming (forward-only) oracle, oracle.stream_segment.

The reading (documented with the others in the design notes): a live stream
runs only the forward scan, carried from segment to segment, and chunk c
reads the forward state before the chunk ahead of it, R_c = F_{max(c-1,0)}.
These tests tie it to facts that do not come from the function itself: a
brute-force frame loop with explicit indices, the affine structure of the
scan (the state enters linearly), causality, and the invariance of the
result under cutting the stream into segments.
"""
import numpy as np
import pytest

import oracle


def _clip(rng, T, U, d, anchors_alpha=(0.9, 1.0)):
    K = rng.standard_normal((T, U, d))
    K /= np.linalg.norm(K, axis=-1, keepdims=True)
    V = rng.standard_normal((T, U, d))
    Q = rng.standard_normal((T, U, d))
    beta = rng.uniform(0.1, 1.0, T)
    alpha = rng.uniform(*anchors_alpha, (T, d))
    return Q, K, V, beta, alpha


def _update(S, Kt, Vt, bt, at):
    """The frame solve written out as the normal equations of the objective:
    S (I + A) = S Diag(alpha) + B, solved for S (no explicit inverse)."""
    A = bt * Kt.T @ Kt
    B = bt * Vt.T @ Kt
    rhs = S * at[None, :] + B
    return np.linalg.solve((np.eye(A.shape[0]) + A).T, rhs.T).T


@pytest.mark.parametrize("anchor_first", [False, True])
def test_brute_force_indices(anchor_first):
    # chunk = 1: every frame is its own chunk, so frame t reads the state
    # after frames 0..t-2 (S_prev for t = 0, S_in for t = 1)
    rng = np.random.default_rng(3)
    T, U, d = 6, 4, 5
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S_prev = rng.standard_normal((d, d))
    S_in = rng.standard_normal((d, d))
    O, F = oracle.stream_segment(Q, K, V, beta, alpha, S_prev, S_in, chunk=1, anchor_first=anchor_first)
    states = [S_in]
    for t in range(T):
        S = states[-1] if (anchor_first and t == 0) else _update(states[-1], K[t], V[t], beta[t], alpha[t])
        states.append(S)
    for t in range(T):
        want = np.zeros((U, d)) if (anchor_first and t == 0) else Q[t] @ (S_prev if t == 0 else states[t - 1]).T
        np.testing.assert_allclose(O[t], want, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(F, np.stack(states), rtol=1e-11, atol=1e-12)


def test_state_enters_affinely():
    # the scan is affine in its initial state: F(S) = F(0) + (F(2S) - F(0)) / 2
    rng = np.random.default_rng(5)
    T, U, d = 13, 6, 4
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S = rng.standard_normal((d, d))
    Z = np.zeros((d, d))
    _, F0 = oracle.stream_segment(Q, K, V, beta, alpha, Z, Z, chunk=5)
    _, F1 = oracle.stream_segment(Q, K, V, beta, alpha, S, S, chunk=5)
    _, F2 = oracle.stream_segment(Q, K, V, beta, alpha, 2 * S, 2 * S, chunk=5)
    np.testing.assert_allclose(F1, F0 + (F2 - F0) / 2, rtol=1e-10, atol=1e-12)


def test_forward_states_match_the_bidirectional_scan():
    # started from S^T / 2 over the whole clip without anchors, the stream's
    # states are the forward states of the bidirectional scan
    rng = np.random.default_rng(8)
    T, U, d = 12, 5, 4
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S_T = rng.standard_normal((d, d))
    F_bi, _ = oracle.scan_states(K, V, beta, alpha, S_T, chunk=5, anchors=0)
    half = 0.5 * S_T
    _, F = oracle.stream_segment(Q, K, V, beta, alpha, half, half, chunk=5)
    np.testing.assert_allclose(F, F_bi, rtol=1e-12, atol=1e-13)


def test_causal():
    # chunk c must not depend on frames in chunks c - 1 or later
    rng = np.random.default_rng(9)
    T, U, d, chunk = 20, 4, 4, 5
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S = rng.standard_normal((d, d))
    O, _ = oracle.stream_segment(Q, K, V, beta, alpha, S, S, chunk=chunk)
    K2, V2 = K.copy(), V.copy()
    K2[5:] = rng.standard_normal(K2[5:].shape)
    V2[5:] = rng.standard_normal(V2[5:].shape)
    O2, _ = oracle.stream_segment(Q, K2, V2, beta, alpha, S, S, chunk=chunk)
    # chunks 0..2 read S_prev, F_0 = S_in and F_1 (frames 0..4): unchanged;
    # chunk 3 reads F_2, which takes in frames 5..9
    np.testing.assert_array_equal(O[:15], O2[:15])
    assert np.abs(O[15:] - O2[15:]).max() > 1e-3


@pytest.mark.parametrize("cut", [5, 10, 15])
def test_segments_compose(cut):
    # cutting the stream at a chunk boundary and carrying (F[C-1], F[C])
    # gives the same outputs and states as one segment
    rng = np.random.default_rng(11 + cut)
    T, U, d = 22, 4, 5
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S_T = rng.standard_normal((d, d))
    O, F = oracle.stream_segment(Q, K, V, beta, alpha, S_T, S_T, chunk=5, anchor_first=True)
    O1, F1 = oracle.stream_segment(Q[:cut], K[:cut], V[:cut], beta[:cut], alpha[:cut], S_T, S_T, chunk=5,
                                   anchor_first=True)
    C1 = F1.shape[0] - 1
    O2, F2 = oracle.stream_segment(Q[cut:], K[cut:], V[cut:], beta[cut:], alpha[cut:], F1[C1 - 1], F1[C1],
                                   chunk=5)
    np.testing.assert_array_equal(np.concatenate([O1, O2]), O)
    np.testing.assert_array_equal(np.concatenate([F1, F2[1:]]), F)


# ----------------------------------------------------------- decay bridge
def _decay_only(S, alphas):
    """Carry a state through frames whose write gates are zero: the frame
    solve itself with beta = 0 (no bridge formula involved)."""
    d = S.shape[1]
    for a in alphas:
        S = _update(S, np.zeros((1, d)), np.zeros((1, S.shape[0])), 0.0, a)
    return S


def test_bridged_stream_is_the_decay_only_recurrence():
    # frame t of chunk c reads the state before its window carried through
    # frames f0..t by the recurrence with the window's writes switched off
    rng = np.random.default_rng(21)
    T, U, d, chunk = 17, 3, 4, 5
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S_prev = rng.standard_normal((d, d))
    S_in = rng.standard_normal((d, d))
    a_prev = rng.uniform(0.8, 1.0, d)
    O, F = oracle.stream_segment(Q, K, V, beta, alpha, S_prev, S_in, chunk=chunk, bridge=True, alpha_prev=a_prev)
    for t in range(T):
        c = t // chunk
        if c == 0:
            # the previous segment's last chunk decays S_prev first (one
            # frame whose alpha is that chunk's product), then frames 0..t
            R = _decay_only(S_prev, [a_prev] + [alpha[r] for r in range(0, t + 1)])
        else:
            R = _decay_only(F[c - 1], [alpha[r] for r in range(chunk * (c - 1), t + 1)])
        np.testing.assert_allclose(O[t], Q[t] @ R.T, rtol=1e-11, atol=1e-12)


def test_bridged_stream_without_decay_is_the_plain_stream():
    rng = np.random.default_rng(22)
    T, U, d = 12, 3, 4
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S = rng.standard_normal((d, d))
    ones = np.ones_like(alpha)
    O1, F1 = oracle.stream_segment(Q, K, V, beta, ones, S, S, chunk=5, anchor_first=True, bridge=True,
                                   alpha_prev=np.ones(d))
    O0, F0 = oracle.stream_segment(Q, K, V, beta, ones, S, S, chunk=5, anchor_first=True)
    np.testing.assert_array_equal(O1, O0)
    np.testing.assert_array_equal(F1, F0)


def test_bridge_tail_of_a_segment():
    rng = np.random.default_rng(23)
    alpha = rng.uniform(0.5, 1.0, (12, 3))
    # last chunk of 12 frames in chunks of 5: frames 10, 11
    np.testing.assert_array_equal(oracle.stream_bridge_tail(alpha, 5), alpha[10] * alpha[11])
    # one chunk holding the stream's anchor frame 0: frames 1..4 only
    np.testing.assert_allclose(oracle.stream_bridge_tail(alpha[:5], 5, anchor_first=True),
                               alpha[1] * alpha[2] * alpha[3] * alpha[4], rtol=0, atol=0)


@pytest.mark.parametrize("cuts", [(5,), (10,), (5, 15), (5, 10, 15, 20)])
def test_bridged_segments_compose(cuts):
    # cutting a bridged stream at chunk boundaries and carrying
    # (F[C-1], F[C], the last chunk's decay product) changes nothing
    rng = np.random.default_rng(31 + len(cuts))
    T, U, d = 23, 3, 4
    Q, K, V, beta, alpha = _clip(rng, T, U, d, (0.7, 1.0))
    S_T = rng.standard_normal((d, d))
    O, F = oracle.stream_segment(Q, K, V, beta, alpha, S_T, S_T, chunk=5, anchor_first=True, bridge=True)
    bounds = [0, *cuts, T]
    Sp, Si, ap = S_T, S_T, np.ones(d)
    Os, Fs = [], [F[:1]]
    for a, b in zip(bounds[:-1], bounds[1:]):
        o, f = oracle.stream_segment(Q[a:b], K[a:b], V[a:b], beta[a:b], alpha[a:b], Sp, Si, chunk=5,
                                     anchor_first=a == 0, bridge=True, alpha_prev=ap)
        Os.append(o)
        Fs.append(f[1:])
        C = f.shape[0] - 1
        Sp, Si, ap = f[C - 1], f[C], oracle.stream_bridge_tail(alpha[a:b], 5, anchor_first=a == 0)
    np.testing.assert_allclose(np.concatenate(Os), O, rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(np.concatenate(Fs), F)
