"""Pins of the decay-bridge readout of the oracle (bridge_factors,
bridged_readout).

The reading (listed with the others in the design notes): the forward state
a query chunk reads stops at its window's first frame f0, the backward state
at its window's last frame f1; the window frames write through the softmax
branch, not the memory, but their channel decay still acts, so each state is
carried to the query frame t through Diag(alpha_r), forward over r = f0..t
and backward over r = f1..t; anchor frames (identity transitions) do not
decay. These tests tie the oracle to facts outside its own formula: the
method's frame recurrence run with the window's writes switched off, the
closed form for a constant decay, unit decay reducing to the plain readout,
and anchors not decaying.
"""
import numpy as np
import pytest

import oracle


def _clip(rng, T, U, d):
    K = rng.standard_normal((T, U, d))
    K /= np.linalg.norm(K, axis=-1, keepdims=True)
    V = rng.standard_normal((T, U, d))
    Q = rng.standard_normal((T, U, d))
    beta = rng.uniform(0.1, 1.0, T)
    alpha = rng.uniform(0.6, 1.0, (T, d))
    return Q, K, V, beta, alpha


def test_unit_decay_is_the_plain_readout():
    rng = np.random.default_rng(21)
    T, U, d = 13, 6, 5
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S_T = rng.standard_normal((d, d))
    F, G = oracle.scan_states(K, V, beta, alpha, S_T, 5, 1)
    ones = np.ones_like(alpha)
    np.testing.assert_array_equal(oracle.bridged_readout(Q, F, G, ones, 5, 1), oracle.chunk_readout(Q, F, G, 5, 1))


@pytest.mark.parametrize("anchors", [0, 1])
def test_bridge_is_the_recurrence_with_the_window_writes_off(anchors):
    # For each query frame t: switch off the write gates of every frame of
    # t's window, run the frame recurrence of "Core method" (frame_update)
    # frame by frame in both directions, and compare the states it reaches at
    # t with the two halves of the bridged readout (read with unit queries).
    rng = np.random.default_rng(22 + anchors)
    T, U, d, chunk = 17, 4, 5, 5
    _, K, V, beta, alpha = _clip(rng, T, U, d)
    S_T = rng.standard_normal((d, d))
    eye_q = np.broadcast_to(np.eye(d), (T, d, d)).copy()  # query rows e_k: O_t = R_t
    for t in range(T):
        if oracle.is_anchor(t, T, anchors):
            continue
        c = t // chunk
        lo, hi = chunk * max(c - 1, 0), min(chunk * (c + 2), T) - 1
        b = beta.copy()
        b[lo:hi + 1] = 0.0
        F, G = oracle.scan_states(K, V, b, alpha, S_T, chunk, anchors)
        # forward: from S_T / 2 through frames 0..t
        S = 0.5 * S_T
        for r in range(t + 1):
            if not oracle.is_anchor(r, T, anchors):
                S = oracle.frame_update(S, alpha[r], *oracle.frame_stats(K[r], V[r], b[r]))
        Of = oracle.bridged_readout(eye_q, F, np.zeros_like(G), alpha, chunk, anchors)
        np.testing.assert_allclose(Of[t], S.T, rtol=1e-11, atol=1e-12)
        # backward: from S_T / 2 through frames T-1..t
        S = 0.5 * S_T
        for r in range(T - 1, t - 1, -1):
            if not oracle.is_anchor(r, T, anchors):
                S = oracle.frame_update(S, alpha[r], *oracle.frame_stats(K[r], V[r], b[r]))
        Ob = oracle.bridged_readout(eye_q, np.zeros_like(F), G, alpha, chunk, anchors)
        np.testing.assert_allclose(Ob[t], S.T, rtol=1e-11, atol=1e-12)


def test_constant_decay_closed_form():
    # alpha_r = a for every frame: the factors are powers of a
    rng = np.random.default_rng(23)
    T, d, chunk = 23, 6, 5
    a = rng.uniform(0.5, 1.0, d)
    alpha = np.broadcast_to(a, (T, d)).copy()
    for t in range(T):
        c = t // chunk
        n_f = t - chunk * max(c - 1, 0) + 1
        n_b = min(chunk * (c + 2), T) - t
        pf, pb = oracle.bridge_factors(alpha, t, chunk, 0)
        np.testing.assert_allclose(pf, a ** n_f, rtol=1e-13)
        np.testing.assert_allclose(pb, a ** n_b, rtol=1e-13)


def test_anchor_frames_do_not_decay():
    rng = np.random.default_rng(24)
    T, U, d = 12, 4, 5
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    S_T = rng.standard_normal((d, d))
    F, G = oracle.scan_states(K, V, beta, alpha, S_T, 5, 1)
    a2 = alpha.copy()
    a2[0] = 0.1
    a2[T - 1] = 0.2
    np.testing.assert_array_equal(oracle.bridged_readout(Q, F, G, alpha, 5, 1), oracle.bridged_readout(Q, F, G, a2, 5, 1))
    # without anchors the same change moves the readout
    assert not np.allclose(oracle.bridged_readout(Q, F, G, alpha, 5, 0), oracle.bridged_readout(Q, F, G, a2, 5, 0))


def test_vda_head_bridge_flag():
    rng = np.random.default_rng(25)
    T, U, d = 11, 5, 4
    Q, K, V, beta, alpha = _clip(rng, T, U, d)
    inp = dict(Q=Q, K=K, V=V, beta=beta, alpha=alpha, Kx=rng.standard_normal((6, d)), Vx=rng.standard_normal((6, d)),
               beta_x=1.0)
    r = oracle.vda_head(inp, 5, 1, bridge=True)
    np.testing.assert_array_equal(r["O"], oracle.bridged_readout(Q, r["F"], r["G"], alpha, 5, 1))
