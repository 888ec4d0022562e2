"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to a closed form, an invariant, a brute
force solve or a printed formula of the paper "Video DeltaNet: A Video-Native
Hybrid Attention for Livestream Video Generation" (summary page), chosen so
that a dropped term, a wrong sign, a transposed operand or an off-by-one
window index fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from frame_wise_delta_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _frame(rng, U, dk, dv, near_dup=False):
    K = _unit(rng.standard_normal((U, dk)))
    if near_dup:
        K = _unit(K[:1] + 0.0126 * rng.standard_normal((U, dk)))
    V = rng.standard_normal((U, dv))
    return K, V


# --- (a) U = 1 reduces to the per-token delta rule (Sherman-Morrison) -------
# "Prerequisites / Delta rule": S_t = Sbar_t + beta (v - Sbar_t k) k^T; the
# joint frame solve with a single token takes the step beta / (1 + beta |k|^2).
@pytest.mark.parametrize("seed", range(4))
def test_single_token_is_delta_rule(seed):
    rng = _rng(seed)
    dk, dv = 7, 5
    S_prev = rng.standard_normal((dv, dk))
    alpha = rng.uniform(0.5, 1.0, dk)
    k = rng.standard_normal(dk) * rng.uniform(0.3, 2.0)  # not unit on purpose
    v = rng.standard_normal(dv)
    beta = rng.uniform(0.1, 3.0)
    A, B = oracle.frame_stats(k[None, :], v[None, :], beta)
    S = oracle.frame_update(S_prev, alpha, A, B)
    S_bar = S_prev * alpha[None, :]
    step = beta / (1.0 + beta * k @ k)
    expect = S_bar + step * np.outer(v - S_bar @ k, k)
    np.testing.assert_allclose(S, expect, rtol=1e-12, atol=1e-12)


# --- (b) first-order optimality of the frame objective ("Core method") ------
@pytest.mark.parametrize("near_dup", [False, True])
def test_gradient_vanishes(near_dup):
    rng = _rng(11)
    dk = dv = 16
    U = 40
    K, V = _frame(rng, U, dk, dv, near_dup)
    beta = 0.7
    S_prev = rng.standard_normal((dv, dk))
    alpha = rng.uniform(0.9, 1.0, dk)
    A, B = oracle.frame_stats(K, V, beta)
    S = oracle.frame_update(S_prev, alpha, A, B)
    S_bar = S_prev * alpha[None, :]
    # gradient written token by token from the objective, not from A and B
    grad = S - S_bar
    for u in range(U):
        grad += beta * np.outer(S @ K[u] - V[u], K[u])
    assert np.linalg.norm(grad) <= 1e-12 * np.linalg.norm(S_bar + B)


# --- (d) brute force: the frame objective as one stacked least squares ------
def _brute_frame(S_bar, K, V, beta):
    """argmin_S 1/2||S - S_bar||^2 + sum_u beta_u/2 ||S k_u - v_u||^2 by lstsq
    on vec(S) (column-major), with S k = (k^T kron I) vec(S)."""
    dv, dk = S_bar.shape
    beta = np.broadcast_to(np.asarray(beta, float), (K.shape[0],))
    rows = [np.eye(dv * dk)]
    rhs = [S_bar.reshape(-1, order="F")]
    for u in range(K.shape[0]):
        w = np.sqrt(beta[u])
        rows.append(w * np.kron(K[u][None, :], np.eye(dv)))
        rhs.append(w * V[u])
    x, *_ = np.linalg.lstsq(np.vstack(rows), np.concatenate(rhs), rcond=None)
    return x.reshape(dv, dk, order="F")


@pytest.mark.parametrize("dk,dv,U", [(3, 2, 1), (4, 4, 6), (6, 3, 9), (5, 5, 2)])
def test_frame_update_matches_brute_force(dk, dv, U):
    rng = _rng(100 + dk * 10 + U)
    K = rng.standard_normal((U, dk))
    V = rng.standard_normal((U, dv))
    S_prev = rng.standard_normal((dv, dk))
    alpha = rng.uniform(0.5, 1.0, dk)
    beta = rng.uniform(0.1, 2.0)
    A, B = oracle.frame_stats(K, V, beta)
    S = oracle.frame_update(S_prev, alpha, A, B)
    ref = _brute_frame(S_prev * alpha[None, :], K, V, beta)
    np.testing.assert_allclose(S, ref, rtol=1e-10, atol=1e-10)


def test_per_token_gate_matches_brute_force():
    rng = _rng(5)
    U, dk, dv = 7, 4, 3
    K = rng.standard_normal((U, dk))
    V = rng.standard_normal((U, dv))
    beta = rng.uniform(0.0, 2.0, U)
    A, B = oracle.frame_stats(K, V, beta)
    S = oracle.frame_update(np.zeros((dv, dk)), np.ones(dk), A, B)
    np.testing.assert_allclose(S, _brute_frame(np.zeros((dv, dk)), K, V, beta), rtol=1e-10, atol=1e-10)


def test_text_state_matches_brute_force():
    rng = _rng(6)
    n, d = 9, 4
    Kx = _unit(rng.standard_normal((n, d)))
    Vx = rng.standard_normal((n, d))
    S_T = oracle.text_state(Kx, Vx, 0.8)
    np.testing.assert_allclose(S_T, _brute_frame(np.zeros((d, d)), Kx, Vx, 0.8), rtol=1e-10, atol=1e-10)


# --- (c) Proposition 1: the transition is non-expansive ---------------------
@pytest.mark.parametrize("near_dup", [False, True])
def test_transition_non_expansive(near_dup):
    rng = _rng(21)
    d = 32
    for _ in range(5):
        K, V = _frame(rng, 64, d, d, near_dup)
        beta = rng.uniform(0.1, 1.0)
        alpha = rng.uniform(0.9, 1.0, d)
        A, B = oracle.frame_stats(K, V, beta)
        M, J = oracle.transition(A, B, alpha)
        W = np.linalg.inv(np.eye(d) + A)
        assert np.linalg.norm(W, 2) <= 1.0 + 1e-12
        assert np.linalg.norm(M, 2) <= 1.0 + 1e-12
        # and the map it defines agrees with the solve
        S0 = rng.standard_normal((d, d))
        np.testing.assert_allclose(S0 @ M + J, oracle.frame_update(S0, alpha, A, B), rtol=1e-9, atol=1e-9)


# --- Appendix A.2: correlation awareness (golden values from the page) ------
def test_a2_saturation_golden():
    with open(os.path.join(GOLDEN, "a2_saturation.json")) as f:
        g = json.load(f)
    rng = _rng(31)
    d = 8
    for case in g["repeated_key"]:
        U, beta = case["U"], case["beta"]
        k = _unit(rng.standard_normal(d))
        v = rng.standard_normal(d)
        A, B = oracle.frame_stats(np.tile(k, (U, 1)), np.tile(v, (U, 1)), beta)
        S = oracle.frame_update(np.zeros((d, d)), np.ones(d), A, B)
        np.testing.assert_allclose(S @ k, case["weight"] * v, rtol=1e-12, atol=1e-12)
    for case in g["orthogonal_keys"]:
        beta = case["beta"]
        Kq, _ = np.linalg.qr(rng.standard_normal((d, d)))
        K = Kq.T[:5]  # 5 orthonormal keys
        V = rng.standard_normal((5, d))
        A, B = oracle.frame_stats(K, V, beta)
        S = oracle.frame_update(np.zeros((d, d)), np.ones(d), A, B)
        for u in range(5):
            np.testing.assert_allclose(S @ K[u], case["weight"] * V[u], rtol=1e-12, atol=1e-12)


# --- limits -----------------------------------------------------------------
def test_zero_gate_keeps_decayed_state():
    rng = _rng(41)
    S_prev = rng.standard_normal((5, 6))
    alpha = rng.uniform(0.1, 1.0, 6)
    K, V = _frame(rng, 10, 6, 5)
    A, B = oracle.frame_stats(K, V, 0.0)
    S = oracle.frame_update(S_prev, alpha, A, B)
    # decay scales the key channels (columns) of S
    np.testing.assert_array_equal(S, S_prev * alpha[None, :])


def test_large_gate_tends_to_least_squares():
    rng = _rng(42)
    U, dk, dv = 50, 8, 6
    K = rng.standard_normal((U, dk))
    V = rng.standard_normal((U, dv))
    A, B = oracle.frame_stats(K, V, 1e8)
    S = oracle.frame_update(rng.standard_normal((dv, dk)), np.ones(dk), A, B)
    X, *_ = np.linalg.lstsq(K, V, rcond=None)  # K X ~ V  ->  S = X^T
    np.testing.assert_allclose(S, X.T, rtol=1e-5, atol=1e-5)


# --- scans -------------------------------------------------------------------
def _small_inputs(seed, T=20, U=12, d=6, n_text=5, anchors=1):
    w = synth.Workload("pin", 90 + seed, B=1, H=1, T=T, U=U, d=d, n_text=n_text,
                       dtype="f32", alpha_lo=0.8, anchors=anchors)
    return w, synth.generate_head(w, 0, 0)


@pytest.mark.parametrize("anchors", [0, 1])
def test_time_reversal_swaps_scans(anchors):
    w, inp = _small_inputs(3, T=20, anchors=anchors)
    S_T = oracle.text_state(inp["Kx"], inp["Vx"])
    F, G = oracle.scan_states(inp["K"], inp["V"], inp["beta"], inp["alpha"], S_T, 5, anchors)
    Fr, Gr = oracle.scan_states(inp["K"][::-1], inp["V"][::-1], inp["beta"][::-1], inp["alpha"][::-1], S_T, 5, anchors)
    C = F.shape[0] - 1
    for j in range(C + 1):
        np.testing.assert_allclose(G[j], Fr[C - j], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(F[j], Gr[C - j], rtol=1e-12, atol=1e-12)


def test_ragged_last_chunk_boundaries():
    w, inp = _small_inputs(4, T=12, anchors=0)  # chunks of 5, 5, 2
    S_T = oracle.text_state(inp["Kx"], inp["Vx"])
    F, G = oracle.scan_states(inp["K"], inp["V"], inp["beta"], inp["alpha"], S_T, 5, 0)
    assert F.shape[0] == 4 and G.shape[0] == 4
    # F[3] is the state after every frame; G[0] likewise backwards
    S = 0.5 * S_T
    for t in range(12):
        S = oracle.frame_update(S, inp["alpha"][t], *oracle.frame_stats(inp["K"][t], inp["V"][t], inp["beta"][t]))
        if t == 9:
            np.testing.assert_allclose(F[2], S, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(F[3], S, rtol=1e-12, atol=1e-12)
    S = 0.5 * S_T
    for t in (11, 10):
        S = oracle.frame_update(S, inp["alpha"][t], *oracle.frame_stats(inp["K"][t], inp["V"][t], inp["beta"][t]))
    np.testing.assert_allclose(G[2], S, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("anchors", [0, 1])
def test_chunk_maps_are_the_scan_affine_maps(anchors):
    w, inp = _small_inputs(5, T=17, anchors=anchors)
    S_T = oracle.text_state(inp["Kx"], inp["Vx"])
    F, G = oracle.scan_states(inp["K"], inp["V"], inp["beta"], inp["alpha"], S_T, 5, anchors)
    Mf, Jf, Mb, Jb = oracle.chunk_maps(inp["K"], inp["V"], inp["beta"], inp["alpha"], 5, anchors)
    C = F.shape[0] - 1
    for c in range(C):
        np.testing.assert_allclose(F[c] @ Mf[c] + Jf[c], F[c + 1], rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(G[c + 1] @ Mb[c] + Jb[c], G[c], rtol=1e-11, atol=1e-11)
    # composed per-frame transitions (the definition of step (4)) agree too
    T = w.T
    for c in range(C):
        M = np.eye(w.d)
        J = np.zeros((w.d, w.d))
        for t in range(5 * c, min(5 * c + 5, T)):
            A, B = oracle.frame_stats(inp["K"][t], inp["V"][t], inp["beta"][t])
            Mt, Jt = oracle.transition(A, B, inp["alpha"][t], oracle.is_anchor(t, T, anchors))
            M, J = M @ Mt, J @ Mt + Jt
        np.testing.assert_allclose(M, Mf[c], rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(J, Jf[c], rtol=1e-11, atol=1e-11)


# --- readout -----------------------------------------------------------------
@pytest.mark.parametrize("anchors", [0, 1])
def test_no_frame_outside_any_window_reads_text_once(anchors):
    # C = 2: every chunk's window covers the whole clip, so the summed
    # readouts must give exactly the text state ("no double counting").
    w, inp = _small_inputs(6, T=10, anchors=anchors)
    out = oracle.vda_head(inp, 5, anchors)
    for t in range(10):
        if oracle.is_anchor(t, 10, anchors):
            assert not np.any(out["O"][t])
        else:
            np.testing.assert_allclose(out["O"][t], inp["Q"][t] @ out["S_T"].T, rtol=1e-12, atol=1e-12)


def test_window_excludes_exactly_the_neighbouring_chunks():
    # Only chunk cs writes (beta = 0 elsewhere, no text, no decay): a query
    # chunk sees it iff cs lies outside its window of chunks c-1..c+1.
    w, inp = _small_inputs(7, T=40, anchors=1)
    cs = 4
    b9 = float(np.float32(0.9))
    beta = np.zeros(40, np.float32)
    beta[5 * cs: 5 * cs + 5] = b9
    inp = dict(inp, beta=beta, alpha=np.ones_like(inp["alpha"]), beta_x=0.0)
    out = oracle.vda_head(inp, 5, 1)
    S = np.zeros((w.d, w.d))
    for t in range(5 * cs, 5 * cs + 5):
        S = oracle.frame_update(S, np.ones(w.d), *oracle.frame_stats(inp["K"][t], inp["V"][t], b9))
    Sb = np.zeros((w.d, w.d))
    for t in range(5 * cs + 4, 5 * cs - 1, -1):
        Sb = oracle.frame_update(Sb, np.ones(w.d), *oracle.frame_stats(inp["K"][t], inp["V"][t], b9))
    for t in range(1, 39):
        c = t // 5
        if abs(c - cs) <= 1:
            assert not np.any(out["O"][t]), t
        else:
            ref = inp["Q"][t] @ (S if c > cs else Sb).T
            np.testing.assert_allclose(out["O"][t], ref, rtol=1e-12, atol=1e-12)


def test_anchor_frames_neither_write_nor_read():
    w, inp = _small_inputs(8, T=20, anchors=1)
    out = oracle.vda_head(inp, 5, 1)
    assert not np.any(out["O"][0]) and not np.any(out["O"][19])
    inp2 = dict(inp)
    for k in ("K", "V"):
        x = inp[k].copy()
        x[0] = 3.0 * np.roll(x[0], 1, axis=0)
        x[19] = -x[19]
        inp2[k] = x
    out2 = oracle.vda_head(inp2, 5, 1)
    np.testing.assert_array_equal(out["O"], out2["O"])


def test_readout_is_linear_in_queries():
    w, inp = _small_inputs(9, T=25, anchors=1)
    S_T = oracle.text_state(inp["Kx"], inp["Vx"])
    F, G = oracle.scan_states(inp["K"], inp["V"], inp["beta"], inp["alpha"], S_T, 5, 1)
    Q2 = np.random.default_rng(0).standard_normal(inp["Q"].shape)
    O1 = oracle.chunk_readout(inp["Q"], F, G, 5, 1)
    O2 = oracle.chunk_readout(Q2, F, G, 5, 1)
    O3 = oracle.chunk_readout(2.0 * inp["Q"] - 0.5 * Q2, F, G, 5, 1)
    np.testing.assert_allclose(O3, 2.0 * O1 - 0.5 * O2, rtol=1e-12, atol=1e-12)


def test_planted_mistake_is_caught():
    """A transposed injection (B^T in place of B) must break the optimality pin."""
    rng = _rng(77)
    K, V = _frame(rng, 20, 6, 6)
    A, B = oracle.frame_stats(K, V, 0.5)
    S = oracle.frame_update(np.zeros((6, 6)), np.ones(6), A, B.T)
    grad = S.copy()
    for u in range(20):
        grad += 0.5 * np.outer(S @ K[u] - V[u], K[u])
    assert np.linalg.norm(grad) > 1e-3


def test_synthetic_workloads_have_the_stated_statistics():
    w = synth.WORKLOADS["batched"]
    small = synth.Workload("b", w.index, B=1, H=1, T=2, U=w.U, d=w.d, n_text=8, dtype="bf16",
                           alpha_lo=w.alpha_lo, anchors=1, near_dup=True)
    inp = synth.generate_head(small, 0, 0)
    K = inp["K"][0].astype(np.float64)
    norms = np.linalg.norm(K, axis=1)
    assert np.allclose(norms, 1.0, atol=1e-2)
    # near-duplicate keys: most pairs sharing a prototype have cosine ~0.99
    cos = K @ K.T
    assert np.quantile(cos[np.triu_indices(len(K), 1)], 0.95) > 0.97
    assert np.all(inp["beta"] >= 0.1) and np.all(inp["beta"] <= 1.0)
    assert np.all(inp["alpha"] >= 0.95) and np.all(inp["alpha"] <= 1.0)
    # bf16 storage: the low 16 bits are clear
    assert not np.any(inp["Q"].view(np.uint32) & 0xFFFF)


# --- per-token write gates beta_{t,u} ("Core method" objective) -------------
def test_zero_token_gates_drop_those_tokens():
    # a token whose gate is 0 has no term in the frame objective, so the
    # statistics equal those of the frame without it
    rng = _rng(40)
    K, V = _frame(rng, 9, 5, 4)
    beta = rng.uniform(0.1, 1.0, 9)
    keep = np.array([1, 0, 1, 1, 0, 0, 1, 1, 0], bool)
    A, B = oracle.frame_stats(K, V, np.where(keep, beta, 0.0))
    A2, B2 = oracle.frame_stats(K[keep], V[keep], beta[keep])
    np.testing.assert_allclose(A, A2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(B, B2, rtol=1e-13, atol=1e-13)


def test_equal_token_gates_are_the_frame_gate():
    w = synth.Workload("eq", 90, B=1, H=1, T=12, U=6, d=4, n_text=5, dtype="f32", alpha_lo=0.9,
                       anchors=1)
    inp = synth.generate_head(w, 0, 0)
    tok = dict(inp)
    tok["beta"] = np.repeat(inp["beta"][:, None], w.U, axis=1)
    tok["beta_x"] = np.full(w.n_text, inp["beta_x"])
    a, b = oracle.vda_head(inp, w.chunk, w.anchors), oracle.vda_head(tok, w.chunk, w.anchors)
    for k in ("S_T", "F", "G", "O"):
        np.testing.assert_allclose(b[k], a[k], rtol=1e-12, atol=1e-12)


def test_per_token_scan_matches_frame_by_frame_brute_force():
    # forward boundary states from the stacked least-squares solve of each
    # frame's objective (per-token weights), chained by hand
    rng = _rng(41)
    T, U, d, chunk = 7, 3, 3, 2
    K = np.stack([_frame(rng, U, d, d)[0] for _ in range(T)])
    V = rng.standard_normal((T, U, d))
    beta = rng.uniform(0.0, 1.5, (T, U))
    alpha = rng.uniform(0.6, 1.0, (T, d))
    S_T = rng.standard_normal((d, d))
    F, G = oracle.scan_states(K, V, beta, alpha, S_T, chunk, anchors=0)
    S = 0.5 * S_T
    ref = [S]
    for t in range(T):
        S = _brute_frame(S * alpha[t][None, :], K[t], V[t], beta[t])
        if (t + 1) % chunk == 0 or t == T - 1:
            ref.append(S)
    np.testing.assert_allclose(F, np.stack(ref), rtol=1e-9, atol=1e-9)


def test_per_token_synthetic_gates():
    w = synth.WORKLOADS["small_tb"]
    inp = synth.generate_head(w, 0, 2)
    assert inp["beta"].shape == (w.T, w.U) and inp["beta_x"].shape == (w.n_text,)
    for x in (inp["beta"], inp["beta_x"]):
        assert x.min() >= w.beta_lo and x.max() <= 1.0 and x.std() > 0.2
    # the per-frame workloads keep their gates: the stream of beta is unchanged
    assert synth.generate_head(synth.WORKLOADS["small"], 0, 2)["beta"].shape == (w.T,)


# --- readout epilogue: RMSNorm then a sigmoid gate (step (5)) ----------------
def test_gated_rmsnorm_is_the_library_rmsnorm_times_sigmoid():
    import torch
    rng = _rng(50)
    O = rng.standard_normal((3, 7, 16))
    w = rng.uniform(0.5, 1.5, 16)
    g = rng.standard_normal((3, 7, 16)) * 2
    ref = torch.nn.functional.rms_norm(torch.from_numpy(O), (16,), torch.from_numpy(w), eps=1e-6)
    ref = (ref * torch.sigmoid(torch.from_numpy(g))).numpy()
    np.testing.assert_allclose(oracle.gated_rmsnorm(O, w, g, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_gated_rmsnorm_invariants():
    rng = _rng(51)
    O = rng.standard_normal((5, 32)) * 3
    w = np.ones(32)
    # an open gate leaves unit RMS; a zero logit halves it exactly
    y = oracle.gated_rmsnorm(O, w, np.full_like(O, 60.0), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-12)
    np.testing.assert_allclose(oracle.gated_rmsnorm(O, w, np.zeros_like(O), 0.0), 0.5 * y, rtol=1e-12)
    # scale invariance (eps = 0) and a zero row (anchor) stays zero
    np.testing.assert_allclose(oracle.gated_rmsnorm(7.5 * O, w, O, 0.0), oracle.gated_rmsnorm(O, w, O, 0.0),
                               rtol=1e-12)
    assert not np.any(oracle.gated_rmsnorm(np.zeros((2, 32)), w, O[:2], 1e-6))
