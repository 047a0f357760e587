"""Pins of the ARL2 inter-frame oracle ("Asistir Localmente, Recordar Linealmente",
§2.1-2.2) to facts other than its own formula: the update is one gradient step of a
weighted least-squares loss (checked by finite differences), the delta rule stores
orthonormal key/value pairs exactly, frame-level access, clean-step reads, gate cases."""
import numpy as np
import pytest

from oracle import gdn
from sfa_workloads import gdn_inputs


def _rand(seed, B=1, H=2, T=3, P=5, dk=4, dv=3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T * P, dk))
    k = rng.standard_normal((B, H, T * P, dk)) * 0.3
    v = rng.standard_normal((B, H, T * P, dv))
    alpha = rng.uniform(0.5, 1.0, (B, H, T))
    beta = rng.uniform(0.0, 1.0, (B, H, T * P))
    S0 = rng.standard_normal((B, H, dk, dv))
    return q, k, v, alpha, beta, S0


def test_update_is_a_gradient_step_of_the_weighted_loss():
    # L(S) = 1/2 sum_i beta_i |k_i S - v_i|^2; the update is S' = alpha S - grad L(S).
    # grad L by central differences (exact for a quadratic, up to rounding)
    q, k, v, alpha, beta, S0 = _rand(0, T=1)
    P = 5
    _, S1 = gdn.gdn_frames(q, k, v, alpha, beta, P, S0=S0)
    for h in range(2):
        s = S0[0, h]
        kk, vv, bb = k[0, h], v[0, h], beta[0, h]

        def loss(x):
            r = kk @ x - vv
            return 0.5 * float(np.sum(bb[:, None] * r * r))

        g = np.zeros_like(s)
        eps = 1e-3
        for i in range(s.shape[0]):
            for j in range(s.shape[1]):
                e = np.zeros_like(s)
                e[i, j] = eps
                g[i, j] = (loss(s + e) - loss(s - e)) / (2 * eps)
        assert np.abs(S1[0, h] - (alpha[0, h, 0] * s - g)).max() < 1e-9


def test_orthonormal_pairs_are_stored_exactly():
    # beta = 1, alpha = 1, S0 = 0, frame 0 keys orthonormal: after the frame K S = V,
    # so frame 1 queried with frame 0's keys returns frame 0's values
    rng = np.random.default_rng(1)
    d, P = 6, 4
    basis, _ = np.linalg.qr(rng.standard_normal((d, d)))
    k0 = basis[:P]                      # P orthonormal rows
    v0 = rng.standard_normal((P, 3))
    q = np.zeros((1, 1, 2 * P, d))
    q[0, 0, P:] = k0
    k = np.zeros((1, 1, 2 * P, d))
    k[0, 0, :P] = k0
    v = np.zeros((1, 1, 2 * P, 3))
    v[0, 0, :P] = v0
    O, S = gdn.gdn_frames(q, k, v, np.ones((1, 1, 2)), np.ones((1, 1, 2 * P)), P)
    assert np.abs(O[0, 0, P:] - v0).max() < 1e-12
    assert np.abs(O[0, 0, :P]).max() == 0.0          # frame 0 read the empty state


def test_frame_level_access_and_token_order():
    # every token of frame N reads S_{N-1}: O rows of frame N are Q_N S_{N-1}; permuting
    # the tokens of a frame permutes its rows of O and leaves the final state unchanged
    q, k, v, alpha, beta, S0 = _rand(2)
    P = 5
    O, S = gdn.gdn_frames(q, k, v, alpha, beta, P, S0=S0)
    perm = np.concatenate([n * P + np.random.default_rng(n).permutation(P) for n in range(3)])
    O2, S2 = gdn.gdn_frames(q[:, :, perm], k[:, :, perm], v[:, :, perm], alpha, beta[:, :, perm], P, S0=S0)
    assert np.abs(O2 - O[:, :, perm]).max() < 1e-12
    assert np.abs(S2 - S).max() < 1e-12
    assert np.abs(O[0, 0, :P] - q[0, 0, :P] @ S0[0, 0]).max() < 1e-12


def test_clean_step_reads_do_not_write():
    q, k, v, alpha, beta, S0 = _rand(3)
    P = 5
    O, S = gdn.gdn_frames(q, k, v, alpha, beta, P, S0=S0, update=False)
    assert np.array_equal(S, S0)
    for n in range(3):
        assert np.abs(O[0, 1, n * P:(n + 1) * P] - q[0, 1, n * P:(n + 1) * P] @ S0[0, 1]).max() < 1e-12


def test_gate_special_cases():
    # beta = 0: the state only decays, S_N = (prod alpha) S0
    q, k, v, alpha, beta, S0 = _rand(4)
    P = 5
    O, S = gdn.gdn_frames(q, k, v, alpha, np.zeros_like(beta), P, S0=S0)
    decay = np.prod(alpha, axis=2)
    assert np.abs(S - decay[:, :, None, None] * S0).max() < 1e-12
    # frame 2 reads (alpha_0 alpha_1) S0
    f = alpha[0, 0, 0] * alpha[0, 0, 1]
    assert np.abs(O[0, 0, 2 * P:] - q[0, 0, 2 * P:] @ (f * S0[0, 0])).max() < 1e-12


def test_synthetic_inputs_are_stable():
    # the seeded stand-in for learned maps and gates keeps the state bounded
    q, k, v, a, b = gdn_inputs(1, 2, 8, 200, 64, seed=0)
    O, S = gdn.gdn_frames(q.float().numpy(), k.float().numpy(), v.float().numpy(), a.numpy(), b.numpy(), 200)
    assert np.isfinite(S).all() and np.abs(S).max() < 50 and np.abs(O).max() < 50


def test_planted_mistake_is_caught():
    # dropping the transpose-side weighting (beta applied after K^T instead of per token)
    # is a plausible slip; the gradient-step pin distinguishes it
    q, k, v, alpha, beta, S0 = _rand(5, T=1)
    s, kk, vv, bb = S0[0, 0], k[0, 0], v[0, 0], beta[0, 0]
    wrong = alpha[0, 0, 0] * s + bb.mean() * kk.T @ (vv - kk @ s)
    _, S1 = gdn.gdn_frames(q, k, v, alpha, beta, 5, S0=S0)
    assert np.abs(S1[0, 0] - wrong).max() > 1e-3


def test_linear_form_of_the_update_equals_the_delta_form():
    # the GPU kernels compute S_N = alpha S - M_N S + B_N with M_N = K^T diag(beta) K and
    # B_N = K^T diag(beta) V of frame N alone (formed for all frames before the recurrence);
    # that algebra, run in float64 here, reproduces the oracle's frame-by-frame delta form
    q, k, v, alpha, beta, S0 = _rand(3, B=2, H=2, T=4, P=6, dk=5, dv=4)
    P, T = 6, 4
    o_ref, s_ref = gdn.gdn_frames(q, k, v, alpha, beta, P, S0=S0)
    for b in range(2):
        for h in range(2):
            s = S0[b, h].copy()
            mats = []
            for n in range(T):  # independent of the state: all frames first
                rows = slice(n * P, (n + 1) * P)
                kb = k[b, h, rows] * beta[b, h, rows][:, None]
                mats.append((kb.T @ k[b, h, rows], kb.T @ v[b, h, rows]))
            for n in range(T):
                rows = slice(n * P, (n + 1) * P)
                np.testing.assert_allclose(q[b, h, rows] @ s, o_ref[b, h, rows], rtol=0, atol=1e-12)
                M, Bn = mats[n]
                s = alpha[b, h, n] * s - M @ s + Bn
            np.testing.assert_allclose(s, s_ref[b, h], rtol=0, atol=1e-12)
