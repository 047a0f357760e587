"""ARL2 inter-frame branch (gated delta rule with frame-level state access), float64.
TEST INFRASTRUCTURE ONLY.

"Resumen Técnico: Asistir Localmente, Recordar Linealmente (ARL2)":
  * §2.1 (Rama Inter-Cuadro): a fixed-size recurrent state S replaces the growing KV
    cache; the feature-mapped projections Q', K', V' (per-head 1x1 maps φ applied by the
    caller) drive the gated update  S_N = α_N S_{N-1} + β_N K'_N (V'_N - K'_N S_{N-1})
    and the output  O_inter = Q'_N S_{N-1};
  * §2.2 (Acceso a Nivel de Cuadro): every token of frame N reads the same pre-update
    state S_{N-1}; the state changes only after the whole frame;
  * §2.2 (Actualizaciones de Paso Limpio): during the intermediate denoising steps the
    state is read but not written.

Readings of the page (where it leaves a step open):
  * shapes: Q'_N, K'_N are [P, d_k] and V'_N is [P, d_v] (the frame's tokens as rows);
    S is [d_k, d_v]; the update's correction term is K'_N^T diag(β_N) (V'_N - K'_N S_{N-1})
    (the transpose makes the product [d_k, d_v]);
  * β is per token (the page: per-token learned projection), α per frame: one forget
    factor scales the whole state once per frame update;
  * the state starts from the caller's S_0 (zero for a new video).

Parity status: pinned (tests/test_oracle_gdn.py: the update equals one gradient step of
the weighted least-squares loss ½ Σ_i β_i |k_i S - v_i|² taken by finite differences,
exact storage of orthonormal key/value pairs, frame-level access, clean-step reads, and
gate special cases).
"""
from __future__ import annotations

import numpy as np


def gdn_frames(q, k, v, alpha, beta, P: int, S0=None, update: bool = True):
    """q, k: [B, H, T*P, d_k]; v: [B, H, T*P, d_v]; alpha: [B, H, T]; beta: [B, H, T*P];
    S0: [B, H, d_k, d_v] or None (zeros).  Frames are processed in order; with update
    False every frame reads S0 (clean-step reading: no write).
    Returns O [B, H, T*P, d_v] and the final state [B, H, d_k, d_v], float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    T = L // P
    S = np.zeros((B, H, dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    O = np.zeros((B, H, L, dv))
    for b in range(B):
        for h in range(H):
            s = S[b, h].copy()
            for n in range(T):
                rows = slice(n * P, (n + 1) * P)
                qn, kn, vn = q[b, h, rows], k[b, h, rows], v[b, h, rows]
                O[b, h, rows] = qn @ s                      # every token reads S_{N-1}
                if update:
                    u = vn - kn @ s                         # prediction error of the frame
                    s = alpha[b, h, n] * s + kn.T @ (beta[b, h, rows][:, None] * u)
            S[b, h] = s
    return O, S
