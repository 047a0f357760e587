"""ARL2 inter-frame branch on the GPU (sfa_gdn_forward) against the float64 oracle
("Asistir Localmente, Recordar Linealmente", §2.1-2.2).

Every element of O and of the state is compared with the oracle, one frame at a time:
frame n runs on the GPU as a call of its own from the GPU's state after frame n-1 (the
chained calls reproduce the single call bit for bit, which is asserted), and the oracle
takes the same frame from the same state.  The per-element bound follows from the
kernel's arithmetic, first-order terms of each rounding (bf16 keeps 8 significant bits,
so a round to nearest is off by at most u = 2^-8 relative):

  O_n = bf16( sum_k q_ik bf16(S)_kj )                       (fp32 accumulation)
      |dO_ij| <= u |O_ij| + (u + g) (|Q| |S|)_ij
  S_n = fma(alpha, S, B^ - bf16(M^) bf16(S))               (fp32)
      M^ = sum_i K~_i^T K~_i, B^ = sum_i K~_i^T V~_i with K~ = bf16(sqrt(beta) k),
      V~ = bf16(sqrt(beta) v): each product of two rounded factors is off by 2u,
      bf16(M^) adds u and bf16(S) another u, so with
      Mabs = sum_i beta_i |k_i|^T |k_i| and Babs = sum_i beta_i |k_i|^T |v_i|:
      |dS_kj| <= (4u + g) (Mabs |S|)_kj + (2u + g) Babs_kj + 2^-21 (alpha |S| + |S_n|)_kj
where g = 2^-12 covers the fp32 accumulation inside the tensor cores (at most ~100 adds of
2^-23 each at P = 1560, i.e. < 2^-16) and the square root's own rounding.

A second line compares the GPU chain with the oracle's own chain from the same S_0, per
(batch, head) and frame.  The update is linear in the state, so the state error
propagates as dS_n = (alpha_n I - M_n) dS_{n-1} + r_n with r_n the frame's rounding
(bounded element-wise above, at the GPU's state):
  e_n = ||alpha_n I - M_n||_2 e_{n-1} + ||bound on r_n||_F,   ||S_n^gpu - S_n||_F <= e_n,
  ||O_n^gpu - O_n||_F <= ||Q_n||_2 e_{n-1} + ||bound on O_n's rounding||_F,
with M_n = K_n^T diag(beta_n) K_n (both norms taken in float64).

Worst-case bounds let a small systematic error through (a gate or a step size off by a
per cent stays inside 2u).  Rounding to nearest is unbiased, so with at least 128 tokens
per frame the error's projection on the reference, <dS, S> / <S, S> per (batch, head),
stays near u / sqrt(d^2) (about 1e-4 on these inputs); the tests require it below 2^-10,
which a 1 % change of alpha or beta exceeds several times over.
"""
import numpy as np
import pytest
import torch

from oracle import gdn
from sfa_workloads import WORKLOADS, gdn_inputs

from gpu_helpers import sfa

pytestmark = pytest.mark.gpu

U = 2.0 ** -8      # bf16 unit roundoff
G_ACC = 2.0 ** -12


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _inputs(B, H, T, P, seed, s0_scale=0.5):
    q, k, v, a, b = gdn_inputs(B, H, T, P, 128, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed + 100)
    s0 = s0_scale * torch.randn(B, H, 128, 128, generator=g, dtype=torch.float32)
    return q, k, v, a, b, s0


def _oracle(q, k, v, a, b, P, s0, update=True):
    return gdn.gdn_frames(q.float().numpy(), k.float().numpy(), v.float().numpy(), a.numpy(), b.numpy(), P,
                          S0=None if s0 is None else s0.numpy(), update=update)


def _bound_o(q_n, s_prev, o_ref):
    """Per-element bound on O of one frame read from the state s_prev (float64 numpy)."""
    return U * np.abs(o_ref) + (U + G_ACC) * (np.abs(q_n) @ np.abs(s_prev))


def _bound_s(k_n, v_n, a_n, b_n, s_prev, s_ref):
    """Per-element bound on the state after one frame update from s_prev."""
    kb = np.abs(k_n) * b_n[..., None]
    mabs = np.swapaxes(kb, -1, -2) @ np.abs(k_n)
    babs = np.swapaxes(kb, -1, -2) @ np.abs(v_n)
    return ((4 * U + G_ACC) * (mabs @ np.abs(s_prev)) + (2 * U + G_ACC) * babs
            + 2.0 ** -21 * (a_n[..., None, None] * np.abs(s_prev) + np.abs(s_ref)))


def _ratio(err, bnd):
    """Largest err / bnd; an element with a zero bound must be exact."""
    assert np.all(err[bnd == 0] == 0)
    pos = bnd > 0
    return float((err[pos] / bnd[pos]).max()) if pos.any() else 0.0


def _spec(x):
    """Spectral norm of every matrix in a [..., m, n] float64 array."""
    g = np.swapaxes(x, -1, -2) @ x if x.shape[-2] >= x.shape[-1] else x @ np.swapaxes(x, -1, -2)
    return np.sqrt(np.maximum(np.linalg.eigvalsh(g)[..., -1], 0.0))


def _fro(x):
    return np.sqrt((x * x).sum(axis=(-2, -1)))


BIAS_TOL = 2.0 ** -10


def _bias(err, ref):
    """|<err, ref>| / <ref, ref> per matrix of a [..., m, n] array (0 where ref is 0)."""
    den = (ref * ref).sum(axis=(-2, -1))
    return np.abs((err * ref).sum(axis=(-2, -1))) / np.where(den > 0, den, 1.0)


def check_elementwise(q, k, v, a, b, P, s0, o_full, s_full, update=True):
    """Check a sfa_gdn_forward result (o_full, s_full), computed in one call from state s0
    (CPU tensors; s0 None = zeros), frame by frame: every element against the oracle's
    step from the GPU's own previous state, and every (batch, head, frame) against the
    oracle's chain from s0 within the propagated bound.  Returns the largest fraction of
    its bound reached by an O element, a state element and a chain norm."""
    m = sfa()
    B, H, L, d = q.shape
    T = L // P
    qc, kc, vc, ac, bc = (x.cuda() for x in (q, k, v, a, b))
    state = (torch.zeros(B, H, d, d) if s0 is None else s0).cuda()
    qf, kf, vf = q.double().numpy(), k.double().numpy(), v.double().numpy()
    an, bn = a.double().numpy(), b.double().numpy()
    s_chain = state.cpu().double().numpy()     # the oracle's own chain
    e = np.zeros((B, H))                        # bound on ||S^gpu - S^chain||_F
    worst_o = worst_s = worst_c = 0.0
    for n in range(T):
        rows = slice(n * P, (n + 1) * P)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        o_n, s_n = m.gdn_forward(qc[:, :, rows].contiguous(), kc[:, :, rows].contiguous(),
                                 vc[:, :, rows].contiguous(), ac[:, :, n:n + 1].contiguous(),
                                 bc[:, :, rows].contiguous(), P, state_in=state, update=update,
                                 dev_status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        # the chained frame reproduces the single call's frame bit for bit
        assert torch.equal(o_n.cpu(), o_full[:, :, rows].cpu()), f"frame {n}: chained O differs"
        s_prev = state.cpu().double().numpy()
        qn, kn, vn, bt = qf[:, :, rows], kf[:, :, rows], vf[:, :, rows], bn[:, :, rows]
        o_ref, s_ref = gdn.gdn_frames(qn, kn, vn, an[:, :, n:n + 1], bt, P, S0=s_prev, update=update)
        o_gpu = o_n.float().cpu().double().numpy()
        bnd_o = _bound_o(qn, s_prev, o_ref)
        ratio = _ratio(np.abs(o_gpu - o_ref), bnd_o)
        worst_o = max(worst_o, ratio)
        assert ratio <= 1.0, f"frame {n}: O element error {ratio:.3f} x its bound"
        if P >= 128:
            assert _bias(o_gpu - o_ref, o_ref).max() <= BIAS_TOL, f"frame {n}: O error correlates with O"
        # the oracle's chain: O of this frame within the propagated bound
        o_c, s_c = gdn.gdn_frames(qn, kn, vn, an[:, :, n:n + 1], bt, P, S0=s_chain, update=update)
        rhs = _spec(qn) * e + _fro(bnd_o)
        lhs = _fro(o_gpu - o_c)
        assert np.all(lhs <= rhs), f"frame {n}: O off the oracle's chain by {(lhs / rhs).max():.3f} x its bound"
        worst_c = max(worst_c, float(np.max(np.where(rhs > 0, lhs / np.where(rhs > 0, rhs, 1), 0))))
        if update:
            s_gpu = s_n.cpu().double().numpy()
            bnd_s = _bound_s(kn, vn, an[:, :, n], bt, s_prev, s_ref)
            ratio = _ratio(np.abs(s_gpu - s_ref), bnd_s)
            worst_s = max(worst_s, ratio)
            assert ratio <= 1.0, f"frame {n}: state element error {ratio:.3f} x its bound"
            if P >= 128:
                assert _bias(s_gpu - s_ref, s_ref).max() <= BIAS_TOL, f"frame {n}: state error correlates with S"
            kb = kn * bt[..., None]
            mn = np.swapaxes(kb, -1, -2) @ kn
            amat = an[:, :, n][..., None, None] * np.eye(d) - mn
            e = np.abs(np.linalg.eigvalsh(amat)).max(axis=-1) * e + _fro(bnd_s)
            lhs = _fro(s_gpu - s_c)
            assert np.all(lhs <= e), f"frame {n}: state off the oracle's chain by {(lhs / e).max():.3f} x its bound"
            worst_c = max(worst_c, float((lhs / e).max()))
            state, s_chain = s_n, s_c
        else:
            assert torch.equal(s_n.cpu(), state.cpu())     # read-only: the state passes through
    if update:
        assert torch.equal(state.cpu(), s_full.cpu()), "chained final state differs from the single call"
    return worst_o, worst_s, worst_c


@pytest.mark.parametrize("B,H,T,P", [(2, 2, 3, 200), (1, 3, 5, 1), (1, 2, 2, 384), (1, 1, 4, 130)])
def test_gdn_matches_oracle(B, H, T, P):
    q, k, v, a, b, s0 = _inputs(B, H, T, P, seed=P + T)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, s = sfa().gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), P, state_in=s0.cuda(),
                             dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    check_elementwise(q, k, v, a, b, P, s0, o, s)


def test_gdn_read_only_steps_keep_the_state():
    B, H, T, P = 1, 2, 3, 200
    q, k, v, a, b, s0 = _inputs(B, H, T, P, seed=7)
    o, s = sfa().gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), P, state_in=s0.cuda(), update=False)
    torch.cuda.synchronize()
    assert torch.equal(s.cpu(), s0)                   # not written
    check_elementwise(q, k, v, a, b, P, s0, o, s, update=False)


def test_gdn_state_chains_across_calls():
    # frames [0, 4) in one call == frames [0, 2) then [2, 4) with the state passed on
    B, H, T, P = 1, 2, 4, 136
    q, k, v, a, b, s0 = (x.cuda() for x in _inputs(B, H, T, P, seed=3))
    m = sfa()
    o1, s1 = m.gdn_forward(q, k, v, a, b, P, state_in=s0)
    h = 2 * P
    oa, sa = m.gdn_forward(q[:, :, :h].contiguous(), k[:, :, :h].contiguous(), v[:, :, :h].contiguous(),
                           a[:, :, :2].contiguous(), b[:, :, :h].contiguous(), P, state_in=s0)
    ob, sb = m.gdn_forward(q[:, :, h:].contiguous(), k[:, :, h:].contiguous(), v[:, :, h:].contiguous(),
                           a[:, :, 2:].contiguous(), b[:, :, h:].contiguous(), P, state_in=sa)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, :, :h], oa) and torch.equal(o1[:, :, h:], ob) and torch.equal(s1, sb)


def test_gdn_zero_state_and_in_place_state():
    B, H, T, P = 1, 2, 2, 200
    q, k, v, a, b, s0 = _inputs(B, H, T, P, seed=4)
    m = sfa()
    o, s = m.gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), P)          # state_in NULL
    st = torch.zeros(B, H, 128, 128, device="cuda")
    o2, s2 = m.gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), P, state_in=st, state_out=st)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(s, s2) and s2.data_ptr() == st.data_ptr()
    assert o[:, :, :P].abs().max().item() == 0.0      # frame 0 reads the empty state


def test_gdn_workload_every_element():
    # ARL2 §2.1 at the 24-frame, 12-head workload: every element of every frame of O and
    # of the state, each frame against the oracle from the GPU's previous state, and the
    # whole chain against the oracle's chain
    w = WORKLOADS["gdn"]
    q, k, v, a, b = gdn_inputs(w.B, w.H, w.Tq, w.P, w.d, seed=0)
    o, s = sfa().gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), w.P)
    torch.cuda.synchronize()
    worst_o, worst_s, worst_c = check_elementwise(q, k, v, a, b, w.P, None, o, s)
    o_ref, s_ref = gdn.gdn_frames(q.float().numpy(), k.float().numpy(), v.float().numpy(), a.numpy(), b.numpy(), w.P)
    err = np.abs(o.float().cpu().numpy() - o_ref)
    print(f"gdn workload: largest fraction of the bound {worst_o:.3f} (O elements), {worst_s:.3f} (state "
          f"elements), {worst_c:.3f} (chain); O max-abs error {err.max():.3e} (max |O| {np.abs(o_ref).max():.3e}), "
          f"state relative Frobenius error {_rel(s.cpu().numpy(), s_ref):.3e}")


def test_gdn_rejects_bad_arguments():
    m = sfa()
    q, k, v, a, b, _ = (x.cuda() for x in _inputs(1, 1, 2, 64, seed=1))
    with pytest.raises(ValueError):
        m.gdn_forward(q, k, v, a, b, 48)                 # 128 tokens are not frames of 48
    d64 = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.SfaError):
        m.gdn_forward(d64, d64, d64, a, b, 64, state_out=torch.empty(1, 1, 64, 64, device="cuda"))


def test_gdn_update_needs_the_workspace_and_is_deterministic():
    B, H, T, P = 2, 3, 4, 1000
    q, k, v, a, b, s0 = (x.cuda() for x in _inputs(B, H, T, P, seed=11))
    m = sfa()
    with pytest.raises(m.SfaError):
        m.gdn_forward(q, k, v, a, b, P, state_in=s0, workspace=None)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, s1 = m.gdn_forward(q, k, v, a, b, P, state_in=s0, dev_status=status)
    o2, s2 = m.gdn_forward(q, k, v, a, b, P, state_in=s0)
    torch.cuda.synchronize()
    assert status.item() == 0
    # every CTA of a head runs the same recurrence: no sum depends on the launch order
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    check_elementwise(q.cpu(), k.cpu(), v.cpu(), a.cpu(), b.cpu(), P, s0.cpu(), o1, s1)


def test_gdn_many_heads_one_cta_each():
    # 75 heads leave one CTA per head: every CTA takes all 3 tiles of each frame
    B, H, T, P = 3, 25, 3, 384
    q, k, v, a, b, s0 = _inputs(B, H, T, P, seed=21)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, s = sfa().gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), P, state_in=s0.cuda(),
                             dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    check_elementwise(q, k, v, a, b, P, s0, o, s)


def test_gdn_negative_step_size_is_reported():
    B, H, T, P = 1, 2, 2, 200
    q, k, v, a, b, s0 = (x.cuda() for x in _inputs(B, H, T, P, seed=5))
    b = b.clone()
    b[0, 1, 7] = -0.5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa().gdn_forward(q, k, v, a, b, P, state_in=s0, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == sfa().SFA_ERR_INVALID_ARG


def test_gdn_stalled_recurrence_times_out_and_context_survives():
    # the test hook keeps the recurrence kernel's input state from being signalled ready:
    # its tensor-core warp's first wait runs out after 20 ms, the other roles stop at their
    # next wait, the copy warp lets its copies in flight land, and the call reports
    # SFA_ERR_TIMEOUT; the next call on the same context is correct
    B, H, T, P = 1, 2, 3, 300
    q, k, v, a, b, s0 = _inputs(B, H, T, P, seed=31)
    qc, kc, vc, ac, bc, sc = (x.cuda() for x in (q, k, v, a, b, s0))
    m = sfa()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.gdn_forward(qc, kc, vc, ac, bc, P, state_in=sc, dev_status=status, timeout_us=20000,
                  debug_flags=m.SFA_DEBUG_STALL_GDN_STATE)
    torch.cuda.synchronize()
    assert status.item() == m.SFA_ERR_TIMEOUT
    status.zero_()
    o, s = m.gdn_forward(qc, kc, vc, ac, bc, P, state_in=sc, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    check_elementwise(q, k, v, a, b, P, s0, o, s)
