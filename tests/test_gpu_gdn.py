"""ARL2 inter-frame branch on the GPU (sfa_gdn_forward) against the float64 oracle
("Asistir Localmente, Recordar Linealmente", §2.1-2.2).

Tolerance from the arithmetic: the tensor cores read the state S and the per-token
corrections U as bf16 (relative rounding <= 2^-9 each), everything else is fp32.  One
frame therefore perturbs O and the state update by about 2^-8 relative; over T frames
the errors add (the forget factor only shrinks old ones), so the tests bound the
relative Frobenius error of O and of the final state by T * 2^-8 (at least 2^-7).
"""
import numpy as np
import pytest
import torch

from oracle import gdn
from sfa_workloads import WORKLOADS, gdn_inputs

from gpu_helpers import sfa

pytestmark = pytest.mark.gpu


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _inputs(B, H, T, P, seed, s0_scale=0.5):
    q, k, v, a, b = gdn_inputs(B, H, T, P, 128, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed + 100)
    s0 = s0_scale * torch.randn(B, H, 128, 128, generator=g, dtype=torch.float32)
    return q, k, v, a, b, s0


def _oracle(q, k, v, a, b, P, s0, update=True):
    return gdn.gdn_frames(q.float().numpy(), k.float().numpy(), v.float().numpy(), a.numpy(), b.numpy(), P,
                          S0=s0.numpy(), update=update)


@pytest.mark.parametrize("B,H,T,P", [(2, 2, 3, 200), (1, 3, 5, 1), (1, 2, 2, 384), (1, 1, 4, 130)])
def test_gdn_matches_oracle(B, H, T, P):
    q, k, v, a, b, s0 = _inputs(B, H, T, P, seed=P + T)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, s = sfa().gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), P, state_in=s0.cuda(),
                             dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_ref, s_ref = _oracle(q, k, v, a, b, P, s0)
    tol = max(T * 2.0 ** -8, 2.0 ** -7)
    assert _rel(o.float().cpu().numpy(), o_ref) <= tol
    assert _rel(s.cpu().numpy(), s_ref) <= tol
    # and frame by frame (the first frame reads the exact input state)
    for n in range(T):
        rows = slice(n * P, (n + 1) * P)
        assert _rel(o.float().cpu().numpy()[:, :, rows], o_ref[:, :, rows]) <= tol


def test_gdn_read_only_steps_keep_the_state():
    B, H, T, P = 1, 2, 3, 200
    q, k, v, a, b, s0 = _inputs(B, H, T, P, seed=7)
    o, s = sfa().gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), P, state_in=s0.cuda(), update=False)
    torch.cuda.synchronize()
    assert torch.equal(s.cpu(), s0)                   # not written
    o_ref, _ = _oracle(q, k, v, a, b, P, s0, update=False)
    assert _rel(o.float().cpu().numpy(), o_ref) <= 2.0 ** -7


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


def test_gdn_workload_sampled():
    w = WORKLOADS["gdn"]
    q, k, v, a, b = gdn_inputs(w.B, w.H, w.Tq, w.P, w.d, seed=0)
    o, s = sfa().gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), w.P)
    torch.cuda.synchronize()
    o_ref, s_ref = gdn.gdn_frames(q.float().numpy(), k.float().numpy(), v.float().numpy(), a.numpy(), b.numpy(), w.P)
    tol = w.Tq * 2.0 ** -8
    assert _rel(s.cpu().numpy(), s_ref) <= tol
    for n in (1, 12, 23):
        rows = slice(n * w.P, (n + 1) * w.P)
        assert _rel(o.float().cpu().numpy()[:, :, rows], o_ref[:, :, rows]) <= tol


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
    o_ref, s_ref = _oracle(q.cpu(), k.cpu(), v.cpu(), a.cpu(), b.cpu(), P, s0.cpu())
    tol = T * 2.0 ** -8
    assert _rel(s1.cpu().numpy(), s_ref) <= tol
    assert _rel(o1.float().cpu().numpy(), o_ref) <= tol


def test_gdn_many_heads_one_cta_each():
    # 75 heads leave one CTA per head: every CTA takes all 3 tiles of each frame
    B, H, T, P = 3, 25, 3, 384
    q, k, v, a, b, s0 = _inputs(B, H, T, P, seed=21)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, s = sfa().gdn_forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), P, state_in=s0.cuda(),
                             dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_ref, s_ref = _oracle(q, k, v, a, b, P, s0)
    tol = max(T * 2.0 ** -8, 2.0 ** -7)
    assert _rel(s.cpu().numpy(), s_ref) <= tol
    assert _rel(o.float().cpu().numpy(), o_ref) <= tol


def test_gdn_negative_step_size_is_reported():
    B, H, T, P = 1, 2, 2, 200
    q, k, v, a, b, s0 = (x.cuda() for x in _inputs(B, H, T, P, seed=5))
    b = b.clone()
    b[0, 1, 7] = -0.5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa().gdn_forward(q, k, v, a, b, P, state_in=s0, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == sfa().SFA_ERR_INVALID_ARG
