"""Local and history branches in one launch (sfa_forward_dual) against the oracle.

"ISPA", §2.1 Dual-Stream Warmup: the local branch (current frame + sink) and the full
attention are both needed; with disjoint local and history sets the full attention is
the LSE merge of the branches.  The oracle computes the local branch and the full
attention (over the union of the two lists) directly, in float64.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sfa_workloads import SetSpec, WORKLOADS, Workload, sample_rows, workload_qkv

from gpu_helpers import O_TOL, LSE_TOL, compare, gpu_sets, oracle_sets, sfa

pytestmark = pytest.mark.gpu


def _branches(P, d, B=1, H=3, hist=tuple(range(1, 6)), T=7):
    local = Workload("dual_local", B=B, H=H, Tq=1, Tkv=T, q_off=T - 1, P=P, d=d, n_sink=1, n_prev=0, chunk_len=1,
                     heads=(SetSpec("anchor"),) * H)
    hist_w = Workload("dual_hist", B=B, H=H, Tq=1, Tkv=T, q_off=T - 1, P=P, d=d,
                      heads=(SetSpec("explicit", hist),) * H)
    full = Workload("dual_full", B=B, H=H, Tq=1, Tkv=T, q_off=T - 1, P=P, d=d,
                    heads=(SetSpec("explicit", tuple(sorted(set(hist) | {0, T - 1}))),) * H)
    return local, hist_w, full


def _run(local, hist_w, full, n_split, seed, rows=None):
    m = sfa()
    q, k, v = workload_qkv(local, seed=seed)
    fh, ch = gpu_sets(hist_w)
    fl, cl = gpu_sets(local, Amax=fh.shape[2])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ol, ll, of, lf = m.forward_dual(q.cuda(), k.cuda(), v.cuda(), fl, cl, fh, ch, local.P, n_split,
                                    dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    scale = 1 / math.sqrt(local.d)
    for w, o, l in ((local, ol, ll), (full, of, lf)):
        ofr, ocn = oracle_sets(w, 0, None)
        o_ref, l_ref = oracle.attention(q, k, v, ofr, ocn, w.P, scale, rows=rows)
        o_g = o.float().cpu().reshape(-1, w.d).numpy()
        l_g = l.cpu().reshape(-1).numpy()
        if rows is not None:
            o_g, l_g = o_g[rows], l_g[rows]
        compare(o_g, l_g, o_ref, l_ref)
    return q, k, v, (fl, cl, fh, ch), (ol, ll, of, lf)


@pytest.mark.parametrize("P,d,n_split", [(200, 128, 1), (200, 128, 2), (136, 64, 4), (1, 128, 1), (300, 64, 2),
                                         (200, 128, 0), (136, 64, 0), (1, 128, 0)])
def test_dual_matches_oracle_full_rows(P, d, n_split):
    local, hist_w, full = _branches(P, d, B=2)
    _run(local, hist_w, full, n_split, seed=P + d)


def test_dual_equals_two_forwards_and_a_merge():
    # one launch vs the three-call form (two forwards + sfa_lse_merge): same within the
    # extra bf16 rounding of the partials
    local, hist_w, full = _branches(200, 128)
    q, k, v, (fl, cl, fh, ch), (ol, ll, of, lf) = _run(local, hist_w, full, 1, seed=5)
    m = sfa()
    o1, l1 = m.forward(q.cuda(), k.cuda(), v.cuda(), fl, cl, local.P)
    o2, l2 = m.forward(q.cuda(), k.cuda(), v.cuda(), fh, ch, local.P)
    om, lm = m.lse_merge(o1, l1, o2, l2)
    torch.cuda.synchronize()
    assert (ol.float() - o1.float()).abs().max().item() <= 2 ** -7
    assert (ll - l1).abs().max().item() < 1e-5
    assert (of.float() - om.float()).abs().max().item() <= 2 ** -6
    assert (lf - lm).abs().max().item() < 1e-5


def test_dual_empty_history():
    # a history list that is empty for every head: full == local
    local, _, _ = _branches(160, 128, hist=())
    hist_w = Workload("dual_hist_empty", B=1, H=3, Tq=1, Tkv=7, q_off=6, P=160, d=128,
                      heads=(SetSpec("explicit", ()),) * 3)
    q, k, v = (x.cuda() for x in workload_qkv(local, seed=9))
    fl, cl = gpu_sets(local)
    fh = torch.full_like(fl, -1)
    ch = torch.zeros_like(cl)
    ol, ll, of, lf = sfa().forward_dual(q, k, v, fl, cl, fh, ch, local.P, 2)
    torch.cuda.synchronize()
    assert (ol.float() - of.float()).abs().max().item() <= 2 ** -8
    assert torch.allclose(ll, lf, atol=1e-6, rtol=0)


def test_dual_ispa_workload_sampled():
    local, hist_w, full = WORKLOADS["lsemerge_local"], WORKLOADS["lsemerge_hist"], WORKLOADS["lsemerge_full"]
    rows = sample_rows(local, 256, seed=2, frames=(0,))
    _run(local, hist_w, full, 2, seed=0, rows=rows)


def test_dual_argument_checks():
    m = sfa()
    local, hist_w, _ = _branches(200, 128)
    q, k, v = (x.cuda() for x in workload_qkv(local, seed=1))
    fh, ch = gpu_sets(hist_w)
    fl, cl = gpu_sets(local, Amax=fh.shape[2])
    with pytest.raises(m.SfaError):
        m.forward_dual(q, k, v, fl, cl, fh, ch, local.P, 9)   # 2 * 9 > d / 8
    with pytest.raises(m.SfaError):
        m.forward_dual(q, k, v, fl, cl, fh, ch, local.P, 1, workspace=torch.empty(16, dtype=torch.uint8,
                                                                                     device="cuda"))


def test_dual_scheduled_ispa_workload_sampled():
    # n_split = 0 on the ISPA shape: the local lists one range per unit, the history lists
    # split as planned, longest ranges first
    local, hist_w = WORKLOADS["lsemerge_local"], WORKLOADS["lsemerge_hist"]
    full = WORKLOADS["lsemerge_full"]
    _run(local, hist_w, full, 0, seed=0, rows=sample_rows(local, 256, seed=3))
