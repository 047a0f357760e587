"""GPU LSE merge vs the merge oracle, and the ISPA dual-stream check end to end:
local branch + history branch through sfa_forward, merged by sfa_lse_merge, against
the oracle's full attention over the union of frames."""
import math

import numpy as np
import pytest
import torch

import oracle
from sfa_workloads import WORKLOADS, Workload, SetSpec, qkv, sample_rows

from gpu_helpers import check_sets_equal, compare, sfa

pytestmark = pytest.mark.gpu


def _bf16_round(x):
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rows", [1, 37, 4096, 100003])
def test_merge_kernel_vs_oracle(d, rows):
    rng = np.random.default_rng(rows + d)
    o1 = _bf16_round(rng.standard_normal((rows, d)).astype(np.float32))
    o2 = _bf16_round(rng.standard_normal((rows, d)).astype(np.float32))
    l1 = (rng.standard_normal(rows) * 5).astype(np.float32)
    l2 = (rng.standard_normal(rows) * 5).astype(np.float32)
    # empty branches: one side, the other side, both
    l1[::7] = -np.inf
    l2[::11] = -np.inf
    l1[::13] = -np.inf
    l2[::13] = -np.inf
    o, lse = sfa().lse_merge(o1.cuda(), torch.from_numpy(l1).cuda(), o2.cuda(), torch.from_numpy(l2).cuda())
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.lse_merge(o1.double().numpy(), l1, o2.double().numpy(), l2)
    # fp32 math on identical inputs and one round-to-nearest bf16 rounding of O: every
    # element within half a bf16 ulp (at most 2^-8 of its magnitude, 8 significant bits)
    # plus fp32 slack; far inside the parity bar
    o_g = o.float().cpu().numpy().astype(np.float64)
    bound = 2.0 ** -8 * np.abs(o_ref) * 1.001 + 1e-6
    assert (np.abs(o_g - o_ref) <= bound).all()
    compare(o_g, lse.cpu().numpy(), o_ref, l_ref, o_tol=bound.max(), lse_tol=1e-5)


def test_merge_in_place():
    rng = np.random.default_rng(0)
    rows, d = 3000, 128
    o1 = _bf16_round(rng.standard_normal((rows, d)).astype(np.float32))
    o2 = _bf16_round(rng.standard_normal((rows, d)).astype(np.float32))
    l1 = rng.standard_normal(rows).astype(np.float32)
    l2 = rng.standard_normal(rows).astype(np.float32)
    a, la = o1.cuda(), torch.from_numpy(l1).cuda()
    ref_o, ref_l = sfa().lse_merge(a.clone(), la.clone(), o2.cuda(), torch.from_numpy(l2).cuda())
    sfa().lse_merge(a, la, o2.cuda(), torch.from_numpy(l2).cuda(), out=a, lse=la)
    torch.cuda.synchronize()
    assert torch.equal(a, ref_o) and torch.equal(la, ref_l)


def _branches(P, d, H, seed, n_rows=None):
    wl, wh, wf = (WORKLOADS[n] for n in ("lsemerge_local", "lsemerge_hist", "lsemerge_full"))
    if P != wl.P or d != wl.d or H != wl.H:
        def resize(w):
            return Workload(w.name, B=1, H=H, Tq=w.Tq, Tkv=w.Tkv, q_off=w.q_off, P=P, d=d,
                            n_sink=w.n_sink, n_prev=w.n_prev, chunk_len=w.chunk_len, heads=w.heads[:H])
        wl, wh, wf = resize(wl), resize(wh), resize(wf)
    q, k, v = qkv(1, H, wl.Lq, wl.Lkv, d, seed=seed)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    outs = []
    osets = []
    for w in (wl, wh, wf):
        fr, cn, ofr, ocn = check_sets_equal(w)
        osets.append((ofr, ocn))
        outs.append(sfa().forward(qc, kc, vc, fr, cn, P))
    (o1, l1), (o2, l2), _ = outs
    om, lm = sfa().lse_merge(o1, l1, o2, l2)
    torch.cuda.synchronize()
    rows = None if n_rows is None else sample_rows(wf, n_rows, seed=seed)
    o_ref, l_ref = oracle.attention(q, k, v, *osets[2], P, 1 / math.sqrt(d), rows=rows)
    o_m = om.float().cpu().reshape(-1, d).numpy()
    l_m = lm.cpu().reshape(-1).numpy()
    if rows is not None:
        o_m, l_m = o_m[rows], l_m[rows]
    return compare(o_m, l_m, o_ref, l_ref)


def test_dual_stream_small_full():
    _branches(P=200, d=128, H=3, seed=1)


def test_dual_stream_lsemerge_sampled():
    _branches(P=1560, d=128, H=12, seed=0, n_rows=512)
