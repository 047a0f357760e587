"""Split-KV forward vs the float64 oracle (and vs the unsplit forward).

Every unit's key tiles are cut into n_split ranges that run as separate CTAs and are
merged by their LSE ("ISPA", §2.1); the result must meet the same bar as sfa_forward.
"""
import math

import numpy as np
import pytest
import torch

from sfa_workloads import SetSpec, WORKLOADS, Workload, sample_rows, workload_qkv

from gpu_helpers import check_sets_equal, compare, sfa
import oracle

pytestmark = pytest.mark.gpu

SMALL = {
    "lvsa_p200": Workload("lvsa_p200", B=1, H=3, Tq=12, Tkv=12, q_off=0, P=200, d=128,
                          C=6, W=3, T_per=4, heads=(SetSpec("lvsa"),) * 3),
    "stream_small": Workload("stream_small", B=1, H=5, Tq=2, Tkv=9, q_off=7, P=160, d=128,
                             n_sink=1, n_prev=2, chunk_len=2,
                             heads=(SetSpec("local"), SetSpec("anchor"), SetSpec("memory", (2, 4)),
                                    SetSpec("explicit", (0, 3, 5)), SetSpec("dense"))),
    "lvsa_d64": Workload("lvsa_d64", B=2, H=2, Tq=10, Tkv=10, q_off=0, P=136, d=64,
                         C=5, W=3, T_per=3, heads=(SetSpec("lvsa"),) * 2),
    "tiny_sinkwin": WORKLOADS["tiny_sinkwin"],
}


def _run(w, n_split, seed=1, rows=None, layout="bhld"):
    q, k, v = workload_qkv(w, seed=seed)
    fr, cn, ofr, ocn = check_sets_equal(w)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    out = None
    if layout == "blhd":
        out = torch.empty(w.B, w.Lq, w.H, w.d, dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = sfa().forward_split(qc, kc, vc, fr, cn, w.P, n_split, out=out, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_flat = o.float().cpu().contiguous().reshape(-1, w.d).numpy()
    l_flat = lse.cpu().reshape(-1).numpy()
    o_ref, l_ref = oracle.attention(q, k, v, ofr, ocn, w.P, 1 / math.sqrt(w.d), rows=rows)
    if rows is not None:
        o_flat, l_flat = o_flat[rows], l_flat[rows]
    return compare(o_flat, l_flat, o_ref, l_ref)


@pytest.mark.parametrize("name,n_split", [("lvsa_p200", 2), ("lvsa_p200", 3), ("stream_small", 4),
                                          ("lvsa_d64", 2), ("lvsa_d64", 8), ("tiny_sinkwin", 4)])
def test_split_small_full(name, n_split):
    # tiny_sinkwin has one key tile per unit, so most of its 4 ranges are empty
    _run(SMALL[name], n_split)


def test_split_strided_output():
    _run(SMALL["lvsa_d64"], 3, layout="blhd")


def test_split_matches_unsplit():
    w = SMALL["lvsa_p200"]
    q, k, v = (x.cuda() for x in workload_qkv(w, seed=4))
    fr, cn = __import__("gpu_helpers").gpu_sets(w)
    o1, l1 = sfa().forward(q, k, v, fr, cn, w.P)
    o2, l2 = sfa().forward_split(q, k, v, fr, cn, w.P, 4)
    o3, l3 = sfa().forward_split(q, k, v, fr, cn, w.P, 1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o3) and torch.equal(l1, l3)
    # partial O is rounded to bf16 once more before the merge: within a few bf16 ulps
    assert (o1.float() - o2.float()).abs().max().item() < 2e-3
    assert (l1 - l2).abs().max().item() < 1e-5


@pytest.mark.parametrize("name,n_split", [("stream", 4), ("lsemerge_hist", 8)])
def test_split_full_size_sampled(name, n_split):
    w = WORKLOADS[name]
    _run(w, n_split, seed=0, rows=sample_rows(w, 256, seed=1))


# ---------------------------------------------------------------------------- scheduled
# n_split = 0: the library picks the number of ranges and a one-CTA kernel orders the
# CTAs longest range first.  The result must equal forward_split with the planned number
# of ranges bit for bit (same ranges, same merge order), which also shows that every
# (unit, range) ran exactly once, and meet the oracle bar.

def _planned(w, q, k, v, fr, cn):
    m = sfa()
    desc = m.attn_desc(q, k, v, torch.empty_like(q), w.P, fr.shape[2])
    return m.split_plan(desc)[0]


@pytest.mark.parametrize("name", ["lvsa_p200", "stream_small", "lvsa_d64", "tiny_sinkwin"])
def test_scheduled_small_full(name):
    w = SMALL[name]
    _run(w, 0)
    q, k, v = (x.cuda() for x in workload_qkv(w, seed=1))
    fr, cn = __import__("gpu_helpers").gpu_sets(w)
    kp = _planned(w, q, k, v, fr, cn)
    o0, l0 = sfa().forward_split(q, k, v, fr, cn, w.P, 0)
    ok, lk = sfa().forward_split(q, k, v, fr, cn, w.P, kp)
    torch.cuda.synchronize()
    assert torch.equal(o0, ok) and torch.equal(l0, lk)


@pytest.mark.parametrize("name", ["stream", "lsemerge_hist"])
def test_scheduled_full_size(name):
    w = WORKLOADS[name]
    _run(w, 0, seed=0, rows=sample_rows(w, 256, seed=2, frames=(0,)))
    q, k, v = (x.cuda() for x in workload_qkv(w, seed=0))
    fr, cn = __import__("gpu_helpers").gpu_sets(w)
    kp = _planned(w, q, k, v, fr, cn)
    assert kp > 1  # a sub-wave grid is split
    o0, l0 = sfa().forward_split(q, k, v, fr, cn, w.P, 0)
    ok, lk = sfa().forward_split(q, k, v, fr, cn, w.P, kp)
    torch.cuda.synchronize()
    assert torch.equal(o0, ok) and torch.equal(l0, lk)


def test_scheduled_many_waves_keeps_one_range():
    # 1280 units (more than 8 waves of 148 SMs): one range per unit, the output written
    # directly; identical to the plain forward
    w = Workload("waves", B=2, H=8, Tq=40, Tkv=40, q_off=0, P=512, d=128, C=5, W=3, T_per=4,
                 heads=(SetSpec("lvsa"),) * 8)
    q, k, v = (x.cuda() for x in workload_qkv(w, seed=3))
    fr, cn = __import__("gpu_helpers").gpu_sets(w)
    assert _planned(w, q, k, v, fr, cn) == 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1 = sfa().forward(q, k, v, fr, cn, w.P)
    o0, l0 = sfa().forward_split(q, k, v, fr, cn, w.P, 0, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(o0, o1) and torch.equal(l0, l1)


def test_scheduled_bad_list_is_reported():
    w = SMALL["stream_small"]
    q, k, v = (x.cuda() for x in workload_qkv(w, seed=1))
    fr, cn = __import__("gpu_helpers").gpu_sets(w)
    bad = fr.clone()
    bad[1, 0, 0] = w.Tkv  # out of range
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa().forward_split(q, k, v, bad, cn, w.P, 0, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == sfa().SFA_ERR_BAD_SET
