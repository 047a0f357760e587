"""Paged key/value caches: K/V read through a per-head logical-frame -> slot table.

"Head Forcing", §2: each head keeps its own cache of frames.  The physical caches here
hold the logical frames at shuffled slots (some consecutive, so runs span several
slots) and NaN in every unused slot: rows past a run's end must never reach O.  The
oracle sees the logical K/V (an input rearrangement only).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sfa_workloads import SetSpec, Workload, workload_qkv

from gpu_helpers import check_sets_equal, compare, gpu_sets, sfa

pytestmark = pytest.mark.gpu

W = Workload("paged", B=2, H=5, Tq=2, Tkv=9, q_off=7, P=200, d=128, n_sink=1, n_prev=2, chunk_len=2,
             heads=(SetSpec("local"), SetSpec("anchor"), SetSpec("memory", (2, 4)),
                    SetSpec("explicit", (0, 3, 5)), SetSpec("dense")))


def _slot_table(H, T, n_slots, seed):
    # per head: frames placed in shuffled blocks of 1-3 consecutive slots
    rng = np.random.default_rng(seed)
    table = np.zeros((H, T), np.int32)
    for h in range(H):
        free = list(range(n_slots))
        f = 0
        while f < T:
            run = min(int(rng.integers(1, 4)), T - f)
            starts = [s for s in free if all(s + i in free for i in range(run))]
            s0 = int(rng.choice(starts))
            for i in range(run):
                table[h, f + i] = s0 + i
                free.remove(s0 + i)
            f += run
    return table


def _paged_caches(k, v, table, n_slots, P):
    B, H, _, d = k.shape
    kc = torch.full((B, H, n_slots * P, d), float("nan"), dtype=torch.bfloat16)
    vc = torch.full((B, H, n_slots * P, d), float("nan"), dtype=torch.bfloat16)
    for h in range(H):
        for f in range(table.shape[1]):
            s = int(table[h, f])
            kc[:, h, s * P:(s + 1) * P] = k[:, h, f * P:(f + 1) * P]
            vc[:, h, s * P:(s + 1) * P] = v[:, h, f * P:(f + 1) * P]
    return kc, vc


@pytest.mark.parametrize("seed", [0, 1])
def test_paged_matches_oracle_with_nan_in_unused_slots(seed):
    w = W
    n_slots = w.Tkv + 6
    q, k, v = workload_qkv(w, seed=seed)
    table = _slot_table(w.H, w.Tkv, n_slots, seed)
    kc, vc = _paged_caches(k, v, table, n_slots, w.P)
    fr, cn, ofr, ocn = check_sets_equal(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = sfa().forward_paged(q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(table).cuda(), fr, cn, w.P,
                                 w.Tkv, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_ref, l_ref = oracle.attention(q, k, v, ofr, ocn, w.P, 1 / math.sqrt(w.d))
    compare(o.float().cpu().reshape(-1, w.d).numpy(), lse.cpu().reshape(-1).numpy(), o_ref, l_ref)


def test_identity_table_equals_plain_forward():
    w = W
    q, k, v = (x.cuda() for x in workload_qkv(w, seed=3))
    fr, cn = gpu_sets(w)
    table = torch.arange(w.Tkv, dtype=torch.int32).repeat(w.H, 1).contiguous().cuda()
    o1, l1 = sfa().forward(q, k, v, fr, cn, w.P)
    o2, l2 = sfa().forward_paged(q, k, v, table, fr, cn, w.P, w.Tkv)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_slot_out_of_range_reported():
    w = W
    q, k, v = (x.cuda() for x in workload_qkv(w, seed=4))
    fr, cn = gpu_sets(w)
    table = torch.arange(w.Tkv, dtype=torch.int32).repeat(w.H, 1).contiguous()
    table[2, 8] = w.Tkv + 3          # beyond n_slots = T_kv for head 2's own frame 8
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa().forward_paged(q, k, v, table.cuda(), fr, cn, w.P, w.Tkv, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == sfa().SFA_ERR_BAD_SET


def test_plain_forward_ignores_non_finite_unattended_frames():
    # frame 1 follows attended frame 0 in memory but is not attended; with P = 200 the
    # last key tile of frame 0 holds 72 keys, so P V would touch rows of frame 1
    B, H, Tq, Tkv, P, d = 1, 2, 2, 4, 200, 128
    from sfa_workloads import qkv
    q, k, v = qkv(B, H, Tq * P, Tkv * P, d, seed=8)
    k[:, :, P:2 * P] = float("nan")
    v[:, :, P:2 * P] = float("inf")
    frames = np.array([[[0, 2], [0, 3]], [[0, -1], [2, 3]]], np.int32)
    counts = np.array([[2, 2], [1, 2]], np.int32)
    o, lse = sfa().forward(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(frames).cuda(),
                           torch.from_numpy(counts).cuda(), P)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q, k, v, frames, counts, P, 1 / math.sqrt(d))
    compare(o.float().cpu().reshape(-1, d).numpy(), lse.cpu().reshape(-1).numpy(), o_ref, l_ref)
