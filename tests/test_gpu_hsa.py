"""Hierarchical sparse attention on the GPU against the oracle ("Resumen Técnico: LIGHT
FORCING", §2.2): the block lists of sfa_hsa_select against oracle.hsa's selection, and
sfa_forward_blocks against oracle.hsa.attention_blocks on the oracle's own lists.

Selection is an integer result decided by floating-point scores: the GPU ranks fp32
means and dot products, the oracle fp64 ones.  Lists must be identical wherever the
oracle's scores separate the kept from the dropped candidates by more than SCORE_EPS (a
bound far above the fp32 error of a mean over <= 1560 values and a d-term dot product);
where they do not, the GPU list must still be a valid selection under the fp64 scores
within SCORE_EPS.
"""
import math

import numpy as np
import pytest
import torch

from oracle import hsa
from sfa_workloads import WORKLOADS, Workload, SetSpec, qkv, sample_rows, workload_qkv

from gpu_helpers import compare, sfa

pytestmark = pytest.mark.gpu

SCORE_EPS = 1e-4


def _params(w):
    return sfa().set_params(T_kv=w.Tkv, Tq=w.Tq, q_off=w.q_off, n_sink=w.n_sink, n_prev=w.n_prev,
                            chunk_len=w.chunk_len)


def _kw(w):
    return dict(P=w.P, T_kv=w.Tkv, q_off=w.q_off, chunk_len=w.chunk_len, n_prev=w.n_prev, n_sink=w.n_sink,
                k_frames=w.k_frames, k_blocks=w.k_blocks)


def _valid_top(scores: dict, chosen: set, k: int) -> bool:
    """chosen is a top-k set of the candidates in scores within SCORE_EPS: it has
    min(k, n) members and none of the others scores more than SCORE_EPS above any of them."""
    if len(chosen) != min(k, len(scores)) or not chosen <= set(scores):
        return False
    rest = [s for i, s in scores.items() if i not in chosen]
    return not chosen or not rest or min(scores[i] for i in chosen) >= max(rest) - SCORE_EPS


def _frame_sets(fs: dict, n_sel: int, must: set):
    """Every top-n_sel frame set within SCORE_EPS (fs: frame -> fp64 score) that holds
    the frames in must.  A frame scoring more than SCORE_EPS above the (n_sel+1)-th score
    is in every such set, one scoring more than SCORE_EPS below the n_sel-th in none."""
    from itertools import combinations
    order = sorted(fs.values(), reverse=True)
    if n_sel == 0:
        return [set()]
    hi = order[n_sel] if n_sel < len(order) else -math.inf
    lo = order[n_sel - 1]
    fixed = {f for f, s in fs.items() if s > hi + SCORE_EPS}
    band = [f for f, s in fs.items() if f not in fixed and s >= lo - SCORE_EPS]
    out = []
    for extra in combinations(sorted(band), n_sel - len(fixed)):
        F = fixed | set(extra)
        if must <= F and _valid_top(fs, F, n_sel):
            out.append(F)
    return out


def _check_selection(w, q, k, lists_gpu, counts_gpu):
    """Lists identical to the oracle's wherever the fp64 scores decide clearly; elsewhere
    the GPU list must be a valid selection within SCORE_EPS: the always-attended blocks,
    a top-k_frames set of the history frames, and a top-k_blocks set of those frames'
    blocks (a near tie at either level is the only way two valid lists can differ).
    Returns the number of lists that differ."""
    kw = _kw(w)
    Amax = lists_gpu.shape[-1]
    o_lists, o_counts = hsa.build_block_lists(q.float().numpy(), k.float().numpy(), Bmax=Amax, **kw)
    kf, kb = hsa.pool_keys(k.float().numpy(), w.P)
    qb = hsa.pool_queries(q.float().numpy(), w.P)
    nb = hsa.n_key_blocks(w.P)
    fw = {x: kw[x] for x in ("T_kv", "q_off", "chunk_len", "n_prev", "n_sink")}
    n_close = 0
    B, H, Tq, nq = o_counts.shape
    for b in range(B):
        for h in range(H):
            for t in range(Tq):
                always = hsa.always_frames(t, **fw)
                hist = hsa.history_frames(t, **fw)
                for i in range(nq):
                    got = lists_gpu[b, h, t, i, :counts_gpu[b, h, t, i]].tolist()
                    assert all(x == -1 for x in lists_gpu[b, h, t, i, counts_gpu[b, h, t, i]:])
                    want = o_lists[b, h, t, i, :o_counts[b, h, t, i]].tolist()
                    if got == want:
                        continue
                    n_close += 1
                    assert got == sorted(set(got))
                    assert all(f * nb + x in got for f in always for x in range(nb))
                    picked = [g for g in got if g // nb not in always]
                    fs = {f: float(np.dot(qb[b, h, t, i], kf[b, h, f])) for f in hist}
                    n_sel = min(w.k_frames, len(hist))
                    ok = False
                    for F in _frame_sets(fs, n_sel, {g // nb for g in picked}):
                        bs = {f * nb + x: float(np.dot(qb[b, h, t, i], kb[b, h, f, x])) for f in F for x in range(nb)}
                        if _valid_top(bs, set(picked), w.k_blocks):
                            ok = True
                            break
                    assert ok, f"list ({b}, {h}, {t}, {i}) is not a valid selection: {got} (oracle {want})"
    return n_close


SMALL = [
    Workload("hsa_p200", B=2, H=2, Tq=2, Tkv=9, q_off=7, P=200, d=128, n_sink=1, n_prev=2, chunk_len=2,
             k_frames=2, k_blocks=3, heads=(SetSpec("hsa"),) * 2),
    Workload("hsa_p300_d64", B=1, H=3, Tq=3, Tkv=12, q_off=9, P=300, d=64, n_sink=2, n_prev=1, chunk_len=3,
             k_frames=3, k_blocks=5, heads=(SetSpec("hsa"),) * 3),
    Workload("hsa_p1", B=1, H=2, Tq=2, Tkv=10, q_off=8, P=1, d=128, n_sink=0, n_prev=1, chunk_len=1,
             k_frames=4, k_blocks=2, heads=(SetSpec("hsa"),) * 2),
    Workload("hsa_nohist", B=1, H=1, Tq=2, Tkv=4, q_off=2, P=136, d=128, n_sink=1, n_prev=1, chunk_len=2,
             k_frames=3, k_blocks=4, heads=(SetSpec("hsa"),)),
    Workload("hsa_k0", B=1, H=2, Tq=1, Tkv=8, q_off=7, P=260, d=128, n_sink=1, n_prev=1, chunk_len=1,
             k_frames=0, k_blocks=6, heads=(SetSpec("hsa"),) * 2),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_selection_matches_oracle(w):
    q, k, v = workload_qkv(w, seed=2)
    blocks, counts = sfa().hsa_select(q.cuda(), k.cuda(), _params(w), w.k_frames, w.k_blocks)
    torch.cuda.synchronize()
    n_close = _check_selection(w, q, k, blocks.cpu().numpy(), counts.cpu().numpy())
    assert n_close == 0, f"{n_close} lists decided by near-ties"


def test_selection_exact_ties_go_to_the_smaller_id():
    # every history frame a copy of frame 1: all frame scores tie (the first k_frames
    # history frames win) and every block ties with its copies in the other frames (the
    # copies in the earliest frames win); pooling is per position inside a frame, so the
    # GPU's fp32 scores tie exactly too.  The lists must equal the oracle's.
    w = Workload("hsa_ties", B=1, H=2, Tq=2, Tkv=11, q_off=9, P=300, d=128, n_sink=1, n_prev=1, chunk_len=2,
                 k_frames=3, k_blocks=4, heads=(SetSpec("hsa"),) * 2)
    q, k, v = workload_qkv(w, seed=4)
    k = k.clone()
    for f in range(2, 8):
        k[:, :, f * w.P:(f + 1) * w.P] = k[:, :, w.P:2 * w.P]
    blocks, counts = sfa().hsa_select(q.cuda(), k.cuda(), _params(w), w.k_frames, w.k_blocks)
    torch.cuda.synchronize()
    lists, cnts = hsa.build_block_lists(q.float().numpy(), k.float().numpy(), Bmax=blocks.shape[-1], **_kw(w))
    assert np.array_equal(blocks.cpu().numpy(), lists) and np.array_equal(counts.cpu().numpy(), cnts)


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_forward_blocks_matches_oracle_full_rows(w):
    q, k, v = workload_qkv(w, seed=3)
    Amax = sfa().hsa_max_count(_params(w), w.P, w.k_frames, w.k_blocks)
    lists, counts = hsa.build_block_lists(q.float().numpy(), k.float().numpy(), Bmax=Amax, **_kw(w))
    scale = 1 / math.sqrt(w.d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = sfa().forward_blocks(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(lists).cuda(),
                                  torch.from_numpy(counts).cuda(), w.P, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_ref, l_ref = hsa.attention_blocks(q.float().numpy(), k.float().numpy(), v.float().numpy(), lists, counts,
                                        w.P, scale)
    compare(o.float().cpu().reshape(-1, w.d).numpy(), lse.cpu().reshape(-1).numpy(), o_ref.reshape(-1, w.d),
            l_ref.reshape(-1))


def test_whole_frame_block_lists_equal_frame_lists():
    # lists naming every block of some frames attend to exactly those frames' tokens
    w = Workload("frames", B=1, H=2, Tq=2, Tkv=6, q_off=0, P=200, d=128, heads=(SetSpec("explicit"),) * 2)
    q, k, v = (x.cuda() for x in qkv(w.B, w.H, w.Lq, w.Lkv, w.d, seed=6))
    frame_sets = [[0, 2, 3], [1, 5]]
    nb = hsa.n_key_blocks(w.P)
    nq = hsa.n_query_blocks(w.P)
    frames = torch.full((w.H, w.Tq, 3), -1, dtype=torch.int32)
    fcounts = torch.zeros((w.H, w.Tq), dtype=torch.int32)
    blocks = torch.full((w.B, w.H, w.Tq, nq, 3 * nb), -1, dtype=torch.int32)
    bcounts = torch.zeros((w.B, w.H, w.Tq, nq), dtype=torch.int32)
    for h in range(w.H):
        for t in range(w.Tq):
            fs = frame_sets[(h + t) % 2]
            frames[h, t, :len(fs)] = torch.tensor(fs)
            fcounts[h, t] = len(fs)
            ids = [f * nb + x for f in fs for x in range(nb)]
            blocks[:, h, t, :, :len(ids)] = torch.tensor(ids, dtype=torch.int32)
            bcounts[:, h, t, :] = len(ids)
    o1, l1 = sfa().forward(q, k, v, frames.cuda(), fcounts.cuda(), w.P)
    o2, l2 = sfa().forward_blocks(q, k, v, blocks.cuda(), bcounts.cuda(), w.P)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_block_list_reported():
    w = SMALL[0]
    q, k, v = (x.cuda() for x in workload_qkv(w, seed=1))
    Amax = sfa().hsa_max_count(_params(w), w.P, w.k_frames, w.k_blocks)
    blocks, counts = sfa().hsa_select(q, k, _params(w), w.k_frames, w.k_blocks, Amax=Amax)
    bad = blocks.clone()
    bad[0, 1, 1, 0, 0] = w.Tkv * hsa.n_key_blocks(w.P)  # one past the last block
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa().forward_blocks(q, k, v, bad, counts, w.P, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == sfa().SFA_ERR_BAD_SET


def test_hsa_workload_selection_and_sampled_attention():
    w = WORKLOADS["hsa"]
    q, k, v = workload_qkv(w, seed=0)
    blocks, counts = sfa().hsa_select(q.cuda(), k.cuda(), _params(w), w.k_frames, w.k_blocks)
    torch.cuda.synchronize()
    n_close = _check_selection(w, q, k, blocks.cpu().numpy(), counts.cpu().numpy())
    print(f"hsa workload: {n_close} of {counts.numel()} lists differ from the oracle's, each a valid "
          f"selection within a near tie")
    # attention on the oracle's lists, sampled rows (all rows of query frame 0, 256 per head)
    Amax = blocks.shape[-1]
    lists, cnts = hsa.build_block_lists(q.float().numpy(), k.float().numpy(), Bmax=Amax, **_kw(w))
    o, lse = sfa().forward_blocks(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(lists).cuda(),
                                  torch.from_numpy(cnts).cuda(), w.P)
    torch.cuda.synchronize()
    rows = sample_rows(w, 256, seed=1, frames=(0,))
    o_ref, l_ref = hsa.attention_blocks(q.float().numpy(), k.float().numpy(), v.float().numpy(), lists, cnts,
                                        w.P, 1 / math.sqrt(w.d), rows=rows)
    compare(o.float().cpu().reshape(-1, w.d).numpy()[rows], lse.cpu().reshape(-1).numpy()[rows], o_ref, l_ref)


@pytest.mark.parametrize("n_split", [2, 4, 0])
def test_forward_blocks_split_matches_oracle(n_split):
    w = SMALL[0]
    q, k, v = workload_qkv(w, seed=5)
    Amax = sfa().hsa_max_count(_params(w), w.P, w.k_frames, w.k_blocks)
    lists, counts = hsa.build_block_lists(q.float().numpy(), k.float().numpy(), Bmax=Amax, **_kw(w))
    o, lse = sfa().forward_blocks(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(lists).cuda(),
                                  torch.from_numpy(counts).cuda(), w.P, n_split=n_split)
    torch.cuda.synchronize()
    o_ref, l_ref = hsa.attention_blocks(q.float().numpy(), k.float().numpy(), v.float().numpy(), lists, counts,
                                        w.P, 1 / math.sqrt(w.d))
    compare(o.float().cpu().reshape(-1, w.d).numpy(), lse.cpu().reshape(-1).numpy(), o_ref.reshape(-1, w.d),
            l_ref.reshape(-1))


def test_forward_blocks_scheduled_workload_sampled():
    # n_split = 0 on the hsa workload (252 units of uneven block lists)
    w = WORKLOADS["hsa"]
    q, k, v = workload_qkv(w, seed=0)
    Amax = sfa().hsa_max_count(_params(w), w.P, w.k_frames, w.k_blocks)
    lists, cnts = hsa.build_block_lists(q.float().numpy(), k.float().numpy(), Bmax=Amax, **_kw(w))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = sfa().forward_blocks(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(lists).cuda(),
                                  torch.from_numpy(cnts).cuda(), w.P, n_split=0, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    rows = sample_rows(w, 256, seed=4, frames=(2,))
    o_ref, l_ref = hsa.attention_blocks(q.float().numpy(), k.float().numpy(), v.float().numpy(), lists, cnts,
                                        w.P, 1 / math.sqrt(w.d), rows=rows)
    compare(o.float().cpu().reshape(-1, w.d).numpy()[rows], lse.cpu().reshape(-1).numpy()[rows], o_ref, l_ref)


@pytest.mark.parametrize("w", SMALL + [WORKLOADS["hsa"]], ids=[w.name for w in SMALL] + ["hsa"])
def test_pooled_keys_reused_equal_full_selection(w):
    # keys pooled once (sfa_hsa_pool_keys), then two selections with different queries
    # (sfa_hsa_select_pooled) give the lists of full selections, bit for bit
    m = sfa()
    q, k, _ = (x.cuda() for x in workload_qkv(w, seed=8))
    q2 = torch.flip(q, dims=[2]).contiguous()
    Amax = m.hsa_max_count(_params(w), w.P, w.k_frames, w.k_blocks)
    ws = torch.empty(m.hsa_workspace_bytes(q, k, w.P, Amax), dtype=torch.uint8, device="cuda")
    m.hsa_pool_keys(k, q, w.P, ws, Amax)
    for qq in (q, q2):
        b1, c1 = m.hsa_select_pooled(qq, k, _params(w), w.k_frames, w.k_blocks, ws, Amax=Amax)
        b0, c0 = m.hsa_select(qq, k, _params(w), w.k_frames, w.k_blocks, Amax=Amax)
        torch.cuda.synchronize()
        assert torch.equal(b0, b1) and torch.equal(c0, c1)
