"""Pins of the HSA oracle ("Resumen Técnico: LIGHT FORCING", §2.2) to independent facts:
a hand-worked selection, closed forms of the pooling, brute-force pooling and attention
with math.fsum, selection invariants, and the full-selection case, which must equal the
frame-list attention oracle (itself pinned to library SDPA)."""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import hsa

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    vals = {}
    for line in open(os.path.join(HERE, "golden", "hsa_select_hand.txt")):
        line = line.split("#")[0].strip()
        if line:
            key, *rest = line.split()
            vals[key] = [float(x) for x in rest]
    return vals


def test_hand_worked_selection():
    g = _golden()
    P, T = int(g["P"][0]), int(g["T_kv"][0])
    nb = hsa.n_key_blocks(P)
    assert nb == 3
    d = 4
    qbar = np.zeros(d)
    qbar[0] = 1.0
    kf = np.zeros((T, d))
    kf[:, 0] = g["frame_scores"]
    kb = np.zeros((T, nb, d))
    kb[:, :, 0] = np.asarray(g["block_scores"]).reshape(T, nb)
    got = hsa.select_blocks(qbar, kf, kb, int(g["t"][0]), P=P, T_kv=T, q_off=int(g["q_off"][0]),
                            chunk_len=int(g["chunk_len"][0]), n_prev=int(g["n_prev"][0]),
                            n_sink=int(g["n_sink"][0]), k_frames=int(g["k_frames"][0]),
                            k_blocks=int(g["k_blocks"][0]))
    assert got == [int(x) for x in g["expected"]]


def test_top_k_ties_and_overflow():
    assert hsa.top_k([5, 3, 9, 1], [1.0, 2.0, 2.0, 0.5], 2) == [3, 9]
    assert hsa.top_k([5, 3, 9], [1.0, 1.0, 1.0], 2) == [3, 5]      # equal scores: smaller id
    assert hsa.top_k([4, 2], [0.1, 0.2], 10) == [2, 4]             # k > candidates: all
    assert hsa.top_k([], [], 3) == []


def test_pooling_closed_forms():
    # every token of key block g holds the value g: block means are g, a frame mean is
    # the token-weighted mean of its blocks (P = 300: blocks of 128, 128, 44 tokens)
    B, H, T, P, d = 1, 2, 3, 300, 5
    nb = hsa.n_key_blocks(P)
    k = np.zeros((B, H, T * P, d))
    for f in range(T):
        for b in range(nb):
            lo, hi = hsa.block_tokens(f * nb + b, P)
            k[:, :, lo:hi] = f * nb + b
    kf, kb = hsa.pool_keys(k, P)
    for f in range(T):
        for b in range(nb):
            assert np.all(kb[:, :, f, b] == f * nb + b)
        want = (128 * (3 * f) + 128 * (3 * f + 1) + 44 * (3 * f + 2)) / 300
        assert np.allclose(kf[:, :, f], want, rtol=0, atol=1e-12)
    # query blocks of 256 rows: P = 300 -> rows [0, 256) and [256, 300)
    q = np.zeros((B, H, 2 * P, d))
    q[:, :, :256] = 1.0
    q[:, :, 256:300] = 3.0
    q[:, :, 300:] = -2.0
    qb = hsa.pool_queries(q, P)
    assert qb.shape == (B, H, 2, 2, d)
    assert np.all(qb[:, :, 0, 0] == 1.0) and np.all(qb[:, :, 0, 1] == 3.0) and np.all(qb[:, :, 1] == -2.0)


def test_pooling_brute_force():
    rng = np.random.default_rng(3)
    B, H, T, P, d = 1, 1, 2, 200, 3
    k = rng.standard_normal((B, H, T * P, d))
    kf, kb = hsa.pool_keys(k, P)
    for f in range(T):
        for j in range(d):
            assert abs(kf[0, 0, f, j] - math.fsum(k[0, 0, f * P:(f + 1) * P, j]) / P) < 1e-13
        for b in range(hsa.n_key_blocks(P)):
            lo, hi = hsa.block_tokens(f * hsa.n_key_blocks(P) + b, P)
            for j in range(d):
                assert abs(kb[0, 0, f, b, j] - math.fsum(k[0, 0, lo:hi, j]) / (hi - lo)) < 1e-13


def test_frame_roles():
    kw = dict(T_kv=24, q_off=21, chunk_len=3, n_prev=3, n_sink=1)
    for t in range(3):
        assert hsa.always_frames(t, **kw) == [0, 18, 19, 20, 21, 22, 23]
        assert hsa.history_frames(t, **kw) == list(range(1, 18))
    # query frame 1 of chunk_len 1: chunk {22}, window {21}, sink {0}; history 1..20
    kw1 = dict(T_kv=24, q_off=21, chunk_len=1, n_prev=1, n_sink=1)
    assert hsa.always_frames(1, **kw1) == [0, 21, 22]
    assert hsa.history_frames(1, **kw1) == list(range(1, 21))


def _small(seed=0, P=200, k_frames=2, k_blocks=3):
    from sfa_workloads import qkv_structured
    B, H, Tq, Tkv, d = 1, 2, 2, 9, 16
    q, k, v = qkv_structured(B, H, Tq, Tkv, P, d, seed=seed)
    kw = dict(P=P, T_kv=Tkv, q_off=7, chunk_len=2, n_prev=2, n_sink=1, k_frames=k_frames, k_blocks=k_blocks)
    return q, k, v, kw


def test_selection_invariants():
    q, k, v, kw = _small()
    lists, counts = hsa.build_block_lists(q.float().numpy(), k.float().numpy(), **kw)
    P, nb = kw["P"], hsa.n_key_blocks(kw["P"])
    fw = {x: kw[x] for x in ("T_kv", "q_off", "chunk_len", "n_prev", "n_sink")}
    kf, kb = hsa.pool_keys(k.float().numpy(), P)
    qb = hsa.pool_queries(q.float().numpy(), P)
    B, H, Tq, nq = counts.shape
    for b in range(B):
        for h in range(H):
            for t in range(Tq):
                always = hsa.always_frames(t, **fw)
                hist = hsa.history_frames(t, **fw)
                for i in range(nq):
                    got = lists[b, h, t, i, :counts[b, h, t, i]].tolist()
                    assert got == sorted(set(got)) and all(x >= 0 for x in got)
                    assert all(f * nb + bb in got for f in always for bb in range(nb))
                    picked = [g for g in got if g // nb not in always]
                    frames = sorted({g // nb for g in picked})
                    n_sel = min(kw["k_frames"], len(hist))
                    assert len(picked) == min(kw["k_blocks"], n_sel * nb)
                    # the picked blocks lie in the n_sel best-scored history frames
                    fs = sorted(hist, key=lambda f: (-float(np.dot(qb[b, h, t, i], kf[b, h, f])), f))[:n_sel]
                    assert set(frames) <= set(fs)
                    # and no unpicked block of those frames scores higher than a picked one
                    sc = {g: float(np.dot(qb[b, h, t, i], kb[b, h, g // nb, g % nb])) for f in fs for g in
                          range(f * nb, f * nb + nb)}
                    if picked:
                        worst = min(sc[g] for g in picked)
                        assert all(sc[g] <= worst for g in sc if g not in picked)


def test_full_selection_equals_frame_attention():
    # every history frame and every block kept: the attended set of every query block is
    # all frames before the end of the chunk, so the result must equal the frame-list
    # oracle (pinned to SDPA) on that dense-over-history list
    q, k, v, kw = _small(seed=1, k_frames=99, k_blocks=999)
    lists, counts = hsa.build_block_lists(q.float().numpy(), k.float().numpy(), **kw)
    P = kw["P"]
    scale = 1 / math.sqrt(q.shape[-1])
    o, lse = hsa.attention_blocks(q.float().numpy(), k.float().numpy(), v.float().numpy(), lists, counts, P, scale)
    H, Tq, Tkv = q.shape[1], q.shape[2] // P, kw["T_kv"]
    frames = np.full((H, Tq, Tkv), -1, np.int32)
    cnts = np.zeros((H, Tq), np.int32)
    for t in range(Tq):
        c = t + kw["q_off"]
        end = min(c - c % kw["chunk_len"] + kw["chunk_len"], Tkv)
        frames[:, t, :end] = np.arange(end)
        cnts[:, t] = end
    o_ref, l_ref = oracle.attention(q, k, v, frames, cnts, P, scale)
    assert np.abs(o.reshape(-1, q.shape[-1]) - o_ref).max() < 1e-12
    assert np.abs(lse.reshape(-1) - l_ref).max() < 1e-12


def test_attention_blocks_brute_force_and_rows():
    # a hand-picked list per query block; rows checked with a fsum softmax
    from sfa_workloads import qkv
    P, d = 300, 4
    q, k, v = qkv(1, 1, P, 3 * P, d, seed=5)
    nb = hsa.n_key_blocks(P)
    lists = np.full((1, 1, 1, 2, 5), -1, np.int32)
    counts = np.zeros((1, 1, 1, 2), np.int32)
    lists[0, 0, 0, 0, :3] = [0, 4, 8]          # query rows [0, 256)
    counts[0, 0, 0, 0] = 3
    lists[0, 0, 0, 1, :2] = [2, 3]             # rows [256, 300): block 2 (44 tokens) + block 3
    counts[0, 0, 0, 1] = 2
    qf, kf_, vf = (x.float().numpy().astype(np.float64) for x in (q, k, v))
    rows = np.asarray([0, 100, 255, 256, 299])
    o, lse = hsa.attention_blocks(qf, kf_, vf, lists, counts, P, 0.5, rows=rows)
    for n, r in enumerate(rows):
        i = r // 256
        keys = [j for g in lists[0, 0, 0, i, :counts[0, 0, 0, i]] for j in range(*hsa.block_tokens(int(g), P))]
        s = [0.5 * math.fsum(qf[0, 0, r] * kf_[0, 0, j]) for j in keys]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        l = math.fsum(e)
        assert abs(lse[n] - (m + math.log(l))) < 1e-12
        for c in range(d):
            assert abs(o[n, c] - math.fsum(e[a] * vf[0, 0, keys[a], c] for a in range(len(keys))) / l) < 1e-12
    assert nb == 3
    # the whole-array form agrees with the per-row form
    O, L = hsa.attention_blocks(qf, kf_, vf, lists, counts, P, 0.5)
    assert np.abs(O[0, 0, rows] - o).max() < 1e-13 and np.abs(L[0, 0, rows] - lse).max() < 1e-13


def test_planted_mistakes_are_caught():
    # a plausible slip in the selection (ranking by the smallest scores) breaks the pin
    g = _golden()
    wrong = hsa.top_k([1, 2, 3, 4], [-x for x in g["frame_scores"][1:5]], 2)
    assert wrong != [2, 4]


def test_structured_inputs_give_clear_selections():
    # the synthetic offsets make the pooled keys distinct: on the small cases the
    # oracle's k-th and (k+1)-th frame scores are far apart for nearly every query block
    from sfa_workloads import Workload, SetSpec, qkv_structured
    w = Workload("hsa_p300_d64", B=1, H=3, Tq=3, Tkv=12, q_off=9, P=300, d=64, n_sink=2, n_prev=1, chunk_len=3,
                 k_frames=3, k_blocks=5, heads=(SetSpec("hsa"),) * 3)
    q, k, _ = qkv_structured(w.B, w.H, w.Tq, w.Tkv, w.P, w.d, seed=2)
    kf, _ = hsa.pool_keys(k.float().numpy(), w.P)
    qb = hsa.pool_queries(q.float().numpy(), w.P)
    fw = dict(T_kv=w.Tkv, q_off=w.q_off, chunk_len=w.chunk_len, n_prev=w.n_prev, n_sink=w.n_sink)
    gaps = []
    for h in range(w.H):
        for t in range(w.Tq):
            hist = hsa.history_frames(t, **fw)
            for i in range(qb.shape[3]):
                s = sorted((float(np.dot(qb[0, h, t, i], kf[0, h, f])) for f in hist), reverse=True)
                if len(s) > w.k_frames:
                    gaps.append(s[w.k_frames - 1] - s[w.k_frames])
    assert min(gaps) > 1e-3
