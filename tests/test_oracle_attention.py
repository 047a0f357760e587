"""Pins for the float64 attention oracle (CPU only).

Each check ties the oracle to something other than itself:
  * A(t) = every frame is textbook attention ("LVSA", §2 Mecanismo Central: A(t)
    replaces the full set {0..T-1}) -> library SDPA in float64.
  * A(t) restricted -> library SDPA over the gathered key tokens of A(t).
  * A(t) = {t} -> per-frame bidirectional attention ("ARL2", §2.1 intra-frame branch).
  * LSE -> library logsumexp of the scaled scores ("ISPA", §2.1: LSE state).
  * closed forms: Q = 0, constant V, key shift invariance, key permutation invariance.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import sets as S
from sfa_workloads import WORKLOADS, qkv, workload_qkv


def _sdpa64(q, k, v, scale):
    """float64 library SDPA and logsumexp; q [n, d], k/v [m, d]."""
    q, k, v = (x.to(torch.float64) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(q[None, None], k[None, None],
                                                         v[None, None], scale=scale)[0, 0]
    lse = torch.logsumexp(scale * q @ k.T, dim=-1)
    return o.numpy(), lse.numpy()


def _dense_sets(H, Tq, Tkv):
    frames = np.tile(np.arange(Tkv, dtype=np.int32), (H, Tq, 1))
    counts = np.full((H, Tq), Tkv, dtype=np.int32)
    return frames, counts


@pytest.mark.parametrize("B,H,T,P,d", [(1, 2, 4, 64, 64), (2, 3, 3, 20, 32), (1, 1, 5, 7, 16)])
def test_dense_matches_library_sdpa(B, H, T, P, d):
    q, k, v = qkv(B, H, T * P, T * P, d, seed=3)
    frames, counts = _dense_sets(H, T, T)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attention(q, k, v, frames, counts, P, scale)
    o = o.reshape(B, H, T * P, d)
    lse = lse.reshape(B, H, T * P)
    for b in range(B):
        for h in range(H):
            ro, rl = _sdpa64(q[b, h], k[b, h], v[b, h], scale)
            np.testing.assert_allclose(o[b, h], ro, atol=1e-12, rtol=0)
            np.testing.assert_allclose(lse[b, h], rl, atol=1e-12, rtol=0)


@pytest.mark.parametrize("name", ["tiny_sinkwin", "tiny_dense"])
def test_restricted_matches_gathered_sdpa(name):
    w = WORKLOADS[name]
    q, k, v = workload_qkv(w, seed=0)
    frames, counts = S.workload_sets(w)
    scale = 1.0 / math.sqrt(w.d)
    o, lse = oracle.attention(q, k, v, frames, counts, w.P, scale)
    o = o.reshape(w.B, w.H, w.Lq, w.d)
    lse = lse.reshape(w.B, w.H, w.Lq)
    for h in range(w.H):
        for t in range(w.Tq):
            fr = frames[h, t, :counts[h, t]]
            idx = torch.cat([torch.arange(f * w.P, (f + 1) * w.P) for f in fr])
            rows = slice(t * w.P, (t + 1) * w.P)
            ro, rl = _sdpa64(q[0, h, rows], k[0, h, idx], v[0, h, idx], scale)
            np.testing.assert_allclose(o[0, h, rows], ro, atol=1e-12, rtol=0)
            np.testing.assert_allclose(lse[0, h, rows], rl, atol=1e-12, rtol=0)


def test_random_sets_with_batches_and_heads():
    # differing sets per (head, frame), B=2: catches head/batch/frame indexing slips
    B, H, Tq, Tkv, P, d = 2, 3, 3, 5, 12, 16
    q, k, v = qkv(B, H, Tq * P, Tkv * P, d, seed=11)
    rng = np.random.default_rng(5)
    Amax = 4
    frames = np.full((H, Tq, Amax), -1, np.int32)
    counts = np.zeros((H, Tq), np.int32)
    for h in range(H):
        for t in range(Tq):
            n = rng.integers(1, Amax + 1)
            fr = np.sort(rng.choice(Tkv, n, replace=False))
            frames[h, t, :n] = fr
            counts[h, t] = n
    scale = 0.37
    o, lse = oracle.attention(q, k, v, frames, counts, P, scale)
    o = o.reshape(B, H, Tq * P, d)
    lse = lse.reshape(B, H, Tq * P)
    for b in range(B):
        for h in range(H):
            for t in range(Tq):
                fr = frames[h, t, :counts[h, t]]
                idx = torch.cat([torch.arange(f * P, (f + 1) * P) for f in fr])
                rows = slice(t * P, (t + 1) * P)
                ro, rl = _sdpa64(q[b, h, rows], k[b, h, idx], v[b, h, idx], scale)
                np.testing.assert_allclose(o[b, h, rows], ro, atol=1e-12, rtol=0)
                np.testing.assert_allclose(lse[b, h, rows], rl, atol=1e-12, rtol=0)


def test_intra_frame_only_is_per_frame_attention():
    # ARL2 §2.1: bidirectional softmax inside each frame == A(t) = {t}
    B, H, T, P, d = 1, 2, 4, 24, 32
    q, k, v = qkv(B, H, T * P, T * P, d, seed=7)
    frames = np.arange(T, dtype=np.int32).reshape(1, T, 1).repeat(H, 0)
    counts = np.ones((H, T), np.int32)
    o, lse = oracle.attention(q, k, v, frames, counts, P, 0.2)
    o = o.reshape(B, H, T * P, d)
    for h in range(H):
        for t in range(T):
            r = slice(t * P, (t + 1) * P)
            ro, _ = _sdpa64(q[0, h, r], k[0, h, r], v[0, h, r], 0.2)
            np.testing.assert_allclose(o[0, h, r], ro, atol=1e-12, rtol=0)


def test_zero_query_gives_mean_of_values():
    B, H, T, P, d = 1, 1, 3, 10, 8
    _, k, v = qkv(B, H, T * P, T * P, d, seed=1)
    q = torch.zeros(B, H, T * P, d, dtype=torch.bfloat16)
    frames = np.array([[[0, 2], [1, -1], [0, 1]]], np.int32)
    counts = np.array([[2, 1, 2]], np.int32)
    o, lse = oracle.attention(q, k, v, frames, counts, P, 0.5)
    for t in range(T):
        fr = frames[0, t, :counts[0, t]]
        idx = np.concatenate([np.arange(f * P, (f + 1) * P) for f in fr])
        mean = v[0, 0, idx].double().mean(0).numpy()
        for i in range(t * P, (t + 1) * P):
            np.testing.assert_allclose(o[i], mean, atol=1e-14, rtol=0)
            assert abs(lse[i] - math.log(len(idx))) < 1e-14


def test_constant_values_pass_through():
    B, H, T, P, d = 1, 2, 3, 9, 8
    q, k, _ = qkv(B, H, T * P, T * P, d, seed=2)
    vec = torch.tensor([0.5, -1.25, 3.0, 0.0, 2.0, -0.75, 1.0, 8.0])
    v = vec.expand(B, H, T * P, d).to(torch.bfloat16).contiguous()
    frames, counts = _dense_sets(H, T, T)
    o, _ = oracle.attention(q, k, v, frames, counts, P, 0.3)
    np.testing.assert_allclose(o, np.broadcast_to(vec.numpy(), o.shape), atol=1e-13, rtol=0)


def test_key_shift_invariance():
    # softmax shift invariance: k_j -> k_j + c leaves O unchanged, LSE += scale * q.c
    B, H, T, P, d = 1, 1, 3, 8, 8
    g = torch.Generator().manual_seed(4)
    q = (torch.randint(-8, 9, (B, H, T * P, d), generator=g) * 0.125).to(torch.bfloat16)
    k = (torch.randint(-8, 9, (B, H, T * P, d), generator=g) * 0.25).to(torch.bfloat16)
    v = torch.randn(B, H, T * P, d, generator=g).to(torch.bfloat16)
    c = (torch.arange(d) % 3 - 1).to(torch.float32) * 0.5        # exact in bf16 after adding
    k2 = (k.float() + c).to(torch.bfloat16)
    assert torch.equal(k2.float(), k.float() + c)
    frames = np.array([[[0, 1], [2, -1], [0, 2]]], np.int32)
    counts = np.array([[2, 1, 2]], np.int32)
    scale = 0.7
    o1, l1 = oracle.attention(q, k, v, frames, counts, P, scale)
    o2, l2 = oracle.attention(q, k2, v, frames, counts, P, scale)
    shift = scale * (q[0, 0].double() @ c.double()).numpy()
    np.testing.assert_allclose(o2, o1, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l2, l1 + shift, atol=1e-12, rtol=0)


def test_key_permutation_invariance():
    # the attended key set is a set: permuting tokens inside and across attended frames
    B, H, T, P, d = 1, 1, 4, 6, 8
    q, k, v = qkv(B, H, T * P, T * P, d, seed=9)
    frames = np.array([[[1, 3], [0, 2], [1, 3], [0, 2]]], np.int32)
    counts = np.full((1, 4), 2, np.int32)
    o1, l1 = oracle.attention(q, k, v, frames, counts, P, 0.4)
    # permute tokens inside frame 1 and swap the contents of frames 1 and 3 (both attended
    # together by t=0, t=2)
    perm = torch.arange(T * P)
    inner = torch.randperm(P, generator=torch.Generator().manual_seed(0))
    perm[P:2 * P] = P + inner
    perm[P:2 * P], perm[3 * P:4 * P] = perm[3 * P:4 * P].clone(), perm[P:2 * P].clone()
    o2, l2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], frames, counts, P, 0.4)
    rows = np.r_[0:P, 2 * P:3 * P]
    np.testing.assert_allclose(o2[rows], o1[rows], atol=1e-13, rtol=0)
    np.testing.assert_allclose(l2[rows], l1[rows], atol=1e-13, rtol=0)


def test_empty_set_gives_zero_and_neg_inf():
    q, k, v = qkv(1, 1, 8, 16, 8, seed=0)
    frames = np.array([[[-1], [0]]], np.int32)
    counts = np.array([[0, 1]], np.int32)
    o, lse = oracle.attention(q, k, v, frames, counts, 4, 1.0)
    assert (o[:4] == 0).all() and np.isneginf(lse[:4]).all()
    assert np.isfinite(lse[4:]).all()


def test_sampled_rows_match_full():
    w = WORKLOADS["tiny_sinkwin"]
    q, k, v = workload_qkv(w, seed=0)
    frames, counts = S.workload_sets(w)
    o, lse = oracle.attention(q, k, v, frames, counts, w.P, 0.125)
    rows = np.array([0, 5, 63, 64, 200, 511], np.int64)
    o2, l2 = oracle.attention(q, k, v, frames, counts, w.P, 0.125, rows=rows)
    np.testing.assert_array_equal(o2, o[rows])
    np.testing.assert_array_equal(l2, lse[rows])


def test_brute_force_fsum_rows():
    # a handful of rows recomputed with exactly-rounded sums in pure Python
    w = WORKLOADS["tiny_sinkwin"]
    q, k, v = workload_qkv(w, seed=0)
    frames, counts = S.workload_sets(w)
    scale = 1 / 8
    rows = [3, 70, 130, 255, 256 + 200]
    o, lse = oracle.attention(q, k, v, frames, counts, w.P, scale, rows=np.array(rows))
    qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
    for n, r in enumerate(rows):
        h, i = divmod(r, w.Lq)
        t = i // w.P
        keys = [f * w.P + p for f in frames[h, t, :counts[h, t]] for p in range(w.P)]
        s = [scale * math.fsum(qd[0, h, i] * kd[0, h, j]) for j in keys]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        l_ = math.fsum(e)
        ref = [math.fsum(e[a] * vd[0, h, j, c] for a, j in enumerate(keys)) / l_
               for c in range(w.d)]
        np.testing.assert_allclose(o[n], ref, atol=1e-13, rtol=0)
        assert abs(lse[n] - (m + math.log(l_))) < 1e-13


def test_rejects_bad_frames():
    q, k, v = qkv(1, 1, 4, 8, 4, seed=0)
    with pytest.raises(RuntimeError):
        oracle.attention(q, k, v, np.array([[[5]]], np.int32), np.array([[1]], np.int32), 4, 1.0)
