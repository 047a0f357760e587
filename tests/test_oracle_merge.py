"""Pins for the LSE-merge oracle (CPU only).

"ISPA", §2.1 Dual-Stream Warmup: attention split into a local and a history branch
by the LSE state is merged post hoc into full attention.  The pin is that equality:
merging the oracle's attention over two disjoint frame sets gives the oracle's
attention over their union (itself pinned to library SDPA), plus the empty cases.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import sets as S
from sfa_workloads import WORKLOADS, qkv, workload_qkv


def _attn(q, k, v, lists, P, scale, Tq):
    H = len(lists)
    Amax = max(1, max(len(x) for per_h in lists for x in per_h))
    frames = np.full((H, Tq, Amax), -1, np.int32)
    counts = np.zeros((H, Tq), np.int32)
    for h in range(H):
        for t in range(Tq):
            frames[h, t, :len(lists[h][t])] = lists[h][t]
            counts[h, t] = len(lists[h][t])
    return oracle.attention(q, k, v, frames, counts, P, scale)


@pytest.mark.parametrize("split_seed", [0, 1, 2])
def test_disjoint_branches_merge_to_union(split_seed):
    B, H, Tq, Tkv, P, d = 1, 2, 3, 6, 10, 16
    q, k, v = qkv(B, H, Tq * P, Tkv * P, d, seed=21)
    rng = np.random.default_rng(split_seed)
    full, a1, a2 = [], [], []
    for h in range(H):
        fh, x1, x2 = [], [], []
        for t in range(Tq):
            u = sorted(rng.choice(Tkv, rng.integers(2, Tkv + 1), replace=False).tolist())
            cut = rng.integers(1, len(u))
            pick = set(rng.choice(u, cut, replace=False).tolist())
            fh.append(u)
            x1.append(sorted(pick))
            x2.append(sorted(set(u) - pick))
        full.append(fh), a1.append(x1), a2.append(x2)
    scale = 1 / math.sqrt(d)
    of, lf = _attn(q, k, v, full, P, scale, Tq)
    o1, l1 = _attn(q, k, v, a1, P, scale, Tq)
    o2, l2 = _attn(q, k, v, a2, P, scale, Tq)
    om, lm = oracle.lse_merge(o1, l1, o2, l2)
    np.testing.assert_allclose(om, of, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lm, lf, atol=1e-12, rtol=0)
    om2, lm2 = oracle.lse_merge(o2, l2, o1, l1)
    np.testing.assert_allclose(om2, om, atol=1e-15, rtol=0)
    np.testing.assert_allclose(lm2, lm, atol=1e-15, rtol=0)


def test_ispa_local_history_split_tiny():
    # the lsemerge frame layout shrunk to P=8: local = sink + current, history = 1..12
    wl, wh, wf = (WORKLOADS[n] for n in ("lsemerge_local", "lsemerge_hist", "lsemerge_full"))
    P, d = 8, 16
    q, k, v = qkv(1, 2, P, wl.Tkv * P, d, seed=5)
    out = []
    for w in (wl, wh, wf):
        fr, cn = S.workload_sets(w)
        out.append(oracle.attention(q, k, v, fr[:2], cn[:2], P, 0.25))
    (o1, l1), (o2, l2), (of, lf) = out
    om, lm = oracle.lse_merge(o1, l1, o2, l2)
    np.testing.assert_allclose(om, of, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lm, lf, atol=1e-12, rtol=0)


def test_empty_branch_cases():
    rng = np.random.default_rng(0)
    o1, o2 = rng.standard_normal((3, 4)), rng.standard_normal((3, 4))
    l1 = np.array([0.3, -np.inf, -np.inf])
    l2 = np.array([-np.inf, 1.7, -np.inf])
    o, lse = oracle.lse_merge(o1, l1, o2, l2)
    np.testing.assert_array_equal(o[0], o1[0])
    np.testing.assert_array_equal(o[1], o2[1])
    np.testing.assert_array_equal(o[2], np.zeros(4))
    assert lse[0] == 0.3 and lse[1] == 1.7 and np.isneginf(lse[2])


def test_equal_lse_is_average():
    o1, o2 = np.array([[1.0, 2.0]]), np.array([[3.0, -2.0]])
    o, lse = oracle.lse_merge(o1, np.array([0.5]), o2, np.array([0.5]))
    np.testing.assert_allclose(o, [[2.0, 0.0]], atol=1e-15)
    assert abs(lse[0] - (0.5 + math.log(2.0))) < 1e-15


def test_large_lse_gap_is_stable():
    o1, o2 = np.array([[1.0]]), np.array([[5.0]])
    o, lse = oracle.lse_merge(o1, np.array([1000.0]), o2, np.array([-1000.0]))
    assert o[0, 0] == 1.0 and lse[0] == 1000.0
