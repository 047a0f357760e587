"""Pins for the set oracle (CPU only).

What the pages fix about A(t) ("LVSA: Atención Dispersa Libre de Entrenamiento para
Difusión de Video Largo", §2): A(t) = G ∪ W(t) replaces the full set {0..T-1}; over
T_per consecutive denoising steps every frame is a global anchor exactly once; the
window is extended over anchor overlaps so that |A(t)| ≈ C.  Hand-worked lists live in
tests/golden/sets_hand.txt.
"""
import os

import pytest

from oracle import sets as S
from sfa_workloads import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sets_hand.txt")


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split(":")
            name, h, t, s = lhs.split()
            rows.append((name, int(h), int(t), int(s), [int(x) for x in rhs.split()]))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: f"{r[0]}-h{r[1]}-t{r[2]}-s{r[3]}")
def test_hand_worked_lists(row):
    name, h, t, s, expect = row
    w = WORKLOADS[name]
    frames, counts = S.workload_sets(w, step=s)
    got = frames[h, t, :counts[h, t]].tolist()
    assert got == expect


@pytest.mark.parametrize("s", [0, 1, 2, 3])
def test_lvsa41_invariants(s):
    T, C, W, T_per = 41, 21, 9, 4
    G = S.lvsa_anchors(T, T_per, s)
    for t in range(T):
        a = S.lvsa_set(t, T, C, W, T_per, s)
        assert a == sorted(set(a)) and all(0 <= f < T for f in a)
        assert t in a
        assert G <= set(a)
        lo, hi = S.lvsa_base_window(t, T, W)
        assert hi - lo + 1 == W and lo <= t <= hi
        assert set(range(lo, hi + 1)) <= set(a)
        # |G_s ∪ W_base(t)| <= C everywhere in this workload, so the budget is met exactly
        assert len(G | set(range(lo, hi + 1))) <= C
        assert len(a) == C
        # the window part of A(t) is one contiguous block that contains t
        non_anchor = sorted(set(a) - G)
        win = [f for f in a if f not in G or lo <= f <= hi]
        assert non_anchor == [f for f in non_anchor if min(win) <= f <= max(win)]


@pytest.mark.parametrize("T,T_per", [(41, 4), (121, 6), (7, 3), (5, 8)])
def test_each_frame_anchor_once_per_period(T, T_per):
    # LVSA §2.1: over T_per consecutive steps each frame is a global anchor exactly once
    for s0 in range(0, 3 * T_per):
        hits = [0] * T
        for s in range(s0, s0 + T_per):
            for f in S.lvsa_anchors(T, T_per, s):
                hits[f] += 1
        assert hits == [1] * T


@pytest.mark.parametrize("s", range(6))
def test_long121_budget_never_truncates(s):
    # C=21 cannot hold |G_s| (20-21 anchors) plus a 13-frame window: the set is G_s ∪ W_base
    T, C, W, T_per = 121, 21, 13, 6
    G = S.lvsa_anchors(T, T_per, s)
    for t in range(T):
        a = S.lvsa_set(t, T, C, W, T_per, s)
        lo, hi = S.lvsa_base_window(t, T, W)
        base = G | set(range(lo, hi + 1))
        assert len(base) > C
        assert set(a) == base
        assert 30 <= len(a) <= 32


@pytest.mark.parametrize("T,C,W", [(10, 20, 3), (10, 3, 10), (10, 10, 1), (1, 1, 1)])
def test_lvsa_degenerates_to_dense(T, C, W):
    # W >= T or C >= T: the window grows to every frame, i.e. the full set {0..T-1}
    for s in range(3):
        for t in range(T):
            assert S.lvsa_set(t, T, C, W, 4, s) == list(range(T))


def test_lvsa_budget_with_small_anchor_period():
    # T_per = 1: every frame is an anchor, so A(t) is dense whatever C and W are
    for t in range(9):
        assert S.lvsa_set(t, 9, 3, 1, 1, 0) == list(range(9))


def test_stream_sizes_and_structure():
    w = WORKLOADS["stream"]
    frames, counts = S.workload_sets(w)
    assert counts[:4].tolist() == [[6] * 3] * 4
    assert counts[4:8].tolist() == [[7] * 3] * 4
    assert counts[8:].tolist() == [[13] * 3] * 4
    for h in range(12):
        for t in range(3):
            a = frames[h, t, :counts[h, t]].tolist()
            assert {18, 19, 20, 21, 22, 23} <= set(a)          # chunk + 3 previous frames
            assert (0 in a) == (h >= 4)                          # sink for anchor/memory heads
            if h >= 8:
                assert set(w.heads[h].extra) <= set(a)


def test_padding_and_amax():
    w = WORKLOADS["tiny_sinkwin"]
    frames, counts = S.workload_sets(w, Amax=5)
    assert frames.shape == (2, 4, 5)
    for h in range(2):
        for t in range(4):
            assert (frames[h, t, counts[h, t]:] == -1).all()
    with pytest.raises(ValueError):
        S.workload_sets(w, Amax=2)


def test_kind_clipping():
    # lists are clipped to [0, T_kv): local window near frame 0, explicit out-of-range frames
    assert S.local_set(1, 10, 1, 3) == [0, 1]
    assert S.head_set("explicit", 0, T_kv=5, extra=(7, 3, 3, -1, 0)) == [0, 3]
    assert S.anchor_set(9, 10, 4, 0, 2) == [0, 1, 8, 9]
