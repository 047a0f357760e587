"""Attended-frame-set oracle (pure Python).  TEST INFRASTRUCTURE ONLY.

Each function follows the method's own steps in the order the pages give
them, written from the description; nothing here is shared with the CUDA path.

LVSA ("LVSA: Atención Dispersa Libre de Entrenamiento para Difusión de Video
Largo", §2 Mecanismo Central):
  A(t) = G_s ∪ W(t), where
  * G_s, rotating global anchors (§2.1): the periodic global frames are shifted by
    s mod T_per at denoising step s, so that over T_per consecutive steps each frame
    is a global anchor exactly once.  Reading: G_s = {f : f mod T_per == s mod T_per}
    (the only periodic set with that property).
  * W(t), expanded adaptive window (§2.2): a local window of W frames; where it
    overlaps the anchors it is extended so that |A(t)| reaches the budget C.
    Readings: the base window is centred on t (an even W puts the extra frame on the
    future side) and shifted inward at the ends of [0, T); it grows one frame at a
    time, alternating future side first, skipping a side that hit the boundary, until
    |A(t)| = min(C, T) or it covers every frame; it never shrinks, so when
    |G_s ∪ base window| > C the set is left larger than C.

Per-head cache kinds ("Head Forcing", §2 Asignación de Caché KV por Cabeza;
"ISPA", §2.1), for query frame t placed at KV frame c = t + q_off, whose chunk is
[c0, c0 + chunk_len) with c0 = c - (c mod chunk_len):
  * local    = the current chunk ∪ the n_prev frames before it
  * anchor   = the first n_sink frames (the sink) ∪ local
  * memory   = anchor ∪ the head's selected history frames
  * explicit = the head's list
  * dense    = every KV frame
All lists are clipped to [0, T_kv), sorted ascending, without duplicates.

Parity status: pinned (tests/test_oracle_sets.py: the LVSA invariants the page
states, hand-computed lists, hand-written streaming lists).
"""
from __future__ import annotations

import numpy as np


def lvsa_anchors(T: int, T_per: int, s: int) -> set:
    """G_s: frames f in [0, T) with f mod T_per == s mod T_per (LVSA §2.1)."""
    phase = s % T_per
    return {f for f in range(T) if f % T_per == phase}


def lvsa_base_window(t: int, T: int, W: int):
    """Base local window [lo, hi] of W frames around t (LVSA §2.2), shifted inside [0, T)."""
    if W >= T:
        return 0, T - 1
    lo = t - (W - 1) // 2
    hi = lo + W - 1
    if lo < 0:
        lo, hi = 0, W - 1
    elif hi > T - 1:
        lo, hi = T - W, T - 1
    return lo, hi


def lvsa_set(t: int, T: int, C: int, W: int, T_per: int, s: int) -> list:
    """A(t) = G_s ∪ W(t), with W(t) grown until |A(t)| = min(C, T) (LVSA §2)."""
    anchors = lvsa_anchors(T, T_per, s)
    lo, hi = lvsa_base_window(t, T, W)
    attended = set(anchors) | set(range(lo, hi + 1))
    target = min(C, T)
    future_turn = True
    while len(attended) < target and not (lo == 0 and hi == T - 1):
        grow_future = (future_turn and hi < T - 1) or lo == 0
        if grow_future:
            hi += 1
            attended.add(hi)
        else:
            lo -= 1
            attended.add(lo)
        future_turn = not future_turn
    return sorted(attended)


def _clip_sort(frames, T_kv):
    return sorted({int(f) for f in frames if 0 <= int(f) < T_kv})


def local_set(c: int, T_kv: int, chunk_len: int, n_prev: int) -> list:
    c0 = c - (c % chunk_len)
    return _clip_sort(range(c0 - n_prev, c0 + chunk_len), T_kv)


def anchor_set(c: int, T_kv: int, chunk_len: int, n_prev: int, n_sink: int) -> list:
    return _clip_sort(list(range(n_sink)) + local_set(c, T_kv, chunk_len, n_prev), T_kv)


def memory_set(c, T_kv, chunk_len, n_prev, n_sink, extra) -> list:
    return _clip_sort(anchor_set(c, T_kv, chunk_len, n_prev, n_sink) + list(extra), T_kv)


def head_set(kind: str, t: int, *, T_kv: int, q_off: int = 0, C: int = 0, W: int = 0,
             T_per: int = 1, step: int = 0, n_sink: int = 0, n_prev: int = 0,
             chunk_len: int = 1, extra=()) -> list:
    """A(h, t) for one head of the given kind; t is the query frame index."""
    c = t + q_off
    if kind == "dense":
        return list(range(T_kv))
    if kind == "lvsa":
        return lvsa_set(c, T_kv, C, W, T_per, step)
    if kind == "local":
        return local_set(c, T_kv, chunk_len, n_prev)
    if kind == "anchor":
        return anchor_set(c, T_kv, chunk_len, n_prev, n_sink)
    if kind == "memory":
        return memory_set(c, T_kv, chunk_len, n_prev, n_sink, extra)
    if kind == "explicit":
        return _clip_sort(extra, T_kv)
    raise ValueError(f"unknown set kind {kind!r}")


def build_sets(kinds, extras, Tq: int, Amax: int, **params):
    """frames int32 [H][Tq][Amax] (padded with -1) and counts int32 [H][Tq]."""
    H = len(kinds)
    frames = np.full((H, Tq, Amax), -1, dtype=np.int32)
    counts = np.zeros((H, Tq), dtype=np.int32)
    for h in range(H):
        for t in range(Tq):
            a = head_set(kinds[h], t, extra=extras[h], **params)
            if len(a) > Amax:
                raise ValueError(f"|A({h},{t})| = {len(a)} exceeds Amax = {Amax}")
            counts[h, t] = len(a)
            frames[h, t, :len(a)] = a
    return frames, counts


def workload_sets(w, step: int = 0, Amax: int | None = None):
    """Sets for a ``sfa_workloads.Workload`` at denoising step ``step``."""
    kinds = [hs.kind for hs in w.heads]
    extras = [hs.extra for hs in w.heads]
    params = dict(T_kv=w.Tkv, q_off=w.q_off, C=w.C, W=w.W, T_per=w.T_per, step=step,
                  n_sink=w.n_sink, n_prev=w.n_prev, chunk_len=w.chunk_len)
    if Amax is None:
        Amax = max(len(head_set(kinds[h], t, extra=extras[h], **params))
                   for h in range(w.H) for t in range(w.Tq))
    return build_sets(kinds, extras, w.Tq, Amax, **params)
