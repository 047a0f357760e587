"""Hierarchical sparse attention (HSA) oracle, float64.  TEST INFRASTRUCTURE ONLY.

Follows "Resumen Técnico: LIGHT FORCING", §2.2 Atención Dispersa Jerárquica (HSA), in
the page's order:
  1. token compression: query and key tokens are mean-pooled per block and per frame;
  2. frame selection: for each query block, a few history frames are retrieved with the
     frame-level pooled keys;
  3. block selection: inside the selected frames, the critical blocks are found with the
     block-level pooled keys;
  4. attention is computed over the selected frame-block pairs only.

Readings where the page is silent:
  * a key block is 128 consecutive tokens of one frame (block b of frame f holds tokens
    [f*P + 128*b, f*P + min(128*(b+1), P))), numbered g = f * nblk + b with
    nblk = ceil(P / 128); a query block is 256 consecutive query rows of one frame
    (the last block of a frame holds the rest);
  * relevance is the dot product of the pooled query with the pooled key (the softmax
    scale is a common positive factor and does not change an order);
  * the sink frames and the local window (the anchor set of the per-head cache kinds:
    the first n_sink frames, the current chunk and the n_prev frames before it) are
    always attended in full; the history candidates are the other frames before the
    current chunk;
  * top-k keeps the k largest scores; equal scores go to the smaller index; k larger
    than the number of candidates keeps them all; block selection ranks the blocks of
    all selected frames together.

Parity status: pinned (tests/test_oracle_hsa.py: hand-built pooling and selection
cases with known answers, invariants, and the full-selection case that reduces to the
pinned frame-list attention).
"""
from __future__ import annotations

import math

import numpy as np

KEY_BLOCK = 128   # tokens per key block
QUERY_BLOCK = 256  # query rows per query block


def n_key_blocks(P: int) -> int:
    return (P + KEY_BLOCK - 1) // KEY_BLOCK


def n_query_blocks(P: int) -> int:
    return (P + QUERY_BLOCK - 1) // QUERY_BLOCK


def block_tokens(g: int, P: int) -> tuple:
    """Token interval [lo, hi) of global key block g."""
    nb = n_key_blocks(P)
    f, b = divmod(g, nb)
    return f * P + b * KEY_BLOCK, f * P + min((b + 1) * KEY_BLOCK, P)


def pool_keys(k: np.ndarray, P: int):
    """Mean-pooled keys (step 1).  k: [B, H, T*P, d] -> frame means [B, H, T, d] and
    block means [B, H, T, nblk, d], float64."""
    k = np.asarray(k, dtype=np.float64)
    B, H, L, d = k.shape
    T, nb = L // P, n_key_blocks(P)
    frames = k.reshape(B, H, T, P, d).mean(axis=3)
    blocks = np.zeros((B, H, T, nb, d))
    for b in range(nb):
        lo, hi = b * KEY_BLOCK, min((b + 1) * KEY_BLOCK, P)
        blocks[:, :, :, b] = k.reshape(B, H, T, P, d)[:, :, :, lo:hi].mean(axis=3)
    return frames, blocks


def pool_queries(q: np.ndarray, P: int) -> np.ndarray:
    """Mean-pooled query blocks (step 1).  q: [B, H, Tq*P, d] -> [B, H, Tq, nqb, d]."""
    q = np.asarray(q, dtype=np.float64)
    B, H, L, d = q.shape
    Tq, nq = L // P, n_query_blocks(P)
    out = np.zeros((B, H, Tq, nq, d))
    for i in range(nq):
        lo, hi = i * QUERY_BLOCK, min((i + 1) * QUERY_BLOCK, P)
        out[:, :, :, i] = q.reshape(B, H, Tq, P, d)[:, :, :, lo:hi].mean(axis=3)
    return out


def always_frames(t: int, *, T_kv: int, q_off: int, chunk_len: int, n_prev: int, n_sink: int) -> list:
    """Frames attended in full by query frame t: the sink and the local window."""
    c = t + q_off
    c0 = c - c % chunk_len
    fr = set(range(min(n_sink, T_kv))) | set(range(max(c0 - n_prev, 0), min(c0 + chunk_len, T_kv)))
    return sorted(fr)


def history_frames(t: int, *, T_kv: int, q_off: int, chunk_len: int, n_prev: int, n_sink: int) -> list:
    """Candidate frames for the selection: before the current chunk, not always attended."""
    c = t + q_off
    c0 = c - c % chunk_len
    keep = set(always_frames(t, T_kv=T_kv, q_off=q_off, chunk_len=chunk_len, n_prev=n_prev, n_sink=n_sink))
    return [f for f in range(min(c0, T_kv)) if f not in keep]


def top_k(ids, scores, k: int) -> list:
    """The k ids with the largest scores; equal scores go to the smaller id."""
    order = sorted(range(len(ids)), key=lambda i: (-scores[i], ids[i]))
    return sorted(ids[i] for i in order[:k])


def select_blocks(qbar: np.ndarray, kf: np.ndarray, kb: np.ndarray, t: int, *, P: int, T_kv: int, q_off: int,
                  chunk_len: int, n_prev: int, n_sink: int, k_frames: int, k_blocks: int) -> list:
    """Steps 2-3 for one query block: the sorted global key-block ids it attends.

    qbar: [d] pooled query; kf: [T_kv, d] frame keys; kb: [T_kv, nblk, d] block keys."""
    nb = n_key_blocks(P)
    kw = dict(T_kv=T_kv, q_off=q_off, chunk_len=chunk_len, n_prev=n_prev, n_sink=n_sink)
    cand = history_frames(t, **kw)
    f_scores = [float(np.dot(qbar, kf[f])) for f in cand]
    chosen = top_k(cand, f_scores, k_frames)
    blk = [f * nb + b for f in chosen for b in range(nb)]
    b_scores = [float(np.dot(qbar, kb[g // nb, g % nb])) for g in blk]
    picked = top_k(blk, b_scores, k_blocks)
    full = [f * nb + b for f in always_frames(t, **kw) for b in range(nb)]
    return sorted(set(full) | set(picked))


def build_block_lists(q, k, *, P: int, T_kv: int, q_off: int, chunk_len: int, n_prev: int, n_sink: int,
                      k_frames: int, k_blocks: int, Bmax: int | None = None):
    """Block lists for every (b, h, t, query block): ([B, H, Tq, nqb, Bmax] int32, -1 padded;
    counts [B, H, Tq, nqb] int32)."""
    kf, kb = pool_keys(k, P)
    qb = pool_queries(q, P)
    B, H, Tq, nq, _ = qb.shape
    lists = [[[[select_blocks(qb[b, h, t, i], kf[b, h], kb[b, h], t, P=P, T_kv=T_kv, q_off=q_off,
                              chunk_len=chunk_len, n_prev=n_prev, n_sink=n_sink, k_frames=k_frames,
                              k_blocks=k_blocks)
                for i in range(nq)] for t in range(Tq)] for h in range(H)] for b in range(B)]
    m = max(len(x) for a in lists for bb in a for c in bb for x in c)
    Bmax = m if Bmax is None else Bmax
    assert Bmax >= m
    out = np.full((B, H, Tq, nq, Bmax), -1, np.int32)
    cnt = np.zeros((B, H, Tq, nq), np.int32)
    for b in range(B):
        for h in range(H):
            for t in range(Tq):
                for i in range(nq):
                    x = lists[b][h][t][i]
                    out[b, h, t, i, :len(x)] = x
                    cnt[b, h, t, i] = len(x)
    return out, cnt


def attention_blocks(q, k, v, lists, counts, P: int, scale: float, rows=None):
    """Step 4: float64 softmax attention of each query row over the key blocks listed
    for its query block.  q: [B, H, Tq*P, d]; k, v: [B, H, T_kv*P, d]; lists/counts as
    build_block_lists returns.  Returns O [B, H, Tq*P, d] and LSE [B, H, Tq*P] (natural
    log of the sum of exp(scale * q.k)); with `rows` (flat indices into [B*H*Tq*P]) only
    those rows are computed (O and LSE then have one entry per listed row)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, Lq, d = q.shape
    Tq = Lq // P

    def keys_of(b, h, t, i):
        idx = []
        for g in lists[b, h, t, i, :counts[b, h, t, i]]:
            lo, hi = block_tokens(int(g), P)
            idx.extend(range(lo, hi))
        return np.asarray(idx, dtype=np.int64)

    def one(b, h, p_rows, t, i):
        ks = keys_of(b, h, t, i)
        qr = q[b, h, p_rows]
        if len(ks) == 0:
            return np.zeros((len(p_rows), d)), np.full(len(p_rows), -math.inf)
        s = scale * (qr @ k[b, h, ks].T)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1)
        return (e @ v[b, h, ks]) / l[:, None], m[:, 0] + np.log(l)

    if rows is None:
        O = np.zeros((B, H, Lq, d))
        LSE = np.zeros((B, H, Lq))
        for b in range(B):
            for h in range(H):
                for t in range(Tq):
                    for i in range(n_query_blocks(P)):
                        lo, hi = t * P + i * QUERY_BLOCK, t * P + min((i + 1) * QUERY_BLOCK, P)
                        o, lse = one(b, h, np.arange(lo, hi), t, i)
                        O[b, h, lo:hi] = o
                        LSE[b, h, lo:hi] = lse
        return O, LSE
    rows = np.asarray(rows, dtype=np.int64)
    O = np.zeros((len(rows), d))
    LSE = np.zeros(len(rows))
    for n, r in enumerate(rows):
        b, rem = divmod(int(r), H * Lq)
        h, p = divmod(rem, Lq)
        t, pp = divmod(p, P)
        o, lse = one(b, h, np.asarray([p]), t, pp // QUERY_BLOCK)
        O[n] = o[0]
        LSE[n] = lse[0]
    return O, LSE
