"""Seeded synthetic workloads for frame-sparse attention.

This module only draws inputs and names workload shapes. It holds none of the
method's arithmetic (no attention, no set construction, no merge), so both the
CPU oracle's callers and the CUDA path's callers can take their inputs from it.

Shapes follow the video-DiT workloads the method is described on:
  * "LVSA: Atención Dispersa Libre de Entrenamiento para Difusión de Video Largo",
    §2 Mecanismo Central / Complejidad: T latent frames of P tokens, budget C.
    Wan-2.1-1.3B-like: 30x52 patch grid -> P = 1560, H = 12, d = 128, C = 21.
  * "Head Forcing", §2 (per-head KV caches): local / anchor / memory heads.
  * "ISPA", §2.1 Dual-Stream Warmup: local (current + sink) and history branches.
  * "Resumen Técnico: LIGHT FORCING", §2.2 (HSA): an autoregressive chunk that
    selects history frames, then blocks, by mean-pooled keys.
  * "Asistir Localmente, Recordar Linealmente (ARL2)", §2.1-2.2: the inter-frame branch
    (a gated delta rule over frames), with synthetic feature-mapped inputs and gates.

The real activations of those models are not available; Q, K and V are drawn
i.i.d. N(0, 1) in fp32 and rounded to bf16, which has the right shapes, dtype
and value scale (unit-variance projections) but no trained structure.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class SetSpec:
    """How one head builds its attended frame sets (kind names are strings)."""

    kind: str                      # 'dense' | 'lvsa' | 'local' | 'anchor' | 'memory' | 'explicit'
    extra: tuple = ()              # explicit / memory frames (absolute KV frame indices)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Tq: int
    Tkv: int
    q_off: int
    P: int
    d: int
    # set parameters (shared by all heads)
    C: int = 0
    W: int = 0
    T_per: int = 1
    steps: tuple = (0,)
    n_sink: int = 0
    n_prev: int = 0
    chunk_len: int = 1
    heads: tuple = field(default_factory=tuple)   # one SetSpec per head
    # hierarchical selection (HSA): history frames kept per query block, then key blocks
    k_frames: int = 0
    k_blocks: int = 0

    @property
    def Lq(self) -> int:
        return self.Tq * self.P

    @property
    def Lkv(self) -> int:
        return self.Tkv * self.P


def memory_history_frames(n_heads: int, seed: int = 0, n_hist: int = 17, n_pick: int = 6):
    """Seeded episodic-memory picks for memory heads (one draw per head, in head order).

    Each draw is ``n_pick`` distinct frames from the history frames 1..n_hist
    (frame 0 is the sink, already in the anchor part of the set).  The pages select
    these by scene novelty on real key embeddings ("Head Forcing", §2, Memoria
    Episódica); without a trained model a seeded uniform draw stands in.
    """
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n_heads):
        pick = rng.choice(n_hist, n_pick, replace=False) + 1
        out.append(tuple(int(x) for x in pick))
    return out


def _stream_heads():
    mem = memory_history_frames(4, seed=0)
    heads = [SetSpec("local")] * 4 + [SetSpec("anchor")] * 4
    heads += [SetSpec("memory", extra=m) for m in mem]
    return tuple(heads)


WORKLOADS = {
    # 4 frames x 64 tokens, 2 heads, d=64: dense pattern and sink + window {0, t-1, t}
    "tiny_dense": Workload("tiny_dense", B=1, H=2, Tq=4, Tkv=4, q_off=0, P=64, d=64,
                           heads=(SetSpec("dense"),) * 2),
    "tiny_sinkwin": Workload("tiny_sinkwin", B=1, H=2, Tq=4, Tkv=4, q_off=0, P=64, d=64,
                             n_sink=1, n_prev=1, chunk_len=1,
                             heads=(SetSpec("anchor"),) * 2),
    # LVSA at a Wan-2.1-1.3B-like shape (41 latent frames, 30x52 patches)
    "lvsa41": Workload("lvsa41", B=1, H=12, Tq=41, Tkv=41, q_off=0, P=1560, d=128,
                       C=21, W=9, T_per=4, steps=(0, 1, 2, 3),
                       heads=(SetSpec("lvsa"),) * 12),
    # streaming AR chunk: 3 query frames after 21 history frames, per-head caches
    "stream": Workload("stream", B=1, H=12, Tq=3, Tkv=24, q_off=21, P=1560, d=128,
                       n_sink=1, n_prev=3, chunk_len=3, heads=_stream_heads()),
    # long video: 121 latent frames
    "long121": Workload("long121", B=1, H=12, Tq=121, Tkv=121, q_off=0, P=1560, d=128,
                        C=21, W=13, T_per=6, steps=(0, 1, 2, 3, 4, 5),
                        heads=(SetSpec("lvsa"),) * 12),
    # LSE-decomposed attention: frame 0 = sink, 1..12 history, 13 = current (query)
    "lsemerge_local": Workload("lsemerge_local", B=1, H=12, Tq=1, Tkv=14, q_off=13, P=1560,
                               d=128, n_sink=1, n_prev=0, chunk_len=1,
                               heads=(SetSpec("anchor"),) * 12),
    "lsemerge_hist": Workload("lsemerge_hist", B=1, H=12, Tq=1, Tkv=14, q_off=13, P=1560,
                              d=128, heads=(SetSpec("explicit", extra=tuple(range(1, 13))),) * 12),
    "lsemerge_full": Workload("lsemerge_full", B=1, H=12, Tq=1, Tkv=14, q_off=13, P=1560,
                              d=128, heads=(SetSpec("dense"),) * 12),
    # HSA: the streaming chunk of "stream"; sink + local window always, plus the 24 best
    # 128-token blocks of the 4 best history frames (of 17) per 256-row query block
    # ARL2 inter-frame branch: 24 frames of the 30x52-patch shape, one state per head
    "gdn": Workload("gdn", B=1, H=12, Tq=24, Tkv=24, q_off=0, P=1560, d=128, heads=(SetSpec("gdn"),) * 12),
    "hsa": Workload("hsa", B=1, H=12, Tq=3, Tkv=24, q_off=21, P=1560, d=128,
                    n_sink=1, n_prev=3, chunk_len=3, k_frames=4, k_blocks=24,
                    heads=(SetSpec("hsa"),) * 12),
}


def qkv(B: int, H: int, Lq: int, Lkv: int, d: int, seed: int = 0):
    """Q, K, V as contiguous bf16 CPU tensors [B, H, L, d].

    One ``torch.Generator('cpu')`` seeded with ``seed`` draws Q, then K, then V,
    each ``randn`` in fp32, rounded to bf16 (round-to-nearest-even).
    """
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(B, H, Lq, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(B, H, Lkv, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(B, H, Lkv, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v


def workload_qkv(w: Workload, seed: int = 0):
    if w.k_frames:
        return qkv_structured(w.B, w.H, w.Tq, w.Tkv, w.P, w.d, seed)
    return qkv(w.B, w.H, w.Lq, w.Lkv, w.d, seed)


def qkv_structured(B: int, H: int, Tq: int, Tkv: int, P: int, d: int, seed: int = 0, sigma: float = 0.5,
                   key_block: int = 128, query_block: int = 256):
    """Q, K, V as in ``qkv`` plus per-frame and per-block offsets, so that pooled keys differ.

    Real video features are correlated within a frame and within a spatial block; an
    i.i.d. draw pools to almost nothing and makes any selection among frames arbitrary.
    After the Q, K, V draws of ``qkv`` the same generator draws, in this order,
    N(0, sigma^2) offset vectors per (b, h, KV frame), per (b, h, KV frame, key block of
    ``key_block`` tokens) and per (b, h, query frame, query block of ``query_block``
    rows); each K token gets its frame's and its block's offsets added, each Q row its
    block's, in fp32 before the rounding to bf16.  V is unchanged.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(B, H, Tq * P, d, generator=g, dtype=torch.float32)
    k = torch.randn(B, H, Tkv * P, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, Tkv * P, d, generator=g, dtype=torch.float32)
    nkb = (P + key_block - 1) // key_block
    nqb = (P + query_block - 1) // query_block
    frame_off = sigma * torch.randn(B, H, Tkv, d, generator=g, dtype=torch.float32)
    block_off = sigma * torch.randn(B, H, Tkv, nkb, d, generator=g, dtype=torch.float32)
    query_off = sigma * torch.randn(B, H, Tq, nqb, d, generator=g, dtype=torch.float32)
    kb_of_token = torch.arange(P) // key_block
    qb_of_row = torch.arange(P) // query_block
    k = k.view(B, H, Tkv, P, d) + frame_off[:, :, :, None, :] + block_off[:, :, :, kb_of_token, :]
    q = q.view(B, H, Tq, P, d) + query_off[:, :, :, qb_of_row, :]
    return (q.reshape(B, H, Tq * P, d).to(torch.bfloat16), k.reshape(B, H, Tkv * P, d).to(torch.bfloat16),
            v.to(torch.bfloat16))


def sample_rows(w: Workload, n_per_head: int, seed: int = 0, frames=()):
    """Seeded flat query-row indices ``(b*H + h)*Lq + i`` for sampled parity checks.

    Takes every row of each frame in ``frames`` (all heads, all batches) plus
    ``n_per_head`` uniformly drawn rows per (b, h).  Returned sorted, unique, int64.
    """
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(w.B):
        for h in range(w.H):
            base = (b * w.H + h) * w.Lq
            for t in frames:
                rows.append(base + t * w.P + np.arange(w.P, dtype=np.int64))
            if n_per_head:
                rows.append(base + rng.integers(0, w.Lq, size=n_per_head, dtype=np.int64))
    if not rows:
        return np.zeros(0, dtype=np.int64)
    return np.unique(np.concatenate(rows)).astype(np.int64)


def gdn_inputs(B: int, H: int, T: int, P: int, d: int, seed: int = 0):
    """Inputs of the ARL2 inter-frame branch: Q', K' [B, H, T*P, d] bf16 with unit-norm
    rows, V' [B, H, T*P, d] bf16, alpha [B, H, T] fp32, beta [B, H, T*P] fp32.

    The page's feature maps, gates and step sizes are learned; a seeded stand-in keeps
    the recurrence well conditioned the way a trained one is: one
    ``torch.Generator('cpu')`` draws, in this order, Q', K', V' ~ N(0, 1) (Q', K' rows
    then divided by their norm, in fp32, before the rounding to bf16), alpha =
    sigmoid(N(2, 1)) per frame and beta = sigmoid(N(0, 1)) * d / P per token (a frame's
    P unit keys act as one step of size about beta * P / d on the state).
    """
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(B, H, T * P, d, generator=g, dtype=torch.float32)
    k = torch.randn(B, H, T * P, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, T * P, d, generator=g, dtype=torch.float32)
    q = q / q.norm(dim=-1, keepdim=True)
    k = k / k.norm(dim=-1, keepdim=True)
    alpha = torch.sigmoid(torch.randn(B, H, T, generator=g, dtype=torch.float32) + 2.0)
    beta = torch.sigmoid(torch.randn(B, H, T * P, generator=g, dtype=torch.float32)) * (d / P)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), alpha, beta
