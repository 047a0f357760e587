"""LSE merge oracle (numpy float64).  TEST INFRASTRUCTURE ONLY.

"ISPA", §2.1 Dual-Stream Warmup and contribution 2: the log-sum-exp state that
attention kernels keep per row lets attention be split into a local and a
history branch and recombined afterwards.  For disjoint key sets K1, K2 with
partial results (O1, L1) and (O2, L2), where L = ln sum exp(scores):

    L = ln(exp(L1) + exp(L2)) = M + ln(exp(L1 - M) + exp(L2 - M)),  M = max(L1, L2)
    O = exp(L1 - L) * O1 + exp(L2 - L) * O2

which is exactly attention over K1 ∪ K2.  An empty branch has L = -inf and
contributes nothing; both empty gives O = 0, L = -inf.

Parity status: pinned (tests/test_oracle_merge.py: merge of two disjoint
oracle attentions equals the oracle attention over the union; -inf cases).
"""
from __future__ import annotations

import numpy as np


def lse_merge(o1, lse1, o2, lse2):
    o1 = np.asarray(o1, dtype=np.float64)
    o2 = np.asarray(o2, dtype=np.float64)
    l1 = np.asarray(lse1, dtype=np.float64)
    l2 = np.asarray(lse2, dtype=np.float64)
    m = np.maximum(l1, l2)
    both_empty = np.isneginf(m)
    m_safe = np.where(both_empty, 0.0, m)
    with np.errstate(invalid="ignore"):
        w1 = np.where(np.isneginf(l1), 0.0, np.exp(l1 - m_safe))
        w2 = np.where(np.isneginf(l2), 0.0, np.exp(l2 - m_safe))
    total = w1 + w2
    lse = np.where(both_empty, -np.inf, m_safe + np.log(np.where(both_empty, 1.0, total)))
    denom = np.where(both_empty, 1.0, total)
    o = (w1 / denom)[..., None] * o1 + (w2 / denom)[..., None] * o2
    o = np.where(both_empty[..., None], 0.0, o)
    return o, lse
