"""Oracle one-pass catalog scorer.

SPRINT (paper summary), inference paragraph and closing paragraph: one pass of
the model yields an L-by-M table of per-position token scores; every valid SID
of the prefix trie is scored by the sum of its tokens' log-probabilities and
the top-K are returned. The SID-level similarity term of that page needs a
trained user vector and is not part of this scorer.

Reading: the input table holds per-position log-probabilities (or any
per-position scores; a constant shift per (request, position) shifts every SID
of the request equally and leaves the ranking unchanged). Ties are broken by
leaf id ascending; fewer than K leaves are padded with (-inf, -1).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import numpy as np


def catalog_score_topk(trie, logp, K: int):
    """logp: [R, L, V] -> dict(score [R, K] float64, leaf [R, K] int64)."""
    logp = np.asarray(logp, dtype=np.float64)
    R, L, _ = logp.shape
    leaves = trie.leaves                         # [N, L], leaf id = row index
    N = leaves.shape[0]
    out_score = np.full((R, K), -np.inf)
    out_leaf = np.full((R, K), -1, dtype=np.int64)
    leaf_ids = np.arange(N, dtype=np.int64)
    for r in range(R):
        total = np.zeros(N)
        for lv in range(L):
            total += logp[r, lv, leaves[:, lv]]
        order = np.lexsort((leaf_ids, -total))[:K]
        out_score[r, :order.shape[0]] = total[order]
        out_leaf[r, :order.shape[0]] = order
    return {"score": out_score, "leaf": out_leaf}
