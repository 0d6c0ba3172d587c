"""Oracle one-pass catalog scorer.

SPRINT (paper summary), inference paragraph and closing paragraph: one pass of
the model yields an L-by-M table of per-position token scores; every valid SID
of the prefix trie is scored by the sum of its tokens' log-probabilities and
the top-K are returned. With a user vector per request and an embedding per
SID, the same paragraph's SID-level similarity term is added: the inner
product of the two (one pass gives the table and a user vector; scoring a SID
is a lookup plus one matrix product). The page gives no weight between the
two terms; any scale lives in the user vector.

Parity unpinned against a printed example (the page prints none); pinned by
brute force on tiny catalogs, by the zero-embedding special case (equal to the
token-only scorer) and by the zero-table case (ranking by similarity alone).

Reading: the input table holds per-position log-probabilities (or any
per-position scores; a constant shift per (request, position) shifts every SID
of the request equally and leaves the ranking unchanged). Ties are broken by
leaf id ascending; fewer than K leaves are padded with (-inf, -1).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import numpy as np


def catalog_score_topk(trie, logp, K: int, user=None, sid_emb_bf16_bits=None):
    """logp: [R, L, V] -> dict(score [R, K] float64, leaf [R, K] int64).

    user: optional [R, d] (float); sid_emb_bf16_bits: [N, d] bf16 bits, row j
    the embedding of leaf j. With both, every SID's score also gets
    <user[r], emb[j]> (bf16 widened exactly, products summed in float64)."""
    logp = np.asarray(logp, dtype=np.float64)
    R, L, _ = logp.shape
    leaves = trie.leaves                         # [N, L], leaf id = row index
    N = leaves.shape[0]
    out_score = np.full((R, K), -np.inf)
    out_leaf = np.full((R, K), -1, dtype=np.int64)
    leaf_ids = np.arange(N, dtype=np.int64)
    sim = None
    if user is not None:
        emb = (np.asarray(sid_emb_bf16_bits, dtype=np.uint16).astype(np.uint32) << 16)
        emb = emb.view(np.float32).astype(np.float64)               # [N, d]
        sim = np.asarray(user, dtype=np.float64) @ emb.T             # [R, N]
    for r in range(R):
        total = np.zeros(N)
        for lv in range(L):
            total += logp[r, lv, leaves[:, lv]]
        if sim is not None:
            total = total + sim[r]
        order = np.lexsort((leaf_ids, -total))[:K]
        out_score[r, :order.shape[0]] = total[order]
        out_leaf[r, :order.shape[0]] = order
    return {"score": out_score, "leaf": out_leaf}
