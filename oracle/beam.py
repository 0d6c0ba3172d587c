"""Oracle beam step, beam search and finalize (float64, plain loops).

What one step computes (flashrec 0.1.0, introduction and Features > Decoding;
the readings below fill in what the page leaves open):

For every live beam row b of request r, with parent score s_b and trie node p_b:
  1. lse_b = log sum_{c < V} exp(z_bc) over the level's FULL codebook
     (log-probabilities of the whole SID token range; invalid codes are masked
     to -inf afterwards, with no renormalisation over the valid children);
  2. every valid child code c of p_b (ascending) becomes a candidate with
     score s_b + (z_bc - lse_b), parent slot b, code c, child node id;
  3. the request's candidates are ordered by (score desc, parent asc, code asc)
     -- "deterministic top-k at temperature 0" (Features > Serving, "API") with
     the tie-break made explicit -- and the first n are kept, best first;
  4. missing entries (fewer than n candidates) are (-inf, -1, -1, -1).

A row is dead (skipped, its logits never looked at) when its parent score is
-inf or its node is negative. At step 0 each request has one live row: the
root (node 0, score 0). Without a trie (``trie is None``) every code of the
level is valid and child node ids are -1 (Quickstart: with no catalog the
engine decodes the full vocabulary).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def log_softmax_full(z: np.ndarray) -> np.ndarray:
    """log-softmax over every entry of z, in float64 (max-shifted log-sum-exp)."""
    z = np.asarray(z, dtype=np.float64)
    m = np.max(z)
    lse = m + np.log(np.sum(np.exp(z - m)))
    return z - lse


def _widen(logits) -> np.ndarray:
    """Logits as float64: fp32 values, or bf16 given as uint16 bit patterns."""
    a = np.asarray(logits)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def beam_step(trie, step: int, logits, parent_scores, parent_nodes,
              R: int, B_in: int, n: int, V: int):
    """One expansion step. Returns dict of arrays [R, n]: score, parent, code, node.

    logits: [R*B_in, >= V] (float32 / float64, or uint16 bf16 bits), row-major,
            row = r*B_in + b; only the first V columns are used.
    parent_scores, parent_nodes: [R*B_in].
    """
    z_all = _widen(logits)
    parent_scores = np.asarray(parent_scores, dtype=np.float64).reshape(-1)
    parent_nodes = np.asarray(parent_nodes, dtype=np.int64).reshape(-1)
    out_score = np.full((R, n), NEG_INF)
    out_parent = np.full((R, n), -1, dtype=np.int64)
    out_code = np.full((R, n), -1, dtype=np.int64)
    out_node = np.full((R, n), -1, dtype=np.int64)

    for r in range(R):
        sc, pa, co, no = [], [], [], []
        for b in range(B_in):
            row = r * B_in + b
            s = parent_scores[row]
            p = parent_nodes[row]
            if s == NEG_INF or (trie is not None and p < 0):
                continue
            logp = log_softmax_full(z_all[row, :V])
            if trie is None:
                codes = np.arange(V, dtype=np.int64)
                child = np.full(V, -1, dtype=np.int64)
            else:
                codes, child = trie.children(step, int(p))
            sc.append(s + logp[codes])
            pa.append(np.full(codes.shape[0], b, dtype=np.int64))
            co.append(codes)
            no.append(child)
        if not sc:
            continue
        sc, pa, co, no = (np.concatenate(x) for x in (sc, pa, co, no))
        # Primary key score descending, then parent ascending, then code ascending.
        order = np.lexsort((co, pa, -sc))[:n]
        k = order.shape[0]
        out_score[r, :k] = sc[order]
        out_parent[r, :k] = pa[order]
        out_code[r, :k] = co[order]
        out_node[r, :k] = no[order]
    return {"score": out_score, "parent": out_parent, "code": out_code, "node": out_node}


def beam_finalize(bp_parent, bp_code, last_score, last_node):
    """Backtrack back-pointers into ranked SIDs.

    bp_parent, bp_code: [depth, R, n] (step t's parent slot and code per output rank).
    Returns sids [R, n, depth], leaf [R, n] (the last step's node id), score [R, n].
    Padded beams (code -1 at the last step) come back as all -1 with score -inf.
    """
    bp_parent = np.asarray(bp_parent)
    bp_code = np.asarray(bp_code)
    depth, R, n = bp_parent.shape
    sids = np.full((R, n, depth), -1, dtype=np.int64)
    leaf = np.full((R, n), -1, dtype=np.int64)
    score = np.full((R, n), NEG_INF)
    for r in range(R):
        for k in range(n):
            if bp_code[depth - 1, r, k] < 0:
                continue
            slot = k
            for t in range(depth - 1, -1, -1):
                sids[r, k, t] = bp_code[t, r, slot]
                slot = bp_parent[t, r, slot]
            leaf[r, k] = last_node[r, k]
            score[r, k] = last_score[r, k]
    return {"sids": sids, "leaf": leaf, "score": score}


def beam_search(trie, R: int, n: int, depth: int, V: int, logits_for_rows, widths=None):
    """Full constrained beam search from the root.

    logits_for_rows(step, prefixes, requests) -> logits [rows, V] for the given
    live prefixes (int array [rows, step]) of the given requests (int array
    [rows]); dead rows are never asked for.
    widths: optional beams per request (each <= n): after every step request r
    keeps its widths[r] best and the rest of its n slots become padding
    (several requests of different widths sharing one step, flashrec 0.1.0,
    Features > Decoding, "Scheduling").
    Returns finalize's dict plus per-step outputs (``steps``).
    """
    parent_scores = np.zeros(R)                    # step 0: one root row per request
    parent_nodes = np.zeros(R, dtype=np.int64)
    prefixes = np.zeros((R, 1, 0), dtype=np.int64)  # [R, B_in, step]
    B_in = 1
    steps = []
    for t in range(depth):
        live = parent_scores.reshape(R, B_in) > NEG_INF
        logits = np.zeros((R * B_in, V))
        flat_live = np.flatnonzero(live.reshape(-1))
        if flat_live.size:
            logits[flat_live] = _widen(
                logits_for_rows(t, prefixes.reshape(R * B_in, t)[flat_live],
                                flat_live // B_in))[:, :V]
        out = beam_step(trie, t, logits, parent_scores, parent_nodes, R, B_in, n, V)
        if widths is not None:
            for r, w in enumerate(widths):
                out["score"][r, w:] = NEG_INF
                for k in ("parent", "code", "node"):
                    out[k][r, w:] = -1
        steps.append(out)
        new_prefixes = np.full((R, n, t + 1), -1, dtype=np.int64)
        for r in range(R):
            for k in range(n):
                p = out["parent"][r, k]
                if p < 0:
                    continue
                new_prefixes[r, k, :t] = prefixes[r, p]
                new_prefixes[r, k, t] = out["code"][r, k]
        prefixes = new_prefixes
        parent_scores = out["score"].reshape(-1)
        parent_nodes = out["node"].reshape(-1)
        B_in = n
    bp_parent = np.stack([s["parent"] for s in steps])
    bp_code = np.stack([s["code"] for s in steps])
    res = beam_finalize(bp_parent, bp_code, steps[-1]["score"], steps[-1]["node"])
    res["steps"] = steps
    return res
