"""Oracle Gumbel top-k step (sampling without replacement at temperature T > 0).

flashrec 0.1.0 (PyPI page), Features > Serving, "API": deterministic top-k at
temperature 0, Gumbel top-k without replacement above it.

Reading (the page names the method and nothing more): every candidate child c
of parent slot b in request r has its usual score x = s_b + log p(c) (the
full-codebook log-softmax of the deterministic step) and gets the key
x + T * G, with G a standard Gumbel variate drawn for (r, b, c, step); the
n largest keys are kept, ranked by key, ties by (parent asc, code asc). Taking
the n largest of x + T*G draws n candidates without replacement with
probabilities proportional to exp(x / T) (the Gumbel-top-k construction:
argmax of x/T + G is a draw from softmax(x/T), and the next-largest keys
continue the draw from what is left). The beams keep their unperturbed score
x, so the next step adds plain log-probabilities. At T = 0 the keys are the
scores and the step is the deterministic one.

The Gumbel variate: Philox4x32 with ten rounds (Salmon, Moraes, Dror, Shaw,
SC'11, "Parallel random numbers: as easy as 1, 2, 3") on the counter
(r, b, c, step) with the 64-bit seed as key; the top 23 bits of its first
output word, v = u >> 9, give U = (v + 1/2) / 2^23 in (0, 1) (exact in fp32, so a
device in single precision sees the same U) and G = -log(-log U), which lies in
[-2.82, 16.64].

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import numpy as np

from .beam import NEG_INF, _widen, log_softmax_full

# Philox4x32 round constants (multipliers and Weyl key increments) as published.
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85
_LO = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """The four output words for counters (c0..c3) (broadcast arrays) and key (k0, k1)."""
    x = [np.asarray(c, dtype=np.uint64) & _LO for c in (c0, c1, c2, c3)]
    x = [a.copy() for a in np.broadcast_arrays(*x)]
    key0, key1 = k0 & 0xFFFFFFFF, k1 & 0xFFFFFFFF
    for i in range(10):
        if i > 0:  # bump the key between rounds
            key0 = (key0 + _W0) & 0xFFFFFFFF
            key1 = (key1 + _W1) & 0xFFFFFFFF
        prod0 = x[0] * _M0
        prod1 = x[2] * _M1
        x = [(prod1 >> np.uint64(32)) ^ x[1] ^ np.uint64(key0), prod1 & _LO,
             (prod0 >> np.uint64(32)) ^ x[3] ^ np.uint64(key1), prod0 & _LO]
    return tuple(a.astype(np.uint32) for a in x)


def gumbel(seed: int, r, b, code, step: int) -> np.ndarray:
    """Standard Gumbel variates for candidates (r, b, code) of `step` (float64)."""
    u = philox4x32_10(r, b, code, step, seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)[0]
    U = ((u >> np.uint32(9)).astype(np.float64) + 0.5) / 8388608.0
    return -np.log(-np.log(U))


def beam_step_gumbel(trie, step: int, logits, parent_scores, parent_nodes,
                     R: int, B_in: int, n: int, V: int, T: float, seed: int):
    """Gumbel top-k step. Returns dict of arrays [R, n]: score (unperturbed),
    key (score + T*G, the ranking key), parent, code, node."""
    z_all = _widen(logits)
    parent_scores = np.asarray(parent_scores, dtype=np.float64).reshape(-1)
    parent_nodes = np.asarray(parent_nodes, dtype=np.int64).reshape(-1)
    out = {k: np.full((R, n), NEG_INF) for k in ("score", "key")}
    for k in ("parent", "code", "node"):
        out[k] = np.full((R, n), -1, dtype=np.int64)
    for r in range(R):
        sc, ky, pa, co, no = [], [], [], [], []
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
            x = s + logp[codes]
            g = gumbel(seed, r, b, codes, step) if T > 0 else np.zeros(codes.shape[0])
            sc.append(x)
            ky.append(x + T * g)
            pa.append(np.full(codes.shape[0], b, dtype=np.int64))
            co.append(codes)
            no.append(child)
        if not sc:
            continue
        sc, ky, pa, co, no = (np.concatenate(v) for v in (sc, ky, pa, co, no))
        order = np.lexsort((co, pa, -ky))[:n]
        k = order.shape[0]
        out["score"][r, :k] = sc[order]
        out["key"][r, :k] = ky[order]
        out["parent"][r, :k] = pa[order]
        out["code"][r, :k] = co[order]
        out["node"][r, :k] = no[order]
    return out
