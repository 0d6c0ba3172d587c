"""Oracle catalog trie: sorted unique SIDs and per-level sorted prefix lists.

flashrec 0.1.0, Features > Decoding ("SID constraint"): decoding is restricted
to the catalog's valid SIDs through a trie. The oracle keeps no dense or CSR
layout; it keeps, per level l, the sorted list of distinct length-l prefixes.
Node ids are ranks in those sorted lists (the root is node 0 of level 0), so a
node's children are a contiguous, code-sorted run of the next level's list.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import numpy as np


class OracleTrie:
    """Trie over a catalog of SIDs.

    sids: int array [N_in, L], duplicates allowed (they collapse to one leaf).
    codes_per_level: V_l for l = 1..L; every code must lie in [0, V_l).
    """

    def __init__(self, sids, codes_per_level):
        sids = np.asarray(sids, dtype=np.int64)
        if sids.ndim != 2 or sids.shape[0] == 0:
            raise ValueError("sids must be a non-empty [N, L] array")
        self.depth = sids.shape[1]
        self.codes_per_level = [int(v) for v in codes_per_level]
        if len(self.codes_per_level) != self.depth:
            raise ValueError("codes_per_level must have one entry per level")
        for lv in range(self.depth):
            col = sids[:, lv]
            if col.min() < 0 or col.max() >= self.codes_per_level[lv]:
                raise ValueError(f"level {lv + 1} has a code outside [0, V)")

        # Leaves: lexicographically sorted distinct SIDs; leaf_rows[j] is the
        # first input row that carries leaf j (the SID -> item map of a catalog).
        leaves, first = np.unique(sids, axis=0, return_index=True)
        self.leaves = leaves
        self.leaf_rows = first.astype(np.int64)

        # prefixes[l]: distinct length-l prefixes, sorted; prefixes[0] = [()]
        # parent[l][j]: node id (at level l-1) of the parent of node j at level l.
        self.prefixes = [np.zeros((1, 0), dtype=np.int64)]
        self.parent = [np.zeros(0, dtype=np.int64)]
        for lv in range(1, self.depth + 1):
            # leaves are sorted, so equal length-lv prefixes are adjacent and
            # the distinct ones come out already in sorted order.
            head = leaves[:, :lv]
            new_prefix = np.ones(head.shape[0], dtype=bool)
            new_prefix[1:] = np.any(head[1:] != head[:-1], axis=1)
            pre = head[new_prefix]
            self.prefixes.append(pre)
            # Parent id: rank of the length-(lv-1) prefix, which increases by one
            # each time that prefix changes along the sorted list.
            par_changes = np.zeros(pre.shape[0], dtype=np.int64)
            if lv > 1:
                par_changes[1:] = np.any(pre[1:, :lv - 1] != pre[:-1, :lv - 1], axis=1)
            self.parent.append(np.cumsum(par_changes))

    # -------------------------------------------------------------- lookups
    def n_nodes(self, level: int) -> int:
        return self.prefixes[level].shape[0]

    def node_ids(self, level: int, prefixes) -> np.ndarray:
        """Node ids of given length-``level`` prefixes (-1 if absent)."""
        prefixes = np.asarray(prefixes, dtype=np.int64).reshape(-1, level)
        table = self.prefixes[level]
        out = np.full(prefixes.shape[0], -1, dtype=np.int64)
        if level == 0:
            out[:] = 0
            return out
        # Map each prefix row to a tuple key and look it up in a dict built once.
        if not hasattr(self, "_index"):
            self._index = {}
        if level not in self._index:
            self._index[level] = {tuple(row): i for i, row in enumerate(table.tolist())}
        idx = self._index[level]
        for i, row in enumerate(prefixes.tolist()):
            out[i] = idx.get(tuple(row), -1)
        return out

    def children(self, level: int, node: int):
        """Child codes (ascending) and child node ids of ``node`` at ``level``.

        The children of node p at level l are the level-(l+1) prefixes whose
        parent is p; they are contiguous in the sorted list.
        """
        par = self.parent[level + 1]
        lo = np.searchsorted(par, node, side="left")
        hi = np.searchsorted(par, node, side="right")
        ids = np.arange(lo, hi, dtype=np.int64)
        codes = self.prefixes[level + 1][lo:hi, level]
        return codes, ids

    def leaf_of_node(self, node: int) -> int:
        """At the last level, node ids are leaf ids (both are ranks of full SIDs)."""
        return int(node)

    def sid_of_node(self, level: int, node: int) -> np.ndarray:
        return self.prefixes[level][node]
