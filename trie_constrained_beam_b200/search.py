"""Device buffers and the step loop of one constrained beam search.

Orchestration only: every step is one ``beam_step`` call, the end is one
``beam_finalize`` call. Step t reads the previous step's outputs as its parent
rows (B_in = 1 at step 0: the root of every request, score 0), and writes its
back-pointers straight into slice t of the [depth][R][n] history.
"""
from __future__ import annotations

import torch

from . import native


class BeamSearch:
    def __init__(self, trie, R: int, n: int, V, depth: int = None, device="cuda",
                 skip_rows: bool = False, temperature: float = 0.0, seed: int = 0,
                 widths=None):
        """widths: optional per-request beam widths (each <= n); request r keeps
        its widths[r] best beams at every step (the rest of its n slots are
        padding), so one launch per step and one captured graph serve requests
        of different widths."""
        self.trie = trie
        self.skip_rows = skip_rows  # beam_step_ex row skipping (same results)
        # temperature > 0: Gumbel top-k draws (beam_step_gumbel), Philox key `seed`
        self.temperature, self.seed = float(temperature), int(seed)
        self.depth = depth if depth is not None else trie.depth
        self.V = list(V) if isinstance(V, (list, tuple)) else [int(V)] * self.depth
        self.R, self.n = R, n
        dev = torch.device(device)
        self.root_scores = torch.zeros(R, dtype=torch.float32, device=dev)
        self.root_nodes = torch.zeros(R, dtype=torch.int32, device=dev)
        self.scores = torch.empty((self.depth, R * n), dtype=torch.float32, device=dev)
        self.nodes = torch.empty((self.depth, R * n), dtype=torch.int32, device=dev)
        self.bp_parent = torch.empty((self.depth, R, n), dtype=torch.int32, device=dev)
        self.bp_code = torch.empty((self.depth, R, n), dtype=torch.int32, device=dev)
        ws = 0
        for t in range(self.depth):
            size = (native.beam_step_gumbel_workspace_size if self.temperature > 0
                    else native.beam_step_workspace_size)
            ws = max(ws, size(R, 1 if t == 0 else n, n, self.V[t]))
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=dev)
        self.widths = None
        if widths is not None:
            w = [int(x) for x in widths]
            if len(w) != R or min(w) < 0 or max(w) > n:
                raise ValueError("widths: one value in [0, n] per request")
            if self.temperature > 0:
                raise ValueError("widths with temperature > 0 is not supported")
            self.widths = torch.tensor(w, dtype=torch.int32, device=dev)
        self.sids = torch.empty((R, n, self.depth), dtype=torch.int32, device=dev)
        self.leaf = torch.empty((R, n), dtype=torch.int32, device=dev)

    def rows(self, t: int) -> int:
        return self.R * (1 if t == 0 else self.n)

    def parents(self, t: int):
        """(parent_scores, parent_nodes, B_in) of step t."""
        if t == 0:
            return self.root_scores, self.root_nodes, 1
        return self.scores[t - 1], self.nodes[t - 1], self.n

    def step(self, t: int, logits, stream=None):
        ps, pn, B_in = self.parents(t)
        if self.temperature > 0:
            native.beam_step_gumbel(self.trie, t, logits, ps, pn, self.R, B_in, self.n,
                                    self.V[t], self.temperature, self.seed, self.scores[t],
                                    self.bp_parent[t], self.bp_code[t], self.nodes[t],
                                    self.workspace, stream=stream)
            return
        native.beam_step(self.trie, t, logits, ps, pn, self.R, B_in, self.n, self.V[t],
                         self.scores[t], self.bp_parent[t], self.bp_code[t], self.nodes[t],
                         self.workspace, stream=stream, skip_rows=self.skip_rows,
                         out_width=self.widths)

    def skipped_rows(self, stream=None) -> int:
        """Rows left unread by row skipping since the last call."""
        return native.beam_step_skipped_rows(self.workspace, stream=stream)

    def finalize(self, stream=None):
        native.beam_finalize(self.depth, self.R, self.n, self.bp_parent, self.bp_code,
                             self.nodes[self.depth - 1], self.sids, self.leaf, stream=stream)
        return self.sids, self.leaf, self.scores[self.depth - 1].view(self.R, self.n)

    def capture(self, logits_per_step, events=None):
        """A CUDA graph of the whole search (every beam_step, then beam_finalize)
        on fixed logits tensors; ``graph.replay()`` runs it on the current stream.

        Call the search once eagerly first (that sets the kernels' shared-memory
        limits outside the capture). ``events``: optional depth + 2 events made
        with ``enable_timing=True, external=True``, recorded before every step,
        before finalize and at the end (per-step device times of a replay).
        """
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=side):
            for t in range(self.depth):
                if events is not None:
                    events[t].record()
                self.step(t, logits_per_step[t])
            if events is not None:
                events[self.depth].record()
            self.finalize()
            if events is not None:
                events[self.depth + 1].record()
        torch.cuda.current_stream().wait_stream(side)
        return g

    def run(self, logits_for_step, stream=None):
        """logits_for_step(t, search) -> logits tensor [rows(t), ld] for step t."""
        for t in range(self.depth):
            self.step(t, logits_for_step(t, self), stream=stream)
        return self.finalize(stream=stream)
