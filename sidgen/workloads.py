"""The five synthetic workloads (shapes, distributions, seeds).

They stand in for the pages' workloads (RecIF-Bench / OneRec traffic, Sohu
traffic, Amazon/Yelp catalogs), none of which is available: SID depth 3-5,
codebooks of 256-8192 codes, beam widths 8-512 across concurrent requests,
catalogs from thousands to millions of SIDs. Seeds: catalog 1000*c + 1,
logits / hidden states 1000*c + 2, lm_head weight 1000*c + 3, user and SID
vectors of the catalog scorer's similarity term 1000*c + 4. Every request's
prefix-hash chain starts from its own root (``host.request_roots``), so concurrent
requests search different logits.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np

from . import host

DENSE, CSR, AUTO = 1, 2, 0


@dataclass
class Workload:
    name: str
    cfg: int
    R: int
    n: int
    depth: int
    V: int
    n_sids: int
    dists: Sequence
    layouts: Optional[List[int]]
    dtype: str            # "f32" or "bf16"
    sigma: float
    K: int = 0            # catalog scorer top-K (0 = not part of the workload)
    table_sigma: float = 0.0
    sim_dim: int = 0      # catalog scorer's SID-level similarity term (user / SID vectors)
    user_sigma: float = 1.0
    emb_sigma: float = 0.25
    hidden_dim: int = 0   # fused lm_head variant
    hidden_sigma: float = 1.0
    weight_sigma: float = 0.02
    notes: str = ""

    @property
    def catalog_seed(self) -> int:
        return 1000 * self.cfg + 1

    @property
    def logits_seed(self) -> int:
        return 1000 * self.cfg + 2

    @property
    def weight_seed(self) -> int:
        return 1000 * self.cfg + 3

    @property
    def sim_seed(self) -> int:
        return 1000 * self.cfg + 4

    @property
    def codes_per_level(self) -> List[int]:
        return [self.V] * self.depth

    def catalog(self) -> np.ndarray:
        return host.draw_catalog(self.catalog_seed, self.n_sids, self.codes_per_level, self.dists)


WORKLOADS = {
    1: Workload("tiny-exhaustive: 1 req x beam 8, depth 3, V=32, 2k SIDs, CSR, fp32", 1,
                R=1, n=8, depth=3, V=32, n_sids=2000, dists=["uniform"] * 3,
                layouts=[CSR] * 3, dtype="f32", sigma=2.0),
    2: Workload("sprint-opq: 32 req x beam 32, depth 4, V=256, 50k SIDs, fp32 + top-10 scorer", 2,
                R=32, n=32, depth=4, V=256, n_sids=50_000, dists=["uniform"] * 4,
                layouts=None, dtype="f32", sigma=1.5, K=10, table_sigma=1.5, sim_dim=64),
    3: Workload("flashrec-concurrency: 64 req x beam 128, depth 3, V=8192, 1M SIDs, CSR, bf16", 3,
                R=64, n=128, depth=3, V=8192, n_sids=1_000_000,
                dists=[("zipf", 1.1), "uniform", "uniform"], layouts=[CSR] * 3, dtype="bf16",
                sigma=3.0),
    4: Workload("wide-beam: 16 req x beam 512, depth 5, V=4096, 8M SIDs, dense L1-2 + CSR L3-5, bf16", 4,
                R=16, n=512, depth=5, V=4096, n_sids=8_000_000,
                dists=[("zipf", 1.2), ("zipf", 1.2), "uniform", "uniform", "uniform"],
                layouts=[DENSE, DENSE, CSR, CSR, CSR], dtype="bf16", sigma=3.0),
    5: Workload("fused-lmhead: 32 req x beam 128, depth 3, V=8192, d=2048, 1M SIDs, bf16", 5,
                R=32, n=128, depth=3, V=8192, n_sids=1_000_000,
                dists=[("zipf", 1.1), "uniform", "uniform"], layouts=None, dtype="bf16",
                sigma=0.0, hidden_dim=2048),
}
