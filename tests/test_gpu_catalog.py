"""GPU parity of catalog_score_topk (one-pass catalog scorer) against the oracle."""
import numpy as np
import pytest

import oracle
from sidgen import host
from sidgen.workloads import WORKLOADS

from parity import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tcb():
    import trie_constrained_beam_b200 as m
    from trie_constrained_beam_b200 import build
    build.build()
    return m


def _score(tcb, trie, table, R, K):
    import torch
    logp = torch.from_numpy(np.ascontiguousarray(table, dtype=np.float32)).cuda()
    out_s = torch.empty((R, K), device="cuda")
    out_l = torch.empty((R, K), dtype=torch.int32, device="cuda")
    ws = torch.zeros(tcb.catalog_score_workspace_size(trie, R, K), dtype=torch.uint8, device="cuda")
    tcb.catalog_score_topk(trie, logp, R, K, out_s, out_l, ws)
    return out_s.cpu().numpy(), out_l.cpu().numpy()


def _check(gs, gl, ref, R, K):
    for r in range(R):
        os_ = ref["score"][r]
        v = int(np.isfinite(os_[:K]).sum())
        assert int(np.isfinite(gs[r]).sum()) == v
        assert np.all(gl[r, v:] == -1)
        np.testing.assert_allclose(gs[r, :v], os_[:v], atol=TOL, rtol=0)
        for k in range(v):
            lo = k == 0 or os_[k - 1] - os_[k] > TOL
            hi = (not np.isfinite(os_[k + 1])) or os_[k] - os_[k + 1] > TOL
            if lo and hi:
                assert gl[r, k] == ref["leaf"][r, k]


def test_catalog_scorer_config2(tcb):
    w = WORKLOADS[2]
    cat = w.catalog()
    otrie = oracle.OracleTrie(cat, w.codes_per_level)
    gtrie = tcb.sid_trie_build(cat, w.codes_per_level, w.layouts)
    table = host.table_logits(w.logits_seed, w.R, w.depth, w.V, w.table_sigma)
    gs, gl = _score(tcb, gtrie, table, w.R, w.K)
    ref = oracle.catalog_score_topk(otrie, table, w.K + 1)
    _check(gs, gl, ref, w.R, w.K)


@pytest.mark.parametrize("seed", range(8))
def test_catalog_scorer_random(tcb, seed):
    rng = np.random.default_rng(300 + seed)
    depth = int(rng.integers(1, 5))
    Vs = [int(rng.integers(1, 300)) for _ in range(depth)]
    n_cat = int(min(np.prod(Vs), rng.integers(1, 20000)))
    cat = host.draw_catalog(seed, n_cat, Vs)
    otrie = oracle.OracleTrie(cat, Vs)
    gtrie = tcb.sid_trie_build(cat, Vs)
    R = int(rng.integers(1, 6))
    K = int(rng.choice([1, 3, 10, 64, 700]))
    Vmax = max(Vs)
    table = rng.normal(0, 1.5, size=(R, depth, Vmax)).astype(np.float32)
    gs, gl = _score(tcb, gtrie, table, R, K)
    ref = oracle.catalog_score_topk(otrie, table, K + 1)
    _check(gs, gl, ref, R, K)


def test_catalog_scorer_equals_exhaustive_beam(tcb):
    """Prefix-independent log-prob tables: top-K of the scorer equals the top-K
    of a beam search wide enough to keep the whole catalog."""
    import torch
    Vs = [16, 16, 16]
    cat = host.draw_catalog(6, 500, Vs)
    gtrie = tcb.sid_trie_build(cat, Vs)
    R, K = 2, 10
    table = host.table_logits(66, R, 3, 16, 1.5).astype(np.float64)
    lp = np.stack([[oracle.log_softmax_full(table[r, lv]) for lv in range(3)] for r in range(R)])
    gs, gl = _score(tcb, gtrie, lp.astype(np.float32), R, K)
    search = tcb.BeamSearch(gtrie, 1, 500, 16, depth=3)
    for r in range(R):
        def logits_for(t, s, r=r):
            rows = s.rows(t)
            return torch.from_numpy(np.repeat(table[r, t][None].astype(np.float32), rows, 0)).cuda()
        sids, leaf, scores = search.run(logits_for)
        assert leaf[0, :K].cpu().numpy().tolist() == gl[r].tolist()
        np.testing.assert_allclose(scores[0, :K].cpu().numpy(), gs[r], atol=3 * TOL)
