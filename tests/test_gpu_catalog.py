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


# ------------------------------------------------------------------ similarity term
def _score_sim(tcb, trie, table, user, emb, R, K):
    import torch
    logp = torch.from_numpy(np.ascontiguousarray(table, dtype=np.float32)).cuda()
    u = torch.from_numpy(np.ascontiguousarray(user, dtype=np.float32)).cuda()
    e = torch.from_numpy(np.ascontiguousarray(emb).view(np.int16)).cuda()
    out_s = torch.empty((R, K), device="cuda")
    out_l = torch.empty((R, K), dtype=torch.int32, device="cuda")
    ws = torch.zeros(tcb.catalog_score_workspace_size(trie, R, K), dtype=torch.uint8, device="cuda")
    tcb.catalog_score_topk_sim(trie, logp, u, e, R, K, out_s, out_l, ws)
    assert tcb.sidbeam_get_device_status(ws) == 0
    return out_s.cpu().numpy(), out_l.cpu().numpy()


def _sim_tol(user, emb):
    """TOL plus the fp32 dot-product bound: d * 2^-24 * max_j sum_k |u_k e_jk|."""
    ef = np.abs(host.bf16_bits_to_f32(emb).astype(np.float64))
    worst = (np.abs(user.astype(np.float64)) @ ef.T).max()
    return TOL + user.shape[1] * 2.0 ** -24 * worst


def _check_tol(gs, gl, ref, R, K, tol):
    for r in range(R):
        os_ = ref["score"][r]
        v = int(np.isfinite(os_[:K]).sum())
        assert int(np.isfinite(gs[r]).sum()) == v
        assert np.all(gl[r, v:] == -1)
        np.testing.assert_allclose(gs[r, :v], os_[:v], atol=tol, rtol=0)
        for k in range(v):
            lo = k == 0 or os_[k - 1] - os_[k] > tol
            hi = (not np.isfinite(os_[k + 1])) or os_[k] - os_[k + 1] > tol
            if lo and hi:
                assert gl[r, k] == ref["leaf"][r, k]


def test_catalog_scorer_similarity_config2(tcb):
    """The SPRINT-like workload (32 requests, 50,000 SIDs, top-10) with d = 64
    user and SID vectors."""
    w = WORKLOADS[2]
    cat = w.catalog()
    otrie = oracle.OracleTrie(cat, w.codes_per_level)
    gtrie = tcb.sid_trie_build(cat, w.codes_per_level, w.layouts)
    table = host.table_logits(w.logits_seed, w.R, w.depth, w.V, w.table_sigma)
    user = host.user_vectors(w.sim_seed, w.R, w.sim_dim, w.user_sigma)
    emb = host.sid_embeddings(w.sim_seed, otrie.leaves.shape[0], w.sim_dim, w.emb_sigma)
    gs, gl = _score_sim(tcb, gtrie, table, user, emb, w.R, w.K)
    ref = oracle.catalog_score_topk(otrie, table, w.K + 1, user, emb)
    plain = oracle.catalog_score_topk(otrie, table, w.K)
    assert not np.array_equal(ref["leaf"][:, :w.K], plain["leaf"])  # the term matters here
    _check_tol(gs, gl, ref, w.R, w.K, _sim_tol(user, emb))


@pytest.mark.parametrize("seed", range(6))
def test_catalog_scorer_similarity_random(tcb, seed):
    rng = np.random.default_rng(700 + seed)
    depth = int(rng.integers(1, 4))
    V = int(rng.choice([3, 16, 100, 256]))
    cat = host.draw_catalog(seed, int(min(V ** depth, rng.integers(1, 5000))), [V] * depth)
    otrie = oracle.OracleTrie(cat, [V] * depth)
    gtrie = tcb.sid_trie_build(cat, [V] * depth, None)
    R = int(rng.integers(1, 6))
    K = int(rng.choice([1, 5, 64, 300]))
    d = int(rng.choice([8, 16, 72, 256]))
    table = host.table_logits(900 + seed, R, depth, V, 1.0)
    user = host.user_vectors(900 + seed, R, d, float(rng.uniform(0.1, 2.0)))
    emb = host.sid_embeddings(900 + seed, otrie.leaves.shape[0], d, float(rng.uniform(0.05, 0.5)))
    gs, gl = _score_sim(tcb, gtrie, table, user, emb, R, K)
    ref = oracle.catalog_score_topk(otrie, table, K + 1, user, emb)
    _check_tol(gs, gl, ref, R, K, _sim_tol(user, emb))


def test_catalog_scorer_similarity_argument_checks(tcb):
    import torch
    from trie_constrained_beam_b200 import native
    cat = host.draw_catalog(1, 40, [8, 8])
    gtrie = tcb.sid_trie_build(cat, [8, 8], None)
    N = 40
    logp = torch.zeros((1, 2, 8), device="cuda")
    out_s = torch.empty((1, 4), device="cuda")
    out_l = torch.empty((1, 4), dtype=torch.int32, device="cuda")
    ws = torch.zeros(tcb.catalog_score_workspace_size(gtrie, 1, 4), dtype=torch.uint8, device="cuda")
    u = torch.zeros((1, 12), device="cuda")                       # d % 8 != 0
    e = torch.zeros((N, 12), dtype=torch.int16, device="cuda")
    with pytest.raises(native.SidbeamError) as ex:
        tcb.catalog_score_topk_sim(gtrie, logp, u, e, 1, 4, out_s, out_l, ws)
    assert ex.value.status == native.SIDBEAM_ERR_INVALID_ARG
