"""Pins that tie the oracle to something other than itself.

* brute force: exhaustive enumeration of every catalog SID with torch's
  float64 log_softmax must equal beam search whenever the beam is at least as
  wide as the catalog (the search then drops nothing);
* library special cases: without a trie a step is torch.topk over
  parent score + torch.log_softmax; lse matches torch.logsumexp; a complete
  catalog gives the trie-free result;
* hand-derived tie cases (all logits equal);
* closed forms: one-hot hidden states pick a weight column exactly; the
  catalog scorer equals beam search under prefix-independent logits;
* invariants: every beam is a catalog leaf, scores never increase along ranks
  or lineages, valid-child probabilities sum to at most one.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from sidgen import host


def _gen_logits_fn(seed, V, sigma):
    def fn(step, prefixes, requests=None):
        return host.row_logits(seed, host.prefix_hashes(prefixes, requests), V, sigma)
    return fn


def _exhaustive(trie, V, logits_fn):
    """Score every catalog SID by summing torch float64 log_softmax terms."""
    leaves = trie.leaves
    L = leaves.shape[1]
    total = np.zeros(leaves.shape[0])
    for lv in range(L):
        z = logits_fn(lv, leaves[:, :lv]).astype(np.float64)
        lp = torch.log_softmax(torch.from_numpy(z), dim=1).numpy()
        total += lp[np.arange(leaves.shape[0]), leaves[:, lv]]
    return total


# ------------------------------------------------------------------ trie
def test_trie_round_trip_and_ids():
    sids = np.array([[2, 1, 0], [0, 3, 1], [2, 1, 0], [0, 3, 0], [1, 0, 2], [0, 0, 0]])
    t = oracle.OracleTrie(sids, [3, 4, 3])
    # Leaves: sorted unique input; leaf_rows point at the first occurrence.
    expect = sorted({tuple(r) for r in sids.tolist()})
    assert [tuple(r) for r in t.leaves.tolist()] == expect
    for j, row in enumerate(t.leaf_rows):
        assert tuple(sids[row]) == expect[j]
        assert all(tuple(sids[k]) != expect[j] for k in range(row))
    # Node counts per level, worked by hand: level-1 {0,1,2}; level-2
    # {(0,0),(0,3),(1,0),(2,1)}; level-3 = the 5 leaves.
    assert [t.n_nodes(lv) for lv in range(4)] == [1, 3, 4, 5]
    codes, ids = t.children(1, 0)              # children of prefix (0,)
    assert codes.tolist() == [0, 3] and ids.tolist() == [0, 1]
    codes, ids = t.children(2, 1)              # children of prefix (0,3)
    assert codes.tolist() == [0, 1] and ids.tolist() == [1, 2]
    # Every node's prefix extends its parent's prefix.
    for lv in range(1, 4):
        for j in range(t.n_nodes(lv)):
            p = t.parent[lv][j]
            assert tuple(t.sid_of_node(lv, j)[:lv - 1]) == tuple(t.sid_of_node(lv - 1, p))


def test_trie_rejects_out_of_range_codes():
    with pytest.raises(ValueError):
        oracle.OracleTrie(np.array([[0, 5]]), [4, 4])


# ------------------------------------------------------------------ brute force
def test_exhaustive_equals_beam_search_config1_shape():
    cat = host.draw_catalog(1001, 2000, [32, 32, 32])
    trie = oracle.OracleTrie(cat, [32, 32, 32])
    fn = _gen_logits_fn(1002, 32, 2.0)
    res = oracle.beam_search(trie, 1, 2000, 3, 32, fn)
    brute = _exhaustive(trie, 32, fn)
    order = np.argsort(-brute, kind="stable")
    # Continuous scores: no exact ties in this fixture, so the order is unique.
    assert np.all(np.diff(brute[order]) < 0)
    got_sids = res["sids"][0]
    assert np.array_equal(got_sids, trie.leaves[order])
    np.testing.assert_allclose(res["score"][0], brute[order], rtol=0, atol=1e-12)
    assert np.array_equal(res["leaf"][0], order)


@pytest.mark.parametrize("case", range(25))
def test_exhaustive_equals_beam_search_random_tiny(case):
    rng = np.random.default_rng(1000 + case)
    L = int(rng.integers(1, 5))
    Vs = [int(v) for v in rng.integers(2, 7, size=L)]
    n_cat = int(rng.integers(1, min(64, int(np.prod(Vs))) + 1))
    cat = host.draw_catalog(case, n_cat, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    V = max(Vs)
    fn = _gen_logits_fn(77 + case, V, 1.7)

    def fn_level(step, prefixes, requests=None):  # per-level codebook: first V_l codes only
        return fn(step, prefixes, requests)[:, :Vs[step]]

    R = 1
    n = n_cat + int(rng.integers(0, 4))
    # Step through by hand with per-level V (the oracle step takes V per call).
    scores = np.zeros(R)
    nodes = np.zeros(R, dtype=np.int64)
    prefixes = np.zeros((1, 0), dtype=np.int64)
    B_in = 1
    bpp, bpc = [], []
    for t in range(L):
        live = scores > -np.inf
        z = np.zeros((R * B_in, Vs[t]))
        z[live] = fn_level(t, prefixes[live])
        out = oracle.beam_step(trie, t, z, scores, nodes, R, B_in, n, Vs[t])
        bpp.append(out["parent"])
        bpc.append(out["code"])
        newp = np.full((n, t + 1), -1, dtype=np.int64)
        for k in range(n):
            if out["parent"][0, k] >= 0:
                newp[k, :t] = prefixes[out["parent"][0, k]]
                newp[k, t] = out["code"][0, k]
        prefixes, scores, nodes, B_in = newp, out["score"].reshape(-1), out["node"].reshape(-1), n
    fin = oracle.beam_finalize(np.stack(bpp), np.stack(bpc), out["score"], out["node"])
    brute = np.zeros(trie.leaves.shape[0])
    for lv in range(L):
        zz = fn_level(lv, trie.leaves[:, :lv]).astype(np.float64)
        lp = torch.log_softmax(torch.from_numpy(zz), dim=1).numpy()
        brute += lp[np.arange(trie.leaves.shape[0]), trie.leaves[:, lv]]
    order = np.argsort(-brute, kind="stable")
    k = trie.leaves.shape[0]
    np.testing.assert_allclose(fin["score"][0, :k], brute[order], atol=1e-12, rtol=0)
    assert {tuple(s) for s in fin["sids"][0, :k].tolist()} == {tuple(s) for s in trie.leaves.tolist()}
    # Padding past the catalog size.
    assert np.all(fin["score"][0, k:] == -np.inf) and np.all(fin["sids"][0, k:] == -1)


# ------------------------------------------------------------------ library special cases
def test_log_softmax_matches_torch_logsumexp():
    rng = np.random.default_rng(3)
    for V in (1, 2, 31, 4096):
        z = rng.normal(0, 3, size=V) * (10 if V == 31 else 1)
        ref = z - torch.logsumexp(torch.from_numpy(z), dim=0).item()
        np.testing.assert_allclose(oracle.log_softmax_full(z), ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("R,B_in,n,V", [(1, 1, 5, 7), (3, 4, 9, 16), (2, 6, 40, 33)])
def test_unconstrained_step_is_topk_of_log_softmax(R, B_in, n, V):
    rng = np.random.default_rng(R * 100 + V)
    z = rng.normal(0, 2, size=(R * B_in, V)).astype(np.float32)
    s = rng.normal(-3, 1, size=R * B_in)
    s[1 % (R * B_in)] = -np.inf                      # one dead row
    out = oracle.beam_step(None, 0, z, s, np.zeros(R * B_in, dtype=np.int64), R, B_in, n, V)
    lp = torch.log_softmax(torch.from_numpy(z.astype(np.float64)), dim=1)
    cand = (torch.from_numpy(s)[:, None] + lp).reshape(R, B_in * V)
    vals, idx = torch.topk(cand, n, dim=1)
    for r in range(R):
        live = torch.isfinite(vals[r])
        k = int(live.sum())
        np.testing.assert_allclose(out["score"][r, :k], vals[r, :k].numpy(), atol=1e-12, rtol=0)
        assert out["parent"][r, :k].tolist() == (idx[r, :k] // V).tolist()
        assert out["code"][r, :k].tolist() == (idx[r, :k] % V).tolist()
        assert np.all(out["score"][r, k:] == -np.inf) and np.all(out["parent"][r, k:] == -1)
        assert np.all(out["node"][r] == -1)


def test_complete_catalog_equals_unconstrained():
    Vs = [4, 5, 3]
    allsids = np.array(list(itertools.product(*[range(v) for v in Vs])))
    trie = oracle.OracleTrie(allsids[::-1], Vs)
    rng = np.random.default_rng(8)
    R, B_in, n = 2, 4, 6
    for step, V in enumerate(Vs):
        z = rng.normal(0, 1, size=(R * B_in, V))
        s = rng.normal(-2, 1, size=R * B_in)
        nodes = rng.integers(0, trie.n_nodes(step), size=R * B_in)
        a = oracle.beam_step(trie, step, z, s, nodes, R, B_in, n, V)
        b = oracle.beam_step(None, step, z, s, nodes, R, B_in, n, V)
        for key in ("score", "parent", "code"):
            assert np.array_equal(a[key], b[key])


# ------------------------------------------------------------------ hand-derived ties
def test_all_equal_logits_pick_lexicographic_first():
    # Catalog over V=4: (0,1) (0,3) (1,0) (2,2) (2,3) (3,1).
    sids = np.array([[2, 3], [0, 1], [3, 1], [1, 0], [0, 3], [2, 2]])
    trie = oracle.OracleTrie(sids, [4, 4])
    V, n = 4, 3
    # Step 0: root row, all 4 codes valid, equal scores -log 4 -> codes 0,1,2 in order.
    o0 = oracle.beam_step(trie, 0, np.zeros((1, V)), [0.0], [0], 1, 1, n, V)
    assert o0["code"][0].tolist() == [0, 1, 2]
    assert o0["parent"][0].tolist() == [0, 0, 0]
    assert o0["node"][0].tolist() == [0, 1, 2]
    np.testing.assert_allclose(o0["score"][0], [-np.log(4)] * 3, atol=1e-15)
    # Step 1: parents (0,) (1,) (2,) with equal scores; children in (parent, code)
    # order: (0,1) (0,3) (1,0) (2,2) (2,3) -> keep the first three.
    o1 = oracle.beam_step(trie, 1, np.zeros((3, V)), o0["score"][0], o0["node"][0], 1, 3, n, V)
    assert o1["parent"][0].tolist() == [0, 0, 1]
    assert o1["code"][0].tolist() == [1, 3, 0]
    assert o1["node"][0].tolist() == [0, 1, 2]
    # A higher parent score wins over the parent-slot tie-break.
    sc = np.array([-1.0, -0.5, -1.0])
    o2 = oracle.beam_step(trie, 1, np.zeros((3, V)), sc, [0, 1, 2], 1, 3, n, V)
    assert o2["parent"][0].tolist() == [1, 0, 0] and o2["code"][0].tolist() == [0, 1, 3]


def test_dead_rows_and_padding():
    sids = np.array([[0, 0], [0, 1], [1, 0]])
    trie = oracle.OracleTrie(sids, [2, 2])
    z = np.array([[100.0, 0.0], [0.0, 0.0]])
    out = oracle.beam_step(trie, 1, z, [-np.inf, -1.0], [0, 1], 1, 2, 4, 2)
    # Row 0 is dead (score -inf): its huge logit never matters. Row 1 (node (1,))
    # has one child, code 0: score -1 + log(1/2).
    assert out["parent"][0].tolist() == [1, -1, -1, -1]
    assert out["code"][0].tolist() == [0, -1, -1, -1]
    assert out["node"][0].tolist() == [2, -1, -1, -1]
    np.testing.assert_allclose(out["score"][0, 0], -1.0 - np.log(2.0), atol=1e-15)
    assert np.all(out["score"][0, 1:] == -np.inf)


def test_finalize_hand_example():
    # depth 3, R=1, n=2. Step 0 codes [5,6]; step 1 rank0 <- slot1 code 7, rank1 <- slot0 code 8;
    # step 2 rank0 <- slot1 code 9, rank1 padded.
    bp_parent = np.array([[[0, 0]], [[1, 0]], [[1, -1]]])
    bp_code = np.array([[[5, 6]], [[7, 8]], [[9, -1]]])
    fin = oracle.beam_finalize(bp_parent, bp_code, np.array([[-1.5, -np.inf]]), np.array([[42, -1]]))
    # rank 0 at step 2 came from step-1 rank 1 (code 8), which came from step-0 rank 0 (code 5).
    assert fin["sids"][0].tolist() == [[5, 8, 9], [-1, -1, -1]]
    assert fin["leaf"][0].tolist() == [42, -1]
    assert fin["score"][0, 0] == -1.5 and fin["score"][0, 1] == -np.inf


# ------------------------------------------------------------------ invariants
def test_invariants_on_config2_shape():
    Vs = [256] * 4
    cat = host.draw_catalog(2001, 50_000, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    catalog = {tuple(r) for r in trie.leaves.tolist()}
    fn = _gen_logits_fn(2002, 256, 1.5)
    R, n = 4, 32
    res = oracle.beam_search(trie, R, n, 4, 256, fn)
    for r in range(R):
        for k in range(n):
            assert tuple(res["sids"][r, k]) in catalog                  # invalid rate 0
            assert res["leaf"][r, k] == trie.node_ids(4, res["sids"][r, k][None])[0]
        assert np.all(np.diff(res["score"][r]) <= 0)                     # ranked best first
    for t in range(1, 4):
        prev, cur = res["steps"][t - 1], res["steps"][t]
        for r in range(R):
            for k in range(n):
                assert cur["score"][r, k] <= prev["score"][r, cur["parent"][r, k]]


def test_valid_child_mass_at_most_one():
    cat = host.draw_catalog(5, 300, [8, 8, 8])
    trie = oracle.OracleTrie(cat, [8, 8, 8])
    rng = np.random.default_rng(2)
    for lv in range(3):
        for node in range(trie.n_nodes(lv)):
            z = rng.normal(0, 2, size=8)
            codes, _ = trie.children(lv, node)
            mass = np.exp(oracle.log_softmax_full(z)[codes]).sum()
            assert mass <= 1.0 + 1e-12
            if codes.shape[0] == 8:
                assert abs(mass - 1.0) < 1e-12


# ------------------------------------------------------------------ catalog scorer
def test_catalog_scorer_brute_force_tiny():
    Vs = [3, 4, 2]
    cat = host.draw_catalog(4, 15, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    rng = np.random.default_rng(4)
    logp = rng.normal(0, 1, size=(2, 3, 4))
    K = 20
    res = oracle.catalog_score_topk(trie, logp, K)
    for r in range(2):
        items = []
        for j, sid in enumerate(trie.leaves.tolist()):
            items.append((sum(logp[r, lv, c] for lv, c in enumerate(sid)), j))
        items.sort(key=lambda x: (-x[0], x[1]))
        k = len(items)
        assert res["leaf"][r, :k].tolist() == [j for _, j in items]
        np.testing.assert_allclose(res["score"][r, :k], [s for s, _ in items], atol=1e-12)
        assert np.all(res["leaf"][r, k:] == -1) and np.all(res["score"][r, k:] == -np.inf)


def test_catalog_scorer_equals_beam_search_prefix_independent():
    Vs = [16, 16, 16]
    cat = host.draw_catalog(6, 500, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    R, K = 3, 10
    table = host.table_logits(66, R, 3, 16, 1.5).astype(np.float64)
    lp = np.stack([[oracle.log_softmax_full(table[r, lv]) for lv in range(3)] for r in range(R)])
    sc = oracle.catalog_score_topk(trie, lp, K)
    for r in range(R):
        def fn(step, prefixes, requests, r=r):  # logits depend on the level only
            return np.repeat(table[r, step][None], prefixes.shape[0], axis=0)
        bs = oracle.beam_search(trie, 1, 500, 3, 16, fn)
        assert bs["leaf"][0, :K].tolist() == sc["leaf"][r].tolist()
        np.testing.assert_allclose(bs["score"][0, :K], sc["score"][r], atol=1e-12)


def test_catalog_scorer_similarity_brute_force_tiny():
    """Token sum plus <user, sid embedding>, written out with Python loops per
    (request, SID); the term must change the ranking somewhere."""
    Vs = [3, 4, 2]
    cat = host.draw_catalog(4, 15, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    rng = np.random.default_rng(5)
    logp = rng.normal(0, 1, size=(3, 3, 4))
    d = 8
    user = host.user_vectors(77, 3, d, 1.0)
    emb = host.sid_embeddings(77, trie.leaves.shape[0], d, 0.5)
    ef = host.bf16_bits_to_f32(emb)
    K = 20
    res = oracle.catalog_score_topk(trie, logp, K, user, emb)
    plain = oracle.catalog_score_topk(trie, logp, K)
    changed = False
    for r in range(3):
        items = []
        for j, sid in enumerate(trie.leaves.tolist()):
            tok = sum(logp[r, lv, c] for lv, c in enumerate(sid))
            dot = sum(float(user[r, k]) * float(ef[j, k]) for k in range(d))
            items.append((tok + dot, j))
        items.sort(key=lambda x: (-x[0], x[1]))
        k = len(items)
        assert res["leaf"][r, :k].tolist() == [j for _, j in items]
        np.testing.assert_allclose(res["score"][r, :k], [x for x, _ in items], atol=1e-12)
        changed |= res["leaf"][r, :k].tolist() != plain["leaf"][r, :k].tolist()
    assert changed


def test_catalog_scorer_zero_embeddings_is_token_only():
    Vs = [16, 16, 16]
    cat = host.draw_catalog(6, 500, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    table = host.table_logits(66, 2, 3, 16, 1.5)
    user = host.user_vectors(66, 2, 16, 1.0)
    zero = np.zeros((trie.leaves.shape[0], 16), dtype=np.uint16)   # bf16 +0.0
    a = oracle.catalog_score_topk(trie, table, 10, user, zero)
    b = oracle.catalog_score_topk(trie, table, 10)
    assert np.array_equal(a["leaf"], b["leaf"]) and np.array_equal(a["score"], b["score"])


def test_catalog_scorer_zero_table_ranks_by_similarity():
    """With every token log-probability 0 the ranking is the similarity's alone:
    the SIDs sorted by the dot product, written out per SID."""
    Vs = [8, 8]
    cat = host.draw_catalog(12, 40, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    d = 16
    user = host.user_vectors(12, 2, d, 1.0)
    emb = host.sid_embeddings(12, trie.leaves.shape[0], d, 0.3)
    ef = host.bf16_bits_to_f32(emb)
    res = oracle.catalog_score_topk(trie, np.zeros((2, 2, 8)), 40, user, emb)
    for r in range(2):
        dots = [(sum(float(user[r, k]) * float(ef[j, k]) for k in range(d)), j)
                for j in range(trie.leaves.shape[0])]
        dots.sort(key=lambda x: (-x[0], x[1]))
        assert res["leaf"][r].tolist() == [j for _, j in dots]


def _random_step_case(seed, V=24, n_cat=400, R=3, B_in=20):
    rng = np.random.default_rng(seed)
    cat = host.draw_catalog(seed, n_cat, [V, V])
    trie = oracle.OracleTrie(cat, [V, V])
    z = rng.normal(0, 2, size=(R * B_in, V))
    ps = np.concatenate([np.sort(rng.uniform(-9, -1, size=B_in))[::-1] for _ in range(R)])
    pn = rng.integers(0, trie.n_nodes(1), size=R * B_in)
    return trie, z, ps, pn, R, B_in, V


@pytest.mark.parametrize("seed", range(4))
def test_rows_below_the_nth_best_never_contribute(seed):
    """The fact row skipping rests on: a child's score never exceeds its
    parent's (log p <= 0), so dropping every row whose parent score is below
    the request's n-th best child leaves the step's result unchanged."""
    trie, z, ps, pn, R, B_in, V = _random_step_case(200 + seed)
    n = 8
    full = oracle.beam_step(trie, 1, z, ps, pn, R, B_in, n, V)
    cut = ps.copy()
    for r in range(R):
        kth = full["score"][r, n - 1]
        rows = slice(r * B_in, (r + 1) * B_in)
        cut[rows] = np.where(ps[rows] < kth, -np.inf, ps[rows])
    assert np.isneginf(cut).any()          # the case does drop rows
    pruned = oracle.beam_step(trie, 1, z, cut, pn, R, B_in, n, V)
    for k in ("score", "parent", "code", "node"):
        assert np.array_equal(full[k], pruned[k])


def test_top_w_is_the_first_w_ranks_of_top_n():
    """The fact per-request widths rest on: the best w candidates of a request
    are the first w ranks of its best n (n >= w), ties included."""
    trie, z, ps, pn, R, B_in, V = _random_step_case(300)
    z = np.round(z * 2) / 2                 # coarse grid: many exact ties
    wide = oracle.beam_step(trie, 1, z, ps, pn, R, B_in, 40, V)
    for w in (1, 7, 23, 40):
        narrow = oracle.beam_step(trie, 1, z, ps, pn, R, B_in, w, V)
        for k in ("score", "parent", "code", "node"):
            assert np.array_equal(wide[k][:, :w], narrow[k])


def test_search_with_widths_equals_separate_searches():
    """Requests of different widths in one search give, request by request, the
    search of that request alone at its own width (padding past the width)."""
    Vs = [8, 8, 8]
    cat = host.draw_catalog(31, 300, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    table = host.table_logits(31, 3, 3, 8, 1.5)

    def fn_for(reqs_map):
        def fn(step, prefixes, requests):
            return np.stack([table[reqs_map[q], step] + 0.01 * prefixes.sum(axis=1)[i]
                             for i, q in enumerate(requests)])
        return fn

    widths = [6, 2, 4]
    res = oracle.beam_search(trie, 3, 6, 3, 8, fn_for([0, 1, 2]), widths=widths)
    for r, w in enumerate(widths):
        one = oracle.beam_search(trie, 1, w, 3, 8, fn_for([r]))
        assert np.array_equal(res["sids"][r, :w], one["sids"][0])
        assert np.array_equal(res["score"][r, :w], one["score"][0])
        assert np.all(res["leaf"][r, w:] == -1)


# ------------------------------------------------------------------ Gumbel top-k
def test_oracle_philox_known_answers():
    """The oracle's own Philox4x32-10 against the published known-answer vectors."""
    for cols in _kat_rows():
        v = [int(x, 16) for x in cols]
        out = oracle.philox4x32_10(v[0], v[1], v[2], v[3], v[4], v[5])
        assert [int(x) for x in out] == v[6:10]


def _kat_rows():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def test_gumbel_at_zero_temperature_is_deterministic_top_k():
    Vs = [16, 16]
    cat = host.draw_catalog(9, 120, Vs)
    trie = oracle.OracleTrie(cat, Vs)
    rng = np.random.default_rng(9)
    R, B_in, n = 2, 6, 10
    z = rng.normal(0, 2, size=(R * B_in, 16))
    ps = np.sort(rng.uniform(-5, -1, size=R * B_in))[::-1]
    pn = rng.integers(0, trie.n_nodes(1), size=R * B_in)
    g = oracle.beam_step_gumbel(trie, 1, z, ps, pn, R, B_in, n, 16, 0.0, 1234)
    d = oracle.beam_step(trie, 1, z, ps, pn, R, B_in, n, 16)
    for k in ("score", "parent", "code", "node"):
        assert np.array_equal(g[k], d[k])


def _draws(z, T, n, seeds):
    """Codes chosen, in rank order, from one root row with every code valid."""
    V = z.shape[0]
    out = []
    for seed in seeds:
        res = oracle.beam_step_gumbel(None, 0, z[None], [0.0], [0], 1, 1, n, V, T, seed)
        out.append(tuple(res["code"][0].tolist()))
    return out


def test_gumbel_top1_draws_follow_tempered_softmax():
    """The top key is a draw from softmax(log p / T): chi-square over 6,000 seeds
    (a sign or scale error in the Gumbel transform fails it)."""
    z = np.array([1.0, 0.2, -0.5, 0.0])
    for T in (1.0, 0.5):
        draws = _draws(z, T, 1, range(6000))
        lp = oracle.log_softmax_full(z)
        p = np.exp(lp / T)
        p /= p.sum()
        counts = np.bincount([d[0] for d in draws], minlength=4)
        exp = p * len(draws)
        chi2 = float(((counts - exp) ** 2 / exp).sum())
        assert chi2 < 20.0, (T, counts, exp)   # 3 dof; P(chi2 > 20) < 2e-4


def test_gumbel_top2_is_without_replacement():
    """The ordered pair (first, second) follows p_a * p_b / (1 - p_a): the second
    key continues the draw without the first."""
    z = np.array([0.8, 0.0, -0.6])
    draws = _draws(z, 1.0, 2, range(6000))
    p = np.exp(oracle.log_softmax_full(z))
    pairs = [(a, b) for a in range(3) for b in range(3) if a != b]
    counts = np.array([sum(1 for d in draws if d == pr) for pr in pairs], dtype=np.float64)
    exp = np.array([p[a] * p[b] / (1 - p[a]) for a, b in pairs]) * len(draws)
    assert all(d[0] != d[1] for d in draws)
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    assert chi2 < 25.0, (counts, exp)          # 5 dof; P(chi2 > 25) < 2e-4


# ------------------------------------------------------------------ lm_head
def test_lmhead_one_hot_picks_weight_column():
    d, V = 16, 10
    w = host.weight_matrix(3, V, d, 0.02)
    one = host.f32_to_bf16_bits(np.eye(d, dtype=np.float32))
    logits = oracle.lmhead_logits(one, w)
    assert np.array_equal(logits, host.bf16_bits_to_f32(w).astype(np.float64).T)
    # Linearity in the hidden state: h1 + h2 (both exact in bf16 and in the sum).
    h = host.f32_to_bf16_bits(np.array([[1.0] * d, [2.0] * d], dtype=np.float32))
    lg = oracle.lmhead_logits(h, w)
    np.testing.assert_allclose(lg[1], 2 * lg[0], rtol=0, atol=1e-15)
