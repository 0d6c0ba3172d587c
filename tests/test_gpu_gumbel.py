"""GPU parity of the Gumbel top-k step (beam_step_gumbel) against the oracle.

The oracle draws its Gumbel variates from its own Philox4x32-10 in float64;
the device draws the same U (exact in fp32) and forms G and the key in fp32.
Ranks are compared under the rule of the deterministic step applied to the
keys: where the oracle's neighbouring keys are further apart than the key
tolerance, (parent, code, node) must match; inside near-ties the device's pick
must be a valid candidate whose oracle key is within that tolerance. The
written score is the unperturbed one and must match within TOL. Key
tolerance: TOL plus T * 2e-5 (G in fp32: two single-precision logarithms of
magnitude below 17, a few ulps each, and one more rounding of z + T*G).
"""
import numpy as np
import pytest

import oracle
from sidgen import host

from parity import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tcb():
    import trie_constrained_beam_b200 as m
    from trie_constrained_beam_b200 import build
    build.build()
    return m


def _run(tcb, trie, step, z, ps, pn, R, B_in, n, V, T, seed, dtype="f32", gumbel=True):
    import torch
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    zt = torch.from_numpy(np.ascontiguousarray(z, dtype=np.float32)).cuda().to(tdt)
    out = dict(score=torch.empty(R * n, device="cuda"),
               parent=torch.empty(R * n, dtype=torch.int32, device="cuda"),
               code=torch.empty(R * n, dtype=torch.int32, device="cuda"),
               node=torch.empty(R * n, dtype=torch.int32, device="cuda"))
    ps_t = torch.from_numpy(np.asarray(ps, np.float32)).cuda()
    pn_t = torch.from_numpy(np.asarray(pn, np.int32)).cuda()
    if gumbel:
        ws = torch.zeros(tcb.beam_step_gumbel_workspace_size(R, B_in, n, V), dtype=torch.uint8,
                         device="cuda")
        tcb.beam_step_gumbel(trie, step, zt, ps_t, pn_t, R, B_in, n, V, T, seed, out["score"],
                             out["parent"], out["code"], out["node"], ws)
    else:
        ws = torch.zeros(tcb.beam_step_workspace_size(R, B_in, n, V), dtype=torch.uint8,
                         device="cuda")
        tcb.beam_step(trie, step, zt, ps_t, pn_t, R, B_in, n, V, out["score"], out["parent"],
                      out["code"], out["node"], ws)
    assert tcb.sidbeam_get_device_status(ws) == 0
    return {k: v.cpu().numpy().reshape(R, n) for k, v in out.items()}


def _compare(g, ref, R, n, T, trie, step, z, ps, pn, B_in, V, seed):
    ktol = TOL + T * 2e-5
    for r in range(R):
        ok = ref["key"][r]
        v = int(np.isfinite(ok).sum())
        assert int(np.isfinite(g["score"][r]).sum()) == v
        assert np.all(g["parent"][r, v:] == -1)
        seen = set()
        for k in range(v):
            gp, gc = int(g["parent"][r, k]), int(g["code"][r, k])
            assert (gp, gc) not in seen
            seen.add((gp, gc))
            lo = k == 0 or ok[k - 1] - ok[k] > ktol
            hi = k + 1 >= v or ok[k] - ok[k + 1] > ktol
            if lo and hi:
                assert (gp, gc, int(g["node"][r, k])) == (
                    int(ref["parent"][r, k]), int(ref["code"][r, k]), int(ref["node"][r, k])), (r, k)
                assert abs(float(g["score"][r, k]) - ref["score"][r, k]) <= TOL
            else:  # near-tie: a valid candidate with that key
                row = r * B_in + gp
                lp = oracle.log_softmax_full(z[row, :V].astype(np.float64))
                x = float(ps[row]) + lp[gc]
                gk = x + T * float(oracle.gumbel(seed, r, gp, np.array([gc]), step)[0])
                assert abs(gk - ok[k]) <= ktol
                assert abs(float(g["score"][r, k]) - x) <= TOL
                if trie is not None:
                    codes, ids = trie.children(step, int(pn[row]))
                    assert gc in set(codes.tolist())


def _case(seed, V, layout, n_cat, R, B_in):
    rng = np.random.default_rng(seed)
    Vs = [V, V]
    cat = host.draw_catalog(seed, n_cat, Vs)
    otrie = oracle.OracleTrie(cat, Vs)
    M = R * B_in
    z = (2.0 * rng.standard_normal((M, V))).astype(np.float32)
    ps = np.concatenate([np.sort(rng.uniform(-6, -1, size=B_in))[::-1] for _ in range(R)])
    ps = ps.astype(np.float32)
    ps[rng.random(M) < 0.05] = -np.inf
    pn = rng.integers(0, otrie.n_nodes(1), size=M).astype(np.int32)
    return cat, otrie, z, ps, pn


@pytest.mark.parametrize("layout,T,dtype", [(2, 1.0, "f32"), (1, 0.5, "f32"), (2, 3.0, "bf16"),
                                            (1, 1.0, "bf16"), (0, 1.0, "f32")])
def test_gumbel_step_matches_oracle(tcb, layout, T, dtype):
    V, R, B_in, n = 256, 3, 40, 32
    cat, otrie, z, ps, pn = _case(11 + layout, V, layout, 4000, R, B_in)
    if dtype == "bf16":
        z = host.bf16_bits_to_f32(host.f32_to_bf16_bits(z))
    gtrie = tcb.sid_trie_build(cat, [V, V], [layout, layout]) if layout else None
    seed = 0x1234_5678_9ABC_DEF0 + layout
    g = _run(tcb, gtrie, 1, z, ps, pn, R, B_in, n, V, T, seed, dtype)
    ref = oracle.beam_step_gumbel(otrie if layout else None, 1, z, ps, pn, R, B_in, n, V, T, seed)
    _compare(g, ref, R, n, T, otrie if layout else None, 1, z, ps, pn, B_in, V, seed)


def test_gumbel_many_children_and_seeds(tcb):
    """Parents with up to ~4,000 children (two-pass walks), V = 4,096 bf16,
    grouped over many CTAs; two seeds give different draws."""
    V, R, B_in, n = 4096, 2, 600, 128
    rng = np.random.default_rng(4)
    cat = np.array([(a, c) for a in range(40)
                    for c in rng.choice(V, size=int(rng.integers(50, 4000)), replace=False)])
    otrie = oracle.OracleTrie(cat, [V, V])
    gtrie = tcb.sid_trie_build(cat, [V, V], [2, 2])
    M = R * B_in
    z = host.bf16_bits_to_f32(host.f32_to_bf16_bits(
        (3.0 * rng.standard_normal((M, V))).astype(np.float32)))
    ps = np.concatenate([np.sort(rng.uniform(-8, -1, size=B_in))[::-1] for _ in range(R)])
    ps = ps.astype(np.float32)
    pn = rng.integers(0, otrie.n_nodes(1), size=M).astype(np.int32)
    outs = []
    for seed in (7, 8):
        g = _run(tcb, gtrie, 1, z, ps, pn, R, B_in, n, V, 1.0, seed, "bf16")
        ref = oracle.beam_step_gumbel(otrie, 1, z, ps, pn, R, B_in, n, V, 1.0, seed)
        _compare(g, ref, R, n, 1.0, otrie, 1, z, ps, pn, B_in, V, seed)
        outs.append(g)
    assert not np.array_equal(outs[0]["code"], outs[1]["code"])


def test_gumbel_zero_temperature_is_beam_step(tcb):
    V, R, B_in, n = 256, 2, 30, 16
    cat, otrie, z, ps, pn = _case(21, V, 2, 3000, R, B_in)
    gtrie = tcb.sid_trie_build(cat, [V, V], [2, 2])
    a = _run(tcb, gtrie, 1, z, ps, pn, R, B_in, n, V, 0.0, 99)
    b = _run(tcb, gtrie, 1, z, ps, pn, R, B_in, n, V, 0.0, 99, gumbel=False)
    for k in a:
        assert np.array_equal(a[k].view(np.uint32), b[k].view(np.uint32))


def test_gumbel_argument_checks(tcb):
    import torch
    from trie_constrained_beam_b200 import native
    z = torch.zeros((4, 8), device="cuda")
    ps = torch.zeros(4, device="cuda")
    pn = torch.zeros(4, dtype=torch.int32, device="cuda")
    o = [torch.empty(4, device="cuda")] + [torch.empty(4, dtype=torch.int32, device="cuda")] * 3
    ws = torch.zeros(tcb.beam_step_gumbel_workspace_size(1, 4, 4, 8), dtype=torch.uint8,
                     device="cuda")
    for T in (-1.0, float("nan"), float("inf")):
        with pytest.raises(native.SidbeamError) as e:
            tcb.beam_step_gumbel(None, 0, z, ps, pn, 1, 4, 4, 8, T, 1, o[0], o[1], o[2], o[3], ws)
        assert e.value.status == native.SIDBEAM_ERR_INVALID_ARG
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(native.SidbeamError) as e:
        tcb.beam_step_gumbel(None, 0, z, ps, pn, 1, 4, 4, 8, 1.0, 1, o[0], o[1], o[2], o[3], small)
    assert e.value.status == native.SIDBEAM_ERR_WORKSPACE


def test_gumbel_wide_beam_step1_shape(tcb):
    """The wide-beam step-1 shape: 16 requests x 512 parent rows (8,192 rows),
    V = 4,096 bf16 logits (sigma 3), a dense child bitmask over a catalog whose
    two levels are Zipf(1.2) (so parents have from a few to thousands of
    children), n = 512, T = 1: every request against the oracle."""
    V, R, B_in, n, T = 4096, 16, 512, 512, 1.0
    rng = np.random.default_rng(41)
    cat = host.draw_catalog(4101, 300_000, [V, V], [("zipf", 1.2), ("zipf", 1.2)])
    otrie = oracle.OracleTrie(cat, [V, V])
    gtrie = tcb.sid_trie_build(cat, [V, V], [1, 1])
    nodes = np.arange(otrie.n_nodes(1))
    pn = np.concatenate([rng.choice(nodes, size=B_in, replace=False) for _ in range(R)])
    pn = pn.astype(np.int32)
    ps = np.concatenate([np.sort(rng.uniform(-9, -2, size=B_in))[::-1] for _ in range(R)])
    ps = ps.astype(np.float32)
    z = host.bf16_bits_to_f32(host.f32_to_bf16_bits(
        (3.0 * rng.standard_normal((R * B_in, V))).astype(np.float32)))
    seed = 0x5EED_0F_6B3E1
    g = _run(tcb, gtrie, 1, z, ps, pn, R, B_in, n, V, T, seed, "bf16")
    ref = oracle.beam_step_gumbel(otrie, 1, z, ps, pn, R, B_in, n, V, T, seed)
    _compare(g, ref, R, n, T, otrie, 1, z, ps, pn, B_in, V, seed)


@pytest.mark.parametrize("layout", [1, 2])
def test_gumbel_rows_over_8kb_shared_memory_path(tcb, layout):
    """fp32 rows of V = 4,096 (16 KB: walked in shared memory, not held in
    registers), parents with up to ~3,000 children and more rows per CTA than
    warps, so the perturbed-score seeding of the first rows runs; both trie
    layouts."""
    V, R, B_in, n = 4096, 2, 300, 64
    rng = np.random.default_rng(40 + layout)
    cat = np.array([(a, c) for a in range(24)
                    for c in rng.choice(V, size=int(rng.integers(200, 3000)), replace=False)])
    otrie = oracle.OracleTrie(cat, [V, V])
    gtrie = tcb.sid_trie_build(cat, [V, V], [layout, layout])
    M = R * B_in
    z = (3.0 * rng.standard_normal((M, V))).astype(np.float32)
    ps = np.concatenate([np.sort(rng.uniform(-8, -1, size=B_in))[::-1] for _ in range(R)])
    ps = ps.astype(np.float32)
    pn = rng.integers(0, otrie.n_nodes(1), size=M).astype(np.int32)
    seed = 0xC0FFEE + layout
    g = _run(tcb, gtrie, 1, z, ps, pn, R, B_in, n, V, 1.0, seed, "f32")
    ref = oracle.beam_step_gumbel(otrie, 1, z, ps, pn, R, B_in, n, V, 1.0, seed)
    _compare(g, ref, R, n, 1.0, otrie, 1, z, ps, pn, B_in, V, seed)
