"""GPU parity of the tcgen05 SID-range lm_head (lmhead_logits) against the oracle.

The oracle multiplies the exactly widened bf16 operands in float64. The GPU
accumulates exact bf16 products in fp32 in an unspecified order, so each
logit may differ from the exact dot product by at most d * 2^-24 times the sum
of the products' magnitudes (the textbook bound for recursive summation);
the tests assert that bound, and that the typical error is far below it.
"""
import numpy as np
import pytest

import oracle
from sidgen import host
from sidgen.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tcb():
    import trie_constrained_beam_b200 as m
    from trie_constrained_beam_b200 import build
    build.build()
    return m


def _dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _run(tcb, hb, wb, ld_pad=0):
    import torch
    M, d = hb.shape
    V = wb.shape[0]
    ld = (V + ld_pad + 3) // 4 * 4
    out = torch.full((M, ld), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    tcb.lmhead_logits(_dev_bf16(hb), _dev_bf16(wb), out, ws)
    assert tcb.sidbeam_get_device_status(ws) == 0
    return out.cpu().numpy()


def _check(got, hb, wb, rows=None):
    h = (hb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    w = (wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if rows is not None:
        h = h[rows]
        got = got[rows]
        hb = hb[rows]
    ref = oracle.lmhead_logits(hb, wb)
    bound = (np.abs(h) @ np.abs(w).T) * h.shape[1] * 2.0 ** -24
    err = np.abs(got[:, :wb.shape[0]] - ref)
    assert np.all(err <= bound + 1e-30), float((err - bound).max())
    assert np.median(err / (bound + 1e-30)) < 0.05


@pytest.mark.parametrize("M,V,d", [(128, 256, 64), (130, 300, 72), (257, 512, 2048),
                                   (64, 8192, 128), (1, 8, 8)])
def test_lmhead_logits_shapes(tcb, M, V, d):
    """Whole tiles, ragged tiles on every side (M, V and the K tail)."""
    rng = np.random.default_rng(M * 7 + V + d)
    hb = host.f32_to_bf16_bits(rng.standard_normal((M, d)).astype(np.float32))
    wb = host.f32_to_bf16_bits((0.02 * rng.standard_normal((V, d))).astype(np.float32))
    got = _run(tcb, hb, wb, ld_pad=5)
    _check(got, hb, wb)
    if got.shape[1] > V:  # padding columns untouched
        assert np.isnan(got[:, V:]).all()


def test_lmhead_logits_fused_workload_shape(tcb):
    """4,096 rows x 8,192 codes x d = 2,048 from the seeded generators; sampled
    rows against the oracle (every tile of the grid is computed)."""
    w = WORKLOADS[5]
    hashes = host.prefix_hashes(np.random.default_rng(5).integers(0, 8192, size=(4096, 1)),
                                np.arange(4096) % w.R)
    hb = host.hidden_states(w.logits_seed, hashes, w.hidden_dim, w.hidden_sigma)
    wb = host.weight_matrix(w.weight_seed, w.V, w.hidden_dim, w.weight_sigma)
    got = _run(tcb, hb, wb)
    rows = np.r_[0:3, 127:130, 2047, 4093:4096]
    _check(got, hb, wb, rows=rows)


def test_lmhead_logits_argument_checks(tcb):
    import torch
    from trie_constrained_beam_b200 import native
    h = torch.zeros((4, 12), dtype=torch.bfloat16, device="cuda")   # d % 8 != 0
    wt = torch.zeros((8, 12), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((4, 8), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(native.SidbeamError) as e:
        tcb.lmhead_logits(h, wt, out, ws)
    assert e.value.status == native.SIDBEAM_ERR_ALIGNMENT


# ------------------------------------------------------------------ fused step
def _fused_case(tcb, trie_o, trie_g, step, R, B_in, n, V, d, seed, level_nodes, w_sigma=0.05):
    """One fused step on seeded inputs; parents are distinct level-`step` nodes
    with scores ranked best-first. Returns GPU outputs and the oracle inputs."""
    import torch
    from trie_constrained_beam_b200 import native
    rng = np.random.default_rng(seed)
    M = R * B_in
    if step == 0:
        pn = np.zeros(M, dtype=np.int32)
        ps = np.zeros(M, dtype=np.float32)
    else:
        pn = np.concatenate([rng.choice(level_nodes, size=B_in, replace=False)
                             for _ in range(R)]).astype(np.int32)
        ps = np.concatenate([np.sort(rng.uniform(-12, -2, size=B_in))[::-1]
                             for _ in range(R)]).astype(np.float32)
        ps[rng.random(M) < 0.05] = -np.inf          # a few dead rows
    hb = host.f32_to_bf16_bits(rng.standard_normal((M, d)).astype(np.float32))
    wb = host.f32_to_bf16_bits((w_sigma * rng.standard_normal((V, d))).astype(np.float32))
    dev = "cuda"
    out_s = torch.empty(R * n, dtype=torch.float32, device=dev)
    out_p, out_c, out_n = (torch.empty(R * n, dtype=torch.int32, device=dev) for _ in range(3))
    ws = torch.zeros(tcb.fused_lmhead_workspace_size(R, B_in, n, V), dtype=torch.uint8, device=dev)
    tcb.fused_lmhead_step(trie_g, step, _dev_bf16(hb), _dev_bf16(wb),
                          torch.from_numpy(ps).to(dev), torch.from_numpy(pn).to(dev),
                          R, B_in, n, out_s, out_p, out_c, out_n, ws)
    assert tcb.sidbeam_get_device_status(ws) == 0
    gpu = {"score": out_s.view(R, n).cpu().numpy(), "parent": out_p.view(R, n).cpu().numpy(),
           "code": out_c.view(R, n).cpu().numpy(), "node": out_n.view(R, n).cpu().numpy()}
    return gpu, hb, wb, ps, pn


def _fused_tol(hb, wb, exact=True):
    """Score tolerance of the fused step, from the inputs alone: the step's TOL
    plus twice the a-priori bound on a logit's error, d * 2^-24 * sum_k
    |h_k| |w_ck| (fp32 recursive summation of exact bf16 products), maximised
    over rows and codes. A score is s + z - lse and neither z nor lse moves by
    more than the largest logit error (log-sum-exp is 1-Lipschitz in the max
    norm). exact=False bounds sum_k |h_k| |w_ck| by ||h|| ||w_c|| (Cauchy-
    Schwarz) instead of forming every product sum."""
    from parity import TOL
    h = (hb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    w = (wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    d = h.shape[1]
    if exact:
        s = float((np.abs(h) @ np.abs(w).T).max())
    else:
        s = float(np.sqrt((h * h).sum(1)).max() * np.sqrt((w * w).sum(1)).max())
    return TOL + 2.0 * d * 2.0 ** -24 * s


@pytest.mark.parametrize("layouts", [[1, 1, 1], [2, 2, 2], [1, 2, 2], None])
def test_fused_step_small_matches_oracle(tcb, layouts):
    """Steps 0-2 of a 3-level, V=512 catalog, every layout and no trie, d = 136
    (a K tail); ranks compared with the tie-aware rule."""
    from parity import compare_step
    V, d, R, B_in, n = 512, 136, 3, 24, 16
    cat = host.draw_catalog(31, 3000, [V] * 3)
    to = oracle.OracleTrie(cat, [V] * 3)
    tg = tcb.sid_trie_build(cat, [V] * 3, layouts) if layouts is not None else None
    for step in range(3):
        Bi = 1 if step == 0 else B_in
        nodes = np.arange(to.n_nodes(step))
        if step > 0 and nodes.size < Bi:
            continue
        gpu, hb, wb, ps, pn = _fused_case(tcb, to, tg, step, R, Bi, n, V, d, 700 + step, nodes)
        z = oracle.lmhead_logits(hb, wb)
        compare_step(gpu, to if tg is not None else None, step, z, ps, pn, R, Bi, n, V,
                     tol=_fused_tol(hb, wb))


def test_fused_step_full_size_sampled_requests(tcb):
    """The fused-lm_head workload at full size (32 x 128 rows, V = 8192,
    d = 2048, W ~ N(0, 0.02), 1M-SID catalog): step 1 on the GPU for every
    request; two requests compared against the oracle."""
    from parity import compare_step
    w = WORKLOADS[5]
    cat = w.catalog()
    to = oracle.OracleTrie(cat, w.codes_per_level)
    tg = tcb.sid_trie_build(cat, w.codes_per_level, w.layouts)
    nodes = np.arange(to.n_nodes(1))
    gpu, hb, wb, ps, pn = _fused_case(tcb, to, tg, 1, w.R, w.n, w.n, w.V, w.hidden_dim, 55, nodes,
                                      w_sigma=w.weight_sigma)
    for r in (0, w.R - 1):
        rows = slice(r * w.n, (r + 1) * w.n)
        z = oracle.lmhead_logits(hb[rows], wb)
        sub = {k: v[r:r + 1] for k, v in gpu.items()}
        compare_step(sub, to, 1, z, ps[rows], pn[rows], 1, w.n, w.n, w.V,
                     tol=_fused_tol(hb[rows], wb))


def test_fused_search_all_requests(tcb):
    """The fused-lm_head workload as a whole search: 32 requests x beam 128,
    depth 3, V = 8192, d = 2048, 1M-SID catalog; the hidden state of every row
    is the seeded generator keyed on the row's prefix hash (as the logits of
    the other workloads are), so each step's rows follow from the previous
    step's beams. Every step is compared for every request with the oracle on
    the same inputs, at the a-priori tolerance of the tensor-core logits."""
    import torch
    from parity import compare_step
    from trie_constrained_beam_b200 import native
    w = WORKLOADS[5]
    cat = w.catalog()
    to = oracle.OracleTrie(cat, w.codes_per_level)
    tg = tcb.sid_trie_build(cat, w.codes_per_level, w.layouts)
    R, n, V, d = w.R, w.n, w.V, w.hidden_dim
    wb = host.weight_matrix(w.weight_seed, V, d, w.weight_sigma)
    w_dev = _dev_bf16(wb)
    hashes = host.request_roots(R)
    ps = np.zeros(R, dtype=np.float32)
    pn = np.zeros(R, dtype=np.int32)
    B_in = 1
    for step in range(w.depth):
        M = R * B_in
        live = np.isfinite(ps)
        hb = np.zeros((M, d), dtype=np.uint16)
        hb[live] = host.hidden_states(w.logits_seed, hashes[live], d, w.hidden_sigma)
        tol = _fused_tol(hb, wb, exact=False)
        out_s = torch.empty(R * n, dtype=torch.float32, device="cuda")
        out_p, out_c, out_n = (torch.empty(R * n, dtype=torch.int32, device="cuda")
                               for _ in range(3))
        ws = torch.zeros(tcb.fused_lmhead_workspace_size(R, B_in, n, V), dtype=torch.uint8,
                         device="cuda")
        tcb.fused_lmhead_step(tg, step, _dev_bf16(hb), w_dev, torch.from_numpy(ps).cuda(),
                              torch.from_numpy(pn).cuda(), R, B_in, n, out_s, out_p, out_c,
                              out_n, ws)
        assert tcb.sidbeam_get_device_status(ws) == 0
        gpu = {"score": out_s.view(R, n).cpu().numpy(), "parent": out_p.view(R, n).cpu().numpy(),
               "code": out_c.view(R, n).cpu().numpy(), "node": out_n.view(R, n).cpu().numpy()}
        z = oracle.lmhead_logits(hb, wb)
        compare_step(gpu, to, step, z, ps, pn, R, B_in, n, V, tol=tol)
        # The next step's rows: the beams just chosen (dead slots stay dead).
        nh = np.zeros(R * n, dtype=np.uint64)
        par, code = gpu["parent"].reshape(-1), gpu["code"].reshape(-1)
        ok = par >= 0
        src = (np.arange(R * n) // n) * B_in + np.where(ok, par, 0)
        nh[ok] = host.child_hash(hashes[src[ok]], step + 1, code[ok].astype(np.uint64))
        hashes, ps, pn, B_in = nh, gpu["score"].reshape(-1).astype(np.float32), \
            gpu["node"].reshape(-1).astype(np.int32), n
