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
