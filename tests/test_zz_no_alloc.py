"""beam_step_noalloc: the allocation-free variant of beam_step.

Some callers cannot allocate device memory when they run a step (a plugin whose
host owns every device allocation, a serving loop that plans all memory up
front). beam_step_noalloc serves them from a fixed scratch array built into the
library. These tests call it through the C ABI and check that it returns what
beam_step returns with a caller-allocated workspace, on two calls in a row.
This file is named to be collected last; it also passes when run on its own.
"""
import numpy as np
import pytest

from sidgen import host
from sidgen.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tcb():
    import trie_constrained_beam_b200 as m
    from sidgen import device
    from trie_constrained_beam_b200 import build
    build.build()
    device.build()
    return m


def _outs(R, n):
    import torch
    return [torch.empty(R * n, dtype=torch.float32, device="cuda")] + [
        torch.empty(R * n, dtype=torch.int32, device="cuda") for _ in range(3)]


def test_noalloc_matches_workspace_path_two_calls(tcb):
    import torch
    from sidgen import device as gdev
    w = WORKLOADS[2]
    R, n = 8, 32
    cat = w.catalog()
    trie = tcb.sid_trie_build(cat, w.codes_per_level, w.layouts)
    hashes = torch.from_numpy(host.request_roots(R).view(np.int64)).to("cuda")
    ps = torch.zeros(R, dtype=torch.float32, device="cuda")
    pn = torch.zeros(R, dtype=torch.int32, device="cuda")
    B_in = 1
    for step in range(2):                       # two calls in a row (step 0, then step 1)
        logits = torch.empty((R * B_in, w.V), dtype=torch.float32, device="cuda")
        gdev.row_logits(w.logits_seed, hashes, w.V, w.sigma, logits)
        ref = _outs(R, n)
        ws = torch.zeros(tcb.beam_step_workspace_size(R, B_in, n, w.V), dtype=torch.uint8,
                         device="cuda")
        tcb.beam_step(trie, step, logits, ps, pn, R, B_in, n, w.V, *ref, ws)
        got = _outs(R, n)
        tcb.beam_step_noalloc(trie, step, logits, ps, pn, R, B_in, n, w.V, *got)
        torch.cuda.synchronize()
        np.testing.assert_allclose(got[0].cpu().numpy(), ref[0].cpu().numpy(), atol=1e-5, rtol=0)
        for a, b in zip(got[1:], ref[1:]):
            assert torch.equal(a, b)
        assert int(torch.isfinite(got[0]).sum()) == R * n
        child = torch.empty((R * n,), dtype=torch.int64, device="cuda")
        gdev.child_hash(hashes, R, B_in, ref[1], ref[2], n, step + 1, child)
        hashes, ps, pn, B_in = child, ref[0], ref[3], n


def test_noalloc_rejects_shapes_beyond_its_scratch(tcb):
    import torch
    R, B_in, n, V = 64, 512, 4096, 1024
    assert tcb.beam_step_workspace_size(R, B_in, n, V) > tcb.native.NOALLOC_SCRATCH_BYTES
    z = torch.zeros((16, 1024), device="cuda")
    s = torch.zeros(16, device="cuda")
    with pytest.raises(tcb.SidbeamError) as e:
        tcb.beam_step_noalloc(None, 0, z, s, None, R, B_in, n, V, *_outs(1, 1))
    assert e.value.status == -4
