"""beam_step_noalloc: the allocation-free variant of beam_step.

Some callers cannot allocate device memory when they run a step (a plugin whose
host owns every device allocation, a serving loop that plans all memory up
front). beam_step_noalloc serves them from a fixed scratch array built into the
library. These tests call it through the C ABI and check that it returns what
beam_step returns with a caller-allocated workspace (bit for bit: the same
kernel over the same row partition), on two calls in a row and on a sequence
of calls of different shapes and dtypes sharing the one scratch array, and
that a call rejected by an argument check enqueues nothing on its stream.
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
        assert torch.equal(got[0].view(torch.int32), ref[0].view(torch.int32))
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


def test_noalloc_shape_sequence_matches_workspace_path(tcb):
    """Calls of different shapes in a row on the shared scratch: a large batch
    (many requests and rows: the most counters to clear), then a small one, then
    bf16 logits with a dense trie level; each against beam_step on a freshly
    zeroed workspace, bit for bit."""
    import torch
    rng = np.random.default_rng(77)
    V = 512
    cat = host.draw_catalog(78, 20_000, [V, V])
    trie_csr = tcb.sid_trie_build(cat, [V, V], [2, 2])
    trie_dense = tcb.sid_trie_build(cat, [V, V], [1, 1])
    n1 = int(tcb.sid_trie_info(trie_csr, 1)[0])
    cases = [(trie_csr, 200, 24, 16, torch.float32), (trie_csr, 3, 5, 7, torch.float32),
             (trie_dense, 40, 32, 32, torch.bfloat16), (None, 9, 11, 13, torch.bfloat16)]
    for trie, R, B_in, n, dt in cases:
        M = R * B_in
        assert tcb.beam_step_workspace_size(R, B_in, n, V) <= tcb.native.NOALLOC_SCRATCH_BYTES
        logits = torch.from_numpy(rng.normal(0, 2, size=(M, V)).astype(np.float32)).cuda().to(dt)
        ps = np.sort(rng.uniform(-8, -1, size=(R, B_in)), axis=1)[:, ::-1].reshape(-1)
        ps = torch.from_numpy(np.ascontiguousarray(ps, dtype=np.float32)).cuda()
        pn = torch.from_numpy(rng.integers(0, n1, size=M).astype(np.int32)).cuda()
        ref = _outs(R, n)
        ws = torch.zeros(tcb.beam_step_workspace_size(R, B_in, n, V), dtype=torch.uint8,
                         device="cuda")
        tcb.beam_step(trie, 1 if trie is not None else 0, logits, ps, pn, R, B_in, n, V, *ref, ws)
        got = _outs(R, n)
        tcb.beam_step_noalloc(trie, 1 if trie is not None else 0, logits, ps, pn, R, B_in, n, V,
                              *got)
        torch.cuda.synchronize()
        assert torch.equal(got[0].view(torch.int32), ref[0].view(torch.int32)), (R, B_in, n)
        for a, b in zip(got[1:], ref[1:]):
            assert torch.equal(a, b), (R, B_in, n)


def test_noalloc_rejected_call_enqueues_nothing(tcb):
    """An argument error is returned before anything reaches the stream: under
    stream capture a rejected call leaves the captured graph empty."""
    import torch
    from cuda.bindings import runtime as rt
    R, B_in, n, V = 2, 4, 8, 64
    z = torch.zeros((R * B_in, V), device="cuda")
    s = torch.zeros(R * B_in, device="cuda")
    outs = _outs(R, n)
    tcb.beam_step_noalloc(None, 0, z, s, None, R, B_in, n, V, *outs)   # first call: set-up
    torch.cuda.synchronize()
    err, stream = rt.cudaStreamCreate()
    assert err == rt.cudaError_t.cudaSuccess
    try:
        for bad in ({"n": 0}, {"logits": z[:, 1:]}, {"V": 65}):
            err, = rt.cudaStreamBeginCapture(stream,
                                             rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
            assert err == rt.cudaError_t.cudaSuccess
            rc = tcb.native.load().beam_step_noalloc(
                None, 0, bad.get("logits", z).data_ptr(), 0, V, s.data_ptr(), None, R, B_in,
                bad.get("n", n), bad.get("V", V), *[o.data_ptr() for o in outs], int(stream))
            assert rc < 0, bad
            err, graph = rt.cudaStreamEndCapture(stream)
            assert err == rt.cudaError_t.cudaSuccess
            err, _, count = rt.cudaGraphGetNodes(graph)
            assert err == rt.cudaError_t.cudaSuccess
            assert count == 0, bad
            rt.cudaGraphDestroy(graph)
    finally:
        rt.cudaStreamDestroy(stream)
