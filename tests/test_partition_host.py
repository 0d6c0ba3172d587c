"""Host-side row partition over CTAs (the launch geometry every kernel uses),
checked on the CPU: every row goes to exactly one CTA, a CTA of a request
group holds only that request's rows, contiguous chunks stay contiguous, the
warps' shares are the CTA's entries w, w + W, ..., and the contributor counts
and first/last CTAs of each request agree with the rows and stay within maxG."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    cuda_inc = "/usr/local/cuda/include"
    if shutil.which("g++") is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime.h")):
        pytest.skip("needs g++ and the CUDA headers")
    out = tmp_path_factory.mktemp("probe") / "partition_probe.so"
    subprocess.run(["g++", "-std=c++17", "-O1", "-shared", "-fPIC", "-I", cuda_inc,
                    "-I", os.path.join(ROOT, "trie_constrained_beam_b200", "csrc"),
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "host", "partition_probe.cpp"), "-o", str(out)],
                   check=True)
    lib = ctypes.CDLL(str(out))
    P = ctypes.c_void_p
    lib.partition_probe.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, P, P, P, P, P, P]
    lib.partition_probe.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("R,B_in,ctas", [(16, 512, 148), (16, 1, 148), (64, 128, 148),
                                         (1, 2000, 148), (160, 40, 148), (1000, 3, 148),
                                         (3, 7, 148), (32, 32, 592), (7, 100000, 148)])
def test_partition_covers_every_row_once(probe, R, B_in, ctas):
    W = 12
    cap = max(1, -(-R * B_in // min(ctas, R * B_in))) + B_in + 1
    grid_max = ctas
    rows = np.full(grid_max * cap, -1, dtype=np.int64)
    counts = np.zeros(grid_max, dtype=np.int32)
    maxG = np.zeros(1, dtype=np.int32)
    first = np.zeros(R, dtype=np.int32)
    last = np.zeros(R, dtype=np.int32)
    contrib = np.zeros(R, dtype=np.int32)
    grid = probe.partition_probe(R, B_in, ctas, W, cap, rows.ctypes.data, counts.ctypes.data,
                                 maxG.ctypes.data, first.ctypes.data, last.ctypes.data,
                                 contrib.ctypes.data)
    assert 0 < grid <= ctas
    seen = np.zeros(R * B_in, dtype=np.int32)
    ctas_of = [set() for _ in range(R)]
    grouped = R <= ctas
    for c in range(grid):
        got = rows[c * cap:c * cap + counts[c]]
        assert np.all((got >= 0) & (got < R * B_in))
        np.add.at(seen, got, 1)
        reqs = set((got // B_in).tolist())
        for r in reqs:
            ctas_of[r].add(c)
        if grouped:
            assert len(reqs) <= 1                         # one request per CTA
        elif counts[c]:
            assert np.array_equal(got, np.arange(got[0], got[0] + counts[c]))  # contiguous
    assert np.all(seen == 1)                              # every row exactly once
    for r in range(R):
        # the CTAs holding rows of r are exactly first..last, at most maxG of them
        assert ctas_of[r] == set(range(first[r], last[r] + 1))
        assert contrib[r] == last[r] - first[r] + 1 <= maxG[0]


@pytest.mark.parametrize("R,maxG,n", [(16, 9, 512), (1, 148, 4096), (1000, 2, 3), (64, 2, 128)])
def test_workspace_layout_parts_fit(probe, R, maxG, n):
    """Every part starts 256-byte aligned, after the end of the one before, and
    the total covers the last: [status 4 B | tickets R x 4 | request bounds R x 8
    | histograms R x 1024 x 4 | part counts R x maxG x 4 | part keys R x maxG x 2n
    x 8 | part values R x maxG x 2n x 4]."""
    probe.workspace_probe.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    probe.workspace_probe.restype = None
    out = np.zeros(8, dtype=np.int64)
    probe.workspace_probe(R, maxG, n, out.ctypes.data)
    sizes = [4, R * 4, R * 8, R * 1024 * 4, R * maxG * 4, R * maxG * 2 * n * 8,
             R * maxG * 2 * n * 4]
    assert out[0] == 0
    for i in range(7):
        assert out[i] % 256 == 0
        end = out[i] + sizes[i]
        assert (out[i + 1] if i < 6 else out[7]) >= end


# (V, bytes per logit, trie bytes staged per row, mask words per warp, n): the
# step shapes of the five workloads, plus edge shapes.
_SHAPES = [(32, 4, 512, 4, 8), (32, 4, 512, 4, 2000), (256, 4, 32, 8, 32), (256, 4, 512, 8, 32),
           (8192, 2, 512, 256, 128), (4096, 2, 512, 128, 512), (4096, 2, 512, 128, 4096),
           (8192, 4, 512, 256, 64), (1, 4, 0, 0, 1), (16384, 4, 512, 512, 16)]


@pytest.mark.parametrize("shape", _SHAPES)
@pytest.mark.parametrize("ctl_bytes", [7424, 12288])
def test_step_plan_regions_aligned_and_disjoint(probe, shape, ctl_bytes):
    """Every region of the plan is aligned for how it is accessed (bulk-copy
    stages and their sizes on 128 bytes, the parent table and mask copies read
    as 16-byte vectors, 64-bit keys), the regions follow one another without
    overlap, and the whole plan fits the 227 KiB budget."""
    V, esize, extra, pw, n = shape
    probe.plan_probe.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p]
    probe.plan_probe.restype = ctypes.c_int
    for reg in ((0, 1) if V * esize <= 8192 else (0,)):
        out = np.zeros(17, dtype=np.int32)
        if not probe.plan_probe(V, esize, extra, pw, n, reg, ctl_bytes, out.ctypes.data):
            assert n > 2000 or reg  # only a huge n (or the register plan) may not fit
            continue
        W, S, Cw, sb, lcb, ctl, bars, meta, chist, whist, wpre, wmask, stage, wkeys, wvals, smem, rg = (
            int(x) for x in out)
        assert 1 <= W <= 12 and 1 <= S <= 8 and Cw >= n + 32 and rg == reg
        assert lcb >= V * esize and lcb % 16 == 0 and sb >= lcb + extra and sb % 128 == 0
        for off, a in ((ctl, 128), (bars, 128), (meta, 16), (chist, 16), (whist, 16),
                       (wpre, 16), (wmask, 16), (stage, 128), (wkeys, 128), (wvals, 16)):
            assert off % a == 0
        ends = [(ctl, ctl_bytes), (bars, W * 8 * 8), (meta, 256 * 16), (chist, 1024),
                (whist, max(W * 1024, 2 * 1024 * 4)), (wpre, W * pw * 4), (wmask, W * pw * 4),
                (stage, W * S * sb), (wkeys, W * Cw * 8), (wvals, W * Cw * 4)]
        for (o1, n1), (o2, _) in zip(ends, ends[1:]):
            assert o1 + n1 <= o2
        assert wvals + W * Cw * 4 <= smem <= 232448
