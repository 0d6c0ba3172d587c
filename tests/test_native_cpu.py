"""CPU checks of the native boundary: the library builds, loads, exports every
symbol include/sidbeam.h declares, and rejects bad arguments on the host before
any launch. No kernel runs here."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from trie_constrained_beam_b200 import build, native
    build.build()
    return native.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "sidbeam.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)
    keywords = {"if", "sizeof", "defined"}
    return sorted({n for n in names if n not in keywords})


def test_header_symbols_exported(lib):
    from trie_constrained_beam_b200 import native
    declared = _declared()
    assert set(declared) == set(native.EXPORTED), declared
    for name in declared:
        assert hasattr(lib, name), name


def test_version_and_error_string(lib):
    from trie_constrained_beam_b200 import native
    assert native.sidbeam_version() == "0.1.0"
    assert isinstance(native.sidbeam_last_error(), str)


def _bad_step(lib, **kw):
    args = dict(trie=None, step=0, logits=0x1000, dtype=0, ld=64, ps=0x2000, pn=0x3000, R=1,
                B_in=1, n=4, V=64, o1=0x4000, o2=0x5000, o3=0x6000, o4=0x7000, ws=0x8000,
                wsb=1 << 20)
    args.update(kw)
    P = ctypes.c_void_p
    return lib.beam_step(args["trie"], args["step"], P(args["logits"]), args["dtype"], args["ld"],
                         P(args["ps"]), P(args["pn"]), args["R"], args["B_in"], args["n"],
                         args["V"], P(args["o1"]), P(args["o2"]), P(args["o3"]), P(args["o4"]),
                         P(args["ws"]), args["wsb"], None)


def test_host_argument_checks(lib):
    assert _bad_step(lib, n=0) == -1
    assert _bad_step(lib, n=5000) == -1
    assert _bad_step(lib, V=0) == -1
    assert _bad_step(lib, V=40000) == -1
    assert _bad_step(lib, dtype=7) == -1
    assert _bad_step(lib, B_in=70000, V=70000) == -1
    assert _bad_step(lib, ld=10) == -1                 # ld < V
    assert _bad_step(lib, logits=0x1008) == -3         # not 16-byte aligned
    assert _bad_step(lib, ld=65) == -3                 # row stride not a multiple of 16 B
    assert _bad_step(lib, ws=0x8010) == -4             # workspace not 256-byte aligned
    assert _bad_step(lib, logits=0) == -1


def test_trie_build_checks_before_device_work(lib):
    from trie_constrained_beam_b200 import native
    with pytest.raises(native.SidbeamError) as e:
        native.sid_trie_build(np.array([[0, 9]]), [4, 4])
    assert e.value.status == -2
    with pytest.raises(native.SidbeamError) as e:
        native.sid_trie_build(np.zeros((2, 17), dtype=np.int32), [4] * 17)
    assert e.value.status == -1


def test_no_cpu_fallback_without_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    from trie_constrained_beam_b200 import native
    # With no usable device every call that needs CUDA fails loudly.
    with pytest.raises(native.SidbeamError) as e:
        native.sid_trie_build(np.array([[0, 1]]), [4, 4])
    assert e.value.status == -6


def test_workspace_size_shapes(lib):
    from trie_constrained_beam_b200 import native
    assert native.beam_step_workspace_size(0, 1, 1, 1) == 0
    assert native.beam_step_workspace_size(1, 1, 5000, 4) == 0
    a = native.beam_step_workspace_size(16, 512, 512, 4096)
    b = native.beam_step_workspace_size(16, 512, 256, 4096)
    assert a > b > 0 and a % 256 == 0


def test_step_options_argument_checks(lib):
    """beam_step_ex, beam_step_gumbel and catalog_score_topk_sim reject bad
    arguments on the host (no device call is made on these paths)."""
    P = ctypes.c_void_p
    base = (None, 0, P(0x1000), 0, 64, P(0x2000), P(0x3000), 1, 1, 4, 64, P(0x4000), P(0x5000),
            P(0x6000), P(0x7000), P(0x8000), 1 << 20, None)
    assert lib.beam_step_ex(*base, 0x4, None) == -1          # unknown flag bit
    assert lib.beam_step_ex(*base[:9], 0, *base[10:], 0, None) == -1   # n_out = 0
    g = (None, 0, P(0x1000), 0, 64, P(0x2000), P(0x3000), 1, 1, 4, 64)
    outs = (P(0x4000), P(0x5000), P(0x6000), P(0x7000), P(0x8000), 1 << 20, None)
    for T in (-1.0, float("nan"), float("inf")):
        assert lib.beam_step_gumbel(*g, ctypes.c_float(T), ctypes.c_uint64(1), *outs) == -1
    assert lib.beam_step_gumbel(*g, ctypes.c_float(1.0), ctypes.c_uint64(1),
                                *outs[:5], 16, None) == -4            # workspace too small
    assert lib.catalog_score_topk_sim(None, P(0x1000), P(0x2000), P(0x3000), 8, 1, 1,
                                      P(0x4000), P(0x5000), P(0x6000), 1 << 20, None) == -1


def test_finalize_argument_checks(lib):
    """beam_finalize rejects bad shapes and NULL pointers on the host, before any
    device call: depth outside 1..SIDBEAM_MAX_DEPTH, R < 1, n outside
    1..SIDBEAM_MAX_BEAM (the kernel keeps parent slots in 16 bits)."""
    P = ctypes.c_void_p
    ptrs = [P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000)]

    def fin(depth, R, n, p=ptrs):
        return lib.beam_finalize(depth, R, n, *p, None)
    assert fin(0, 1, 4) == -1
    assert fin(17, 1, 4) == -1
    assert fin(3, 0, 4) == -1
    assert fin(3, 1, 0) == -1
    assert fin(3, 1, 4097) == -1
    for k in range(5):
        assert fin(3, 1, 4, ptrs[:k] + [None] + ptrs[k + 1:]) == -1
    from trie_constrained_beam_b200 import native
    assert "beam_finalize" in native.sidbeam_last_error()


def test_header_is_plain_c(tmp_path):
    """include/sidbeam.h compiles on its own as C99 (pedantic): no C++ or CUDA
    types leak into the boundary."""
    import shutil
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "sidbeam.h"\n'
                   "int main(void) { sidbeam_trie* t = 0; (void)t;\n"
                   "  return (int)beam_step_workspace_size(1, 1, 1, 1) * 0; }\n")
    import subprocess
    out = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                          "-I", os.path.join(ROOT, "include"), "-c", str(src), "-o",
                          str(tmp_path / "use_header.o")], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
