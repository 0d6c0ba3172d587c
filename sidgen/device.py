"""CUDA twin of the generators (``libsidgen.so``), called with torch tensors.

Build with :func:`build`; the shared object is written next to this file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

from . import host

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsidgen.so")
_SRC = os.path.join(_HERE, "csrc", "sidgen.cu")
_lib = None


def build(force: bool = False) -> str:
    """Compile libsidgen.so for sm_100a (nvcc cross-compiles without a GPU)."""
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(_SRC)):
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = ["nvcc", "-O3", "-shared", "-Xcompiler", "-fPIC", "-lineinfo",
           "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, _SRC]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run sidgen.device.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, U64, F32 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                 ctypes.c_uint64, ctypes.c_float)
        L.sidgen_philox.argtypes = [U64, P, P, I64, P]
        L.sidgen_row_logits.argtypes = [U64, P, I64, I32, I64, F32, I32, I32, P, P]
        L.sidgen_child_hash.argtypes = [P, I32, I32, P, P, I32, I32, P, P]
        L.sidgen_table.argtypes = [U64, I32, I32, I32, F32, P, P]
        L.sidgen_weight.argtypes = [U64, I32, I32, F32, P, P]
        L.sidgen_hidden.argtypes = [U64, P, I64, I32, F32, P, P]
        for f in (L.sidgen_philox, L.sidgen_row_logits, L.sidgen_child_hash, L.sidgen_table,
                  L.sidgen_weight, L.sidgen_hidden):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


def philox(seed: int, ctr, out, stream=None):
    """ctr, out: uint32-bit tensors [n, 4] on the device (int32 dtype is fine)."""
    _check(lib().sidgen_philox(seed & (2**64 - 1), ctr.data_ptr(), out.data_ptr(),
                               ctr.shape[0], _stream(stream)), "sidgen_philox")


def row_logits(seed: int, hashes, V: int, sigma: float, out, stream=None,
               stream_id: int = host.STREAM_BEAM_LOGITS):
    """Fill out[:rows, :V] (fp32 or bf16 tensor [rows, ld]) from int64 hashes [rows]."""
    import torch
    bf16 = 1 if out.dtype == torch.bfloat16 else 0
    _check(lib().sidgen_row_logits(seed & (2**64 - 1), hashes.data_ptr(), hashes.shape[0], V,
                                   out.stride(0), float(host.k_sigma(sigma)), bf16, stream_id,
                                   out.data_ptr(), _stream(stream)), "sidgen_row_logits")


def child_hash(parent_hash, R, B_in, out_parent, out_code, n, level, child, stream=None):
    _check(lib().sidgen_child_hash(parent_hash.data_ptr(), R, B_in, out_parent.data_ptr(),
                                   out_code.data_ptr(), n, level, child.data_ptr(),
                                   _stream(stream)), "sidgen_child_hash")


def table(seed: int, R: int, L: int, V: int, sigma: float, out, stream=None):
    _check(lib().sidgen_table(seed & (2**64 - 1), R, L, V, float(host.k_sigma(sigma)),
                              out.data_ptr(), _stream(stream)), "sidgen_table")


def weight(seed: int, V: int, d: int, sigma: float, out, stream=None):
    _check(lib().sidgen_weight(seed & (2**64 - 1), V, d, float(host.k_sigma(sigma)),
                               out.data_ptr(), _stream(stream)), "sidgen_weight")


def hidden(seed: int, hashes, d: int, sigma: float, out, stream=None):
    _check(lib().sidgen_hidden(seed & (2**64 - 1), hashes.data_ptr(), hashes.shape[0], d,
                               float(host.k_sigma(sigma)), out.data_ptr(), _stream(stream)),
           "sidgen_hidden")
