"""ctypes binding of libsidbeam.so: the C ABI of include/sidbeam.h, same names.

Argument marshalling only: device buffers are torch CUDA tensors (their
data_ptr() is passed), streams are torch.cuda.Stream objects (default: the
current stream). Every computation runs in the library's kernels; there is no
CPU fallback, and loading fails loudly when the shared object is missing.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsidbeam.so")

SIDBEAM_OK = 0
SIDBEAM_ERR_INVALID_ARG = -1
SIDBEAM_ERR_BAD_CATALOG = -2
SIDBEAM_ERR_ALIGNMENT = -3
SIDBEAM_ERR_WORKSPACE = -4
SIDBEAM_ERR_OOM = -5
SIDBEAM_ERR_CUDA = -6
SIDBEAM_ERR_DEVICE_CHECK = -7
SIDBEAM_ERR_TIMEOUT = -8

SIDBEAM_F32 = 0
SIDBEAM_BF16 = 1

LAYOUT_AUTO = 0
LAYOUT_DENSE = 1
LAYOUT_CSR = 2

MAX_DEPTH = 16
MAX_V = 32768
MAX_BEAM = 4096

# Every symbol include/sidbeam.h declares.
EXPORTED = (
    "sid_trie_build", "sid_trie_info", "sid_trie_leaf_rows", "sid_trie_leaf_codes",
    "sid_trie_free", "beam_step_workspace_size", "beam_step", "beam_finalize",
    "catalog_score_workspace_size", "catalog_score_topk", "sidbeam_get_device_status",
    "sidbeam_last_error", "sidbeam_version", "beam_step_noalloc", "lmhead_logits",
    "fused_lmhead_workspace_size", "sidbeam_fused_lmhead_step", "beam_step_ex",
    "beam_step_skipped_rows", "catalog_score_topk_sim", "beam_step_gumbel",
    "beam_step_gumbel_workspace_size",
)

STEP_SKIP_ROWS = 1  # SIDBEAM_STEP_SKIP_ROWS

NOALLOC_SCRATCH_BYTES = 4 << 20


class SidbeamError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"sidbeam status {status}: {message}")
        self.status = status


_lib = None


def load():
    """Load libsidbeam.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing; build it with `python -m trie_constrained_beam_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.sid_trie_build.argtypes = [P, I64, I32, P, P, P, ctypes.POINTER(P)]
    L.sid_trie_info.argtypes = [P, I32, ctypes.POINTER(I64), ctypes.POINTER(I32), ctypes.POINTER(SZ)]
    L.sid_trie_leaf_rows.argtypes = [P, P, P]
    L.sid_trie_leaf_codes.argtypes = [P, P, P]
    L.sid_trie_free.argtypes = [P]
    L.sid_trie_free.restype = None
    L.beam_step_workspace_size.argtypes = [I32, I32, I32, I32]
    L.beam_step_workspace_size.restype = SZ
    L.beam_step.argtypes = [P, I32, P, I32, I64, P, P, I32, I32, I32, I32, P, P, P, P, P, SZ, P]
    L.beam_step_noalloc.argtypes = [P, I32, P, I32, I64, P, P, I32, I32, I32, I32, P, P, P, P, P]
    L.beam_step_ex.argtypes = [P, I32, P, I32, I64, P, P, I32, I32, I32, I32, P, P, P, P, P, SZ, P,
                               ctypes.c_uint, P]
    L.beam_step_skipped_rows.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), P]
    L.beam_step_gumbel_workspace_size.argtypes = [I32, I32, I32, I32]
    L.beam_step_gumbel_workspace_size.restype = SZ
    L.beam_step_gumbel.argtypes = [P, I32, P, I32, I64, P, P, I32, I32, I32, I32, ctypes.c_float,
                                   ctypes.c_uint64, P, P, P, P, P, SZ, P]
    L.beam_finalize.argtypes = [I32, I32, I32, P, P, P, P, P, P]
    L.catalog_score_workspace_size.argtypes = [P, I32, I32]
    L.catalog_score_workspace_size.restype = SZ
    L.catalog_score_topk.argtypes = [P, P, I32, I32, P, P, P, SZ, P]
    L.catalog_score_topk_sim.argtypes = [P, P, P, P, I32, I32, I32, P, P, P, SZ, P]
    L.sidbeam_get_device_status.argtypes = [P, P]
    L.lmhead_logits.argtypes = [P, P, I32, I32, I32, P, I64, P, SZ, P]
    L.fused_lmhead_workspace_size.argtypes = [I32, I32, I32, I32]
    L.fused_lmhead_workspace_size.restype = SZ
    L.sidbeam_fused_lmhead_step.argtypes = [P, I32, P, P, I32, P, P, I32, I32, I32, I32, P, P, P,
                                            P, P, SZ, P]
    L.sidbeam_last_error.argtypes = []
    L.sidbeam_last_error.restype = ctypes.c_char_p
    L.sidbeam_version.argtypes = []
    L.sidbeam_version.restype = ctypes.c_char_p
    for name in ("sid_trie_build", "sid_trie_info", "sid_trie_leaf_rows", "sid_trie_leaf_codes",
                 "beam_step", "beam_step_noalloc", "beam_finalize", "catalog_score_topk",
                 "sidbeam_get_device_status", "lmhead_logits", "sidbeam_fused_lmhead_step",
                 "beam_step_ex", "beam_step_skipped_rows", "catalog_score_topk_sim",
                 "beam_step_gumbel"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(rc: int):
    if rc != SIDBEAM_OK:
        raise SidbeamError(rc, sidbeam_last_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    """cudaStream_t of a torch stream; None means torch's current stream
    (or the legacy default stream when torch sees no device)."""
    if stream is None:
        import torch
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return SIDBEAM_F32
    if t.dtype == torch.bfloat16:
        return SIDBEAM_BF16
    raise TypeError(f"logits dtype {t.dtype} is not float32 or bfloat16")


def sidbeam_last_error() -> str:
    return load().sidbeam_last_error().decode()


def sidbeam_version() -> str:
    return load().sidbeam_version().decode()


class Trie:
    """Owner of a sidbeam_trie handle (freed with sid_trie_free)."""

    def __init__(self, handle, depth, codes_per_level):
        self.handle = handle
        self.depth = depth
        self.codes_per_level = list(codes_per_level)

    @property
    def _as_parameter_(self):
        return self.handle

    def close(self):
        if self.handle:
            load().sid_trie_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def sid_trie_build(sids, codes_per_level, layout_per_level=None, stream=None) -> Trie:
    """sids: host int array [n_sids, depth]."""
    L = load()
    sids = np.ascontiguousarray(sids, dtype=np.int32)
    n, depth = sids.shape
    cpl = np.ascontiguousarray(codes_per_level, dtype=np.int32)
    lay = None if layout_per_level is None else np.ascontiguousarray(layout_per_level, dtype=np.int32)
    out = ctypes.c_void_p()
    rc = L.sid_trie_build(sids.ctypes.data, n, depth, cpl.ctypes.data,
                          None if lay is None else lay.ctypes.data, _stream(stream),
                          ctypes.byref(out))
    _check(rc)
    return Trie(out, depth, cpl.tolist())


def sid_trie_info(trie: Trie, level: int):
    n = ctypes.c_int64()
    lay = ctypes.c_int()
    nb = ctypes.c_size_t()
    _check(load().sid_trie_info(trie.handle, level, ctypes.byref(n), ctypes.byref(lay),
                                ctypes.byref(nb)))
    return n.value, lay.value, nb.value


def sid_trie_leaf_rows(trie: Trie, out, stream=None):
    _check(load().sid_trie_leaf_rows(trie.handle, _ptr(out), _stream(stream)))


def sid_trie_leaf_codes(trie: Trie, out, stream=None):
    _check(load().sid_trie_leaf_codes(trie.handle, _ptr(out), _stream(stream)))


def beam_step_workspace_size(R: int, B_in: int, n_out: int, V: int) -> int:
    return int(load().beam_step_workspace_size(R, B_in, n_out, V))


def beam_step(trie, step, logits, parent_scores, parent_nodes, R, B_in, n_out, V,
              out_scores, out_parent, out_code, out_node, workspace, stream=None, ld=None,
              skip_rows=False, out_width=None):
    """logits: torch [R*B_in, ld] float32/bfloat16 on the device (row stride = ld).
    skip_rows: do not read rows that cannot contribute (beam_step_ex with
    SIDBEAM_STEP_SKIP_ROWS); the results are the same. out_width: optional
    device int32 [R], beams kept per request (the rest of n_out is padding)."""
    if ld is None:
        ld = logits.stride(0)
    args = (None if trie is None else trie.handle, step, _ptr(logits), _dtype_code(logits), ld,
            _ptr(parent_scores), _ptr(parent_nodes), R, B_in, n_out, V, _ptr(out_scores),
            _ptr(out_parent), _ptr(out_code), _ptr(out_node), _ptr(workspace),
            0 if workspace is None else workspace.numel() * workspace.element_size(),
            _stream(stream))
    if skip_rows or out_width is not None:
        rc = load().beam_step_ex(*args, STEP_SKIP_ROWS if skip_rows else 0,
                                 None if out_width is None else _ptr(out_width))
    else:
        rc = load().beam_step(*args)
    _check(rc)


def beam_step_gumbel_workspace_size(R: int, B_in: int, n_out: int, V: int) -> int:
    return int(load().beam_step_gumbel_workspace_size(R, B_in, n_out, V))


def beam_step_gumbel(trie, step, logits, parent_scores, parent_nodes, R, B_in, n_out, V,
                     temperature, seed, out_scores, out_parent, out_code, out_node, workspace,
                     stream=None, ld=None):
    """Gumbel top-k step at `temperature` (0: the deterministic step); `seed`
    keys the Philox stream. Outputs in draw order; scores unperturbed."""
    if ld is None:
        ld = logits.stride(0)
    rc = load().beam_step_gumbel(None if trie is None else trie.handle, step, _ptr(logits),
                                 _dtype_code(logits), ld, _ptr(parent_scores),
                                 _ptr(parent_nodes), R, B_in, n_out, V, float(temperature),
                                 int(seed) & 0xFFFFFFFFFFFFFFFF, _ptr(out_scores),
                                 _ptr(out_parent), _ptr(out_code), _ptr(out_node),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check(rc)


def beam_step_skipped_rows(workspace, stream=None) -> int:
    """Rows row skipping left unread since the last call (the counter resets)."""
    c = ctypes.c_uint32(0)
    _check(load().beam_step_skipped_rows(_ptr(workspace), ctypes.byref(c), _stream(stream)))
    return int(c.value)


def beam_step_noalloc(trie, step, logits, parent_scores, parent_nodes, R, B_in, n_out, V,
                      out_scores, out_parent, out_code, out_node, stream=None, ld=None):
    """beam_step with the library's built-in scratch instead of a workspace; for
    callers that cannot allocate device memory. Calls must not overlap on the GPU."""
    if ld is None:
        ld = logits.stride(0)
    rc = load().beam_step_noalloc(None if trie is None else trie.handle, step, _ptr(logits),
                                  _dtype_code(logits), ld, _ptr(parent_scores),
                                  _ptr(parent_nodes), R, B_in, n_out, V, _ptr(out_scores),
                                  _ptr(out_parent), _ptr(out_code), _ptr(out_node),
                                  _stream(stream))
    _check(rc)


def beam_finalize(depth, R, n, bp_parent, bp_code, last_node, out_sids, out_leaf, stream=None):
    _check(load().beam_finalize(depth, R, n, _ptr(bp_parent), _ptr(bp_code), _ptr(last_node),
                                _ptr(out_sids), _ptr(out_leaf), _stream(stream)))


def catalog_score_workspace_size(trie: Trie, R: int, K: int) -> int:
    return int(load().catalog_score_workspace_size(trie.handle, R, K))


def catalog_score_topk(trie, logp, R, K, out_scores, out_leaf, workspace, stream=None):
    rc = load().catalog_score_topk(trie.handle, _ptr(logp), R, K, _ptr(out_scores),
                                   _ptr(out_leaf), _ptr(workspace),
                                   0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check(rc)


def catalog_score_topk_sim(trie, logp, user, sid_emb, R, K, out_scores, out_leaf, workspace,
                           stream=None):
    """catalog_score_topk plus <user[r], sid_emb[leaf]>: user f32 [R][d], sid_emb
    bf16 [N][d] (leaf-id order), both on the device."""
    d = int(user.shape[1])
    if int(sid_emb.shape[1]) != d:
        raise ValueError("user and sid_emb disagree on d")
    rc = load().catalog_score_topk_sim(trie.handle, _ptr(logp), _ptr(user), _ptr(sid_emb), d, R,
                                       K, _ptr(out_scores), _ptr(out_leaf), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream))
    _check(rc)


def lmhead_logits(hidden, w_sid, out, workspace, stream=None):
    """out[row][c] = sum_k hidden[row][k] * w_sid[c][k] (bf16 in, fp32 out) on the
    tensor cores. hidden [M][d], w_sid [V][d] bf16; out f32 [M][>= V]."""
    M, d = hidden.shape
    V = w_sid.shape[0]
    _check(load().lmhead_logits(_ptr(hidden), _ptr(w_sid), M, V, d, _ptr(out), out.stride(0),
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream)))


def fused_lmhead_workspace_size(R: int, B_in: int, n_out: int, V: int) -> int:
    return int(load().fused_lmhead_workspace_size(R, B_in, n_out, V))


def fused_lmhead_step(trie, step, hidden, w_sid, parent_scores, parent_nodes, R, B_in, n_out,
                      out_scores, out_parent, out_code, out_node, workspace, stream=None):
    """beam_step on logits = hidden @ w_sid.T made on the tensor cores and never
    written out. hidden bf16 [R*B_in][d], w_sid bf16 [V][d]."""
    d = hidden.shape[1]
    V = w_sid.shape[0]
    rc = load().sidbeam_fused_lmhead_step(
        None if trie is None else trie.handle, step, _ptr(hidden), _ptr(w_sid), d,
        _ptr(parent_scores), _ptr(parent_nodes), R, B_in, n_out, V, _ptr(out_scores),
        _ptr(out_parent), _ptr(out_code), _ptr(out_node), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc)


def sidbeam_get_device_status(workspace, stream=None) -> int:
    return int(load().sidbeam_get_device_status(_ptr(workspace), _stream(stream)))
