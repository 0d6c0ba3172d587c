"""Host (numpy) twin of the seeded input generators.

Every routine here is integer arithmetic on numpy uint32/uint64 arrays plus,
for normal draws, one correctly rounded fp32 multiply. The CUDA twin in
``csrc/sidgen.cu`` computes the same bits.

Published definitions used:

* Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
  as 1, 2, 3", SC'11 -- multipliers 0xD2511F53 / 0xCD9E8D57, Weyl key
  increments 0x9E3779B9 / 0xBB67AE85, ten rounds, key bumped between rounds.
* SplitMix64: Steele, Lea, Flood, "Fast splittable pseudorandom number
  generators", OOPSLA'14 -- state increment 0x9E3779B97F4A7C15 and the
  variant-13 finaliser (shifts 30/27/31, multipliers 0xBF58476D1CE4E5B9 and
  0x94D049BB133111EB).
* Irwin-Hall: the sum of eight independent uniform 16-bit integers, centred and
  scaled, approximates a normal with the requested standard deviation (tails
  bounded near +-4.9 sigma).
* Zipf(s) over codes 0..V-1: P(code = k-1) proportional to k**-s, sampled by
  inverse CDF in double precision.
"""
from __future__ import annotations

import math
from typing import Sequence

import numpy as np

# Philox4x32 constants (Salmon et al., SC'11).
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = 0x9E3779B9
_PHILOX_W1 = 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)

# SplitMix64 constants (Steele et al., OOPSLA'14).
GOLDEN_GAMMA = 0x9E3779B97F4A7C15
_SM_C1 = np.uint64(0xBF58476D1CE4E5B9)
_SM_C2 = np.uint64(0x94D049BB133111EB)

# Seed of the prefix-hash chain: the first 64 bits of pi's fractional part, a
# nothing-up-my-sleeve constant. Request r's empty prefix (its trie root) hashes
# to mix(PREFIX_HASH_SEED ^ r): each request stands for its own context, so
# concurrent requests search different logits.
PREFIX_HASH_SEED = 0x243F6A8885A308D3

# Counter word 3 separates the independent streams that one seed feeds.
STREAM_BEAM_LOGITS = 0
STREAM_TABLE = 1
STREAM_HIDDEN = 2
STREAM_WEIGHT = 3
STREAM_USER = 4
STREAM_SID_EMB = 5

_IH_TERMS = 8            # eight 16-bit uniforms per normal draw
_IH_MAX = 65535
_IH_CENTRE = _IH_TERMS * _IH_MAX   # 2*sum - centre is symmetric about 0


def _u64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.uint64)


def splitmix64_mix(z) -> np.ndarray:
    """SplitMix64 finaliser on uint64 values (wrapping arithmetic)."""
    z = _u64(z).copy()
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _SM_C1
        z ^= z >> np.uint64(27)
        z *= _SM_C2
        z ^= z >> np.uint64(31)
    return z


def splitmix64_stream(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of the SplitMix64 stream seeded with ``seed``.

    Output i (0-based) is mix(seed + (i+1)*gamma mod 2**64).
    """
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = _u64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _u64(GOLDEN_GAMMA)
    return splitmix64_mix(state)


def root_hash(request=0):
    """Hash of request ``request``'s empty prefix (scalar or array of requests)."""
    r = _u64(request)
    h = splitmix64_mix(_u64(PREFIX_HASH_SEED) ^ r)
    return h if h.ndim else np.uint64(h)


def request_roots(R: int) -> np.ndarray:
    """Root hashes of requests 0 .. R-1 (uint64 [R])."""
    return root_hash(np.arange(R, dtype=np.uint64))


def child_hash(parent_hash, level: int, code) -> np.ndarray:
    """Hash of a prefix extended by ``code`` at 1-based ``level``."""
    tag = (np.uint64(level) << np.uint64(48)) | _u64(code)
    return splitmix64_mix(_u64(parent_hash) ^ tag)


def prefix_hashes(prefixes: np.ndarray, requests=None) -> np.ndarray:
    """Hashes of an array of prefixes [rows, l] (l may be 0) of the given
    requests (int array [rows]; all request 0 when omitted)."""
    prefixes = np.asarray(prefixes)
    rows = prefixes.shape[0]
    if requests is None:
        h = np.full(rows, root_hash(0), dtype=np.uint64)
    else:
        h = root_hash(np.asarray(requests, dtype=np.uint64).reshape(rows))
    for lv in range(prefixes.shape[1]):
        h = child_hash(h, lv + 1, prefixes[:, lv].astype(np.uint64))
    return h


def philox4x32_10(c0, c1, c2, c3, seed: int):
    """Philox4x32 with ten rounds on arrays of counters; key = (seed lo32, seed hi32)."""
    x0, x1, x2, x3 = (_u64(c) & _MASK32 for c in (c0, c1, c2, c3))
    x0, x1, x2, x3 = np.broadcast_arrays(x0, x1, x2, x3)
    x0, x1, x2, x3 = (a.copy() for a in (x0, x1, x2, x3))
    k0 = seed & 0xFFFFFFFF
    k1 = (seed >> 32) & 0xFFFFFFFF
    for rnd in range(10):
        if rnd:
            k0 = (k0 + _PHILOX_W0) & 0xFFFFFFFF
            k1 = (k1 + _PHILOX_W1) & 0xFFFFFFFF
        p0 = x0 * _PHILOX_M0
        p1 = x2 * _PHILOX_M1
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        x0, x1, x2, x3 = (hi1 ^ x1 ^ np.uint64(k0), lo1, hi0 ^ x3 ^ np.uint64(k1), lo0)
    return (x0.astype(np.uint32), x1.astype(np.uint32),
            x2.astype(np.uint32), x3.astype(np.uint32))


def k_sigma(sigma: float) -> np.float32:
    """fp32 scale that maps the centred Irwin-Hall integer to standard deviation sigma.

    2*sum of eight uniforms on {0..65535} has variance 4*8*(65536**2 - 1)/12;
    the 65536**2 approximation is used (relative error 2e-10).
    """
    return np.float32(sigma / (65536.0 * math.sqrt(8.0 / 3.0)))


def normal_from_counters(seed: int, c0, c1, c2, c3, sigma: float) -> np.ndarray:
    """One approximately N(0, sigma) fp32 draw per Philox counter."""
    r = philox4x32_10(c0, c1, c2, c3, seed)
    s = np.zeros(r[0].shape, dtype=np.int64)
    for w in r:
        w64 = w.astype(np.int64)
        s += (w64 & 0xFFFF) + (w64 >> 16)
    centred = (2 * s - _IH_CENTRE).astype(np.float32)   # exact: |.| < 2**24
    return centred * k_sigma(sigma)                     # one rounded fp32 multiply


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); finite inputs only."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + rounding) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def row_logits(seed: int, hashes: np.ndarray, V: int, sigma: float,
               dtype: str = "f32", stream: int = STREAM_BEAM_LOGITS,
               chunk_rows: int = 256) -> np.ndarray:
    """Logits [rows, V]: element (row, c) = N(0, sigma) draw at counter (h lo, h hi, c, stream).

    ``dtype`` "f32" returns float32; "bf16" returns the bf16 bit patterns (uint16).
    """
    hashes = _u64(hashes).reshape(-1)
    rows = hashes.shape[0]
    out = np.empty((rows, V), dtype=np.float32 if dtype == "f32" else np.uint16)
    codes = np.arange(V, dtype=np.uint64)[None, :]
    for r0 in range(0, rows, chunk_rows):
        h = hashes[r0:r0 + chunk_rows, None]
        x = normal_from_counters(seed, h & _MASK32, h >> np.uint64(32), codes,
                                 np.uint64(stream), sigma)
        out[r0:r0 + chunk_rows] = x if dtype == "f32" else f32_to_bf16_bits(x)
    return out


def table_logits(seed: int, R: int, L: int, V: int, sigma: float) -> np.ndarray:
    """Per-request, per-position score tables [R, L, V] fp32 at counters (r, l, c, STREAM_TABLE)."""
    r = np.arange(R, dtype=np.uint64)[:, None, None]
    lv = np.arange(L, dtype=np.uint64)[None, :, None]
    c = np.arange(V, dtype=np.uint64)[None, None, :]
    return normal_from_counters(seed, r, lv, c, np.uint64(STREAM_TABLE), sigma)


def hidden_states(seed: int, hashes: np.ndarray, d: int, sigma: float = 1.0) -> np.ndarray:
    """bf16 bits [rows, d] at counters (h lo, h hi, k, STREAM_HIDDEN)."""
    h = _u64(hashes).reshape(-1, 1)
    k = np.arange(d, dtype=np.uint64)[None, :]
    x = normal_from_counters(seed, h & _MASK32, h >> np.uint64(32), k,
                             np.uint64(STREAM_HIDDEN), sigma)
    return f32_to_bf16_bits(x)


def weight_matrix(seed: int, V: int, d: int, sigma: float = 0.02,
                  chunk_rows: int = 512) -> np.ndarray:
    """bf16 bits [V, d] at counters (c, k, 0, STREAM_WEIGHT)."""
    out = np.empty((V, d), dtype=np.uint16)
    k = np.arange(d, dtype=np.uint64)[None, :]
    for c0 in range(0, V, chunk_rows):
        c = np.arange(c0, min(V, c0 + chunk_rows), dtype=np.uint64)[:, None]
        x = normal_from_counters(seed, c, k, np.uint64(0), np.uint64(STREAM_WEIGHT), sigma)
        out[c0:c0 + c.shape[0]] = f32_to_bf16_bits(x)
    return out


def user_vectors(seed: int, R: int, d: int, sigma: float) -> np.ndarray:
    """Per-request user vectors f32 [R, d] at counters (r, k, 0, STREAM_USER)."""
    r = np.arange(R, dtype=np.uint64)[:, None]
    k = np.arange(d, dtype=np.uint64)[None, :]
    return normal_from_counters(seed, r, k, np.uint64(0), np.uint64(STREAM_USER), sigma)


def sid_embeddings(seed: int, N: int, d: int, sigma: float, chunk_rows: int = 4096) -> np.ndarray:
    """Per-SID embeddings, bf16 bits [N, d] (row j = leaf id j), at counters
    (j, k, 0, STREAM_SID_EMB)."""
    out = np.empty((N, d), dtype=np.uint16)
    k = np.arange(d, dtype=np.uint64)[None, :]
    for j0 in range(0, N, chunk_rows):
        j = np.arange(j0, min(N, j0 + chunk_rows), dtype=np.uint64)[:, None]
        x = normal_from_counters(seed, j, k, np.uint64(0), np.uint64(STREAM_SID_EMB), sigma)
        out[j0:j0 + j.shape[0]] = f32_to_bf16_bits(x)
    return out


# ---------------------------------------------------------------- catalogs

def _uniform_codes(x: np.ndarray, V: int) -> np.ndarray:
    # Lemire multiply-shift on the top 32 bits: exact integer map to [0, V).
    return (((x >> np.uint64(32)) * np.uint64(V)) >> np.uint64(32)).astype(np.int64)


def _zipf_cdf(V: int, s: float) -> np.ndarray:
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    return cdf / cdf[-1]


def _zipf_codes(x: np.ndarray, cdf: np.ndarray) -> np.ndarray:
    u = (x >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    return np.minimum(np.searchsorted(cdf, u, side="right"), cdf.shape[0] - 1).astype(np.int64)


def draw_catalog(seed: int, n_sids: int, codes_per_level: Sequence[int],
                 dists: Sequence = None) -> np.ndarray:
    """Draw SIDs until ``n_sids`` distinct ones are collected; returns int32 [n_sids, L].

    SID i (in draw order) takes stream outputs i*L .. i*L+L-1, one per level.
    ``dists[l]`` is "uniform" or ("zipf", s). Rows come back in order of first
    appearance; duplicates are dropped.
    """
    L = len(codes_per_level)
    if dists is None:
        dists = ["uniform"] * L
    total = 1
    for v in codes_per_level:
        total *= int(v)
    if n_sids > total:
        raise ValueError(f"cannot draw {n_sids} distinct SIDs from {total} possible")
    bits = [max(1, int(v - 1).bit_length()) for v in codes_per_level]
    if sum(bits) > 63:
        raise ValueError("catalog codes do not pack into 63 bits")
    cdfs = [None if d == "uniform" else _zipf_cdf(int(codes_per_level[i]), float(d[1]))
            for i, d in enumerate(dists)]

    drawn = []
    n_drawn = 0
    batch = max(1024, int(n_sids * 1.05))
    while True:
        x = splitmix64_stream(seed, n_drawn * L, batch * L).reshape(batch, L)
        sids = np.empty((batch, L), dtype=np.int64)
        for lv in range(L):
            if cdfs[lv] is None:
                sids[:, lv] = _uniform_codes(x[:, lv], int(codes_per_level[lv]))
            else:
                sids[:, lv] = _zipf_codes(x[:, lv], cdfs[lv])
        drawn.append(sids)
        n_drawn += batch
        allsids = np.concatenate(drawn)
        packed = np.zeros(allsids.shape[0], dtype=np.uint64)
        for lv in range(L):
            packed = (packed << np.uint64(bits[lv])) | allsids[:, lv].astype(np.uint64)
        _, first = np.unique(packed, return_index=True)
        if first.shape[0] >= n_sids:
            keep = np.sort(first)[:n_sids]
            return allsids[keep].astype(np.int32)
        batch = max(1024, int((n_sids - first.shape[0]) * 2 + 1024))
