"""Parity helpers: run the CUDA path and the oracle on the same seeded inputs
and compare them with the rule the target sets for floating-point selection:

* per request, the ranked scores must agree element-wise within TOL (abs);
* the selected (parent, code) pair -- and the child node -- at rank k must be
  identical whenever the oracle's scores at ranks k-1, k and k+1 are more than
  TOL apart (rank n+1, the first one left out, counts: the oracle is run with
  n+1 outputs for this);
* inside a near-tie group several answers are correct, so there the CUDA
  pair must be a valid, distinct candidate whose oracle score is within TOL.

TOL = 1e-5 follows from fp32 accumulation: |lse error| <= ~2e-6 (16-byte
vector tree sums, at most a few hundred terms per lane, ex2.approx relative
error 2^-22, logf within 1 ulp), plus one rounding of z - lse and one of
s + (z - lse), each at most half an ulp of a value below 64 in magnitude
(1.9e-6). Inputs are the same bits on both sides (bf16 widened exactly).
"""
from __future__ import annotations

import numpy as np

import oracle
from sidgen import host

TOL = 1e-5


def _widen(logits):
    a = np.asarray(logits)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def compare_step(gpu, trie, step, logits, parent_scores, parent_nodes, R, B_in, n, V, tol=TOL):
    """gpu: dict of host arrays [R, n] (score f32, parent, code, node).

    Runs the oracle step on exactly the GPU's inputs and applies the rule.
    Returns the number of ranks compared exactly (for reporting).
    """
    ext = oracle.beam_step(trie, step, logits, parent_scores, parent_nodes, R, B_in, n + 1, V)
    z = None
    exact = 0
    for r in range(R):
        os_ = ext["score"][r]
        gs = np.asarray(gpu["score"][r], dtype=np.float64)
        ov = int(np.isfinite(os_[:n]).sum())
        gv = int(np.isfinite(gs).sum())
        assert ov == gv, f"request {r}: oracle has {ov} beams, GPU {gv}"
        assert np.all(gpu["parent"][r, gv:] == -1) and np.all(gpu["code"][r, gv:] == -1)
        assert np.all(gpu["node"][r, gv:] == -1)
        if gv == 0:
            continue
        err = np.abs(gs[:gv] - os_[:gv]).max()
        assert err <= tol, f"request {r}: score error {err:.3g} > {tol}"
        pairs = set()
        for k in range(gv):
            gp, gc, gn = int(gpu["parent"][r, k]), int(gpu["code"][r, k]), int(gpu["node"][r, k])
            assert (gp, gc) not in pairs, f"request {r}: duplicate candidate ({gp}, {gc})"
            pairs.add((gp, gc))
            lo_gap = k == 0 or os_[k - 1] - os_[k] > tol
            hi_gap = (not np.isfinite(os_[k + 1])) or os_[k] - os_[k + 1] > tol
            if lo_gap and hi_gap:
                assert (gp, gc, gn) == (int(ext["parent"][r, k]), int(ext["code"][r, k]),
                                        int(ext["node"][r, k])), (
                    f"request {r} rank {k}: GPU {(gp, gc, gn)} oracle "
                    f"{(ext['parent'][r, k], ext['code'][r, k], ext['node'][r, k])}")
                exact += 1
                continue
            # Near-tie group: the GPU's pair must be a valid candidate with that score.
            if z is None:
                z = _widen(logits)
            row = r * B_in + gp
            assert 0 <= gp < B_in and 0 <= gc < V
            s = float(parent_scores[row])
            assert np.isfinite(s)
            lp = oracle.log_softmax_full(z[row, :V])
            assert abs(s + lp[gc] - gs[k]) <= tol
            if trie is not None:
                codes, ids = trie.children(step, int(parent_nodes[row]))
                hit = np.flatnonzero(codes == gc)
                assert hit.size == 1, f"request {r} rank {k}: code {gc} is not a child"
                assert int(ids[hit[0]]) == gn
            else:
                assert gn == -1
    return exact


# ---------------------------------------------------------------- GPU search
def run_gpu_search(trie_gpu, R, n, depth, V, seed, sigma, dtype, ld_pad=0, on_step=None,
                   stream=None):
    """Constrained search on the device with device-generated logits keyed by prefix hash.

    on_step(t, logits, parent_scores, parent_nodes, B_in, outputs) is called
    after each step with device tensors (for step-local parity).
    """
    import torch

    import trie_constrained_beam_b200 as tcb
    from sidgen import device as gdev

    search = tcb.BeamSearch(trie_gpu, R, n, V, depth=depth)
    hashes = torch.from_numpy(host.request_roots(R).view(np.int64)).to("cuda")
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    elem = 4 if dtype == "f32" else 2
    for t in range(depth):
        rows = search.rows(t)
        ld = V + ld_pad
        ld = (ld * elem + 15) // 16 * 16 // elem
        logits = torch.empty((rows, ld), dtype=tdt, device="cuda")
        gdev.row_logits(seed, hashes, V, sigma, logits)
        search.step(t, logits, stream=stream)
        status = tcb.sidbeam_get_device_status(search.workspace)
        assert status == 0, f"device status {status} after step {t}"
        ps, pn, B_in = search.parents(t)
        if on_step is not None:
            on_step(t, logits, ps, pn, B_in,
                    dict(score=search.scores[t], parent=search.bp_parent[t],
                         code=search.bp_code[t], node=search.nodes[t]))
        child = torch.empty((R * n,), dtype=torch.int64, device="cuda")
        gdev.child_hash(hashes, R, B_in, search.bp_parent[t], search.bp_code[t], n, t + 1, child)
        hashes = child
    sids, leaf, scores = search.finalize(stream=stream)
    return search, sids, leaf, scores


def to_host_logits(logits, V):
    import torch
    x = logits[:, :V].contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).cpu().numpy().view(np.uint16)
    return x.cpu().numpy()


def oracle_search_with_gaps(trie, R, n, depth, V, seed, sigma, dtype, widths=None):
    """Oracle search (host generator) that also reports, per request, the smallest
    gap over steps between the n-th and the (n+1)-th candidate: a near-tie there
    changes the beam set, so end-to-end parity is only defined where it is wide.
    widths: beams kept per request (each <= n); the gap is then the one at the
    request's own width, and slots past it are padding (as oracle.beam_search)."""
    def fn(step, prefixes, requests):
        return host.row_logits(seed, host.prefix_hashes(prefixes, requests), V, sigma,
                               dtype=dtype)

    scores = np.zeros(R)
    nodes = np.zeros(R, dtype=np.int64)
    prefixes = np.zeros((R, 1, 0), dtype=np.int64)
    B_in = 1
    min_gap = np.full(R, np.inf)
    bpp, bpc, outs = [], [], []
    for t in range(depth):
        flat = prefixes.reshape(R * B_in, t)
        live = np.flatnonzero(scores > -np.inf)
        z = np.zeros((R * B_in, V))
        if live.size:
            z[live] = _widen(fn(t, flat[live], live // B_in))
        ext = oracle.beam_step(trie, t, z, scores, nodes, R, B_in, n + 1, V)
        sc = ext["score"]
        for r in range(R):   # boundary gap: the last kept vs the first left out
            wr = n if widths is None else int(widths[r])
            if wr > 0 and np.isfinite(sc[r, wr]):
                min_gap[r] = min(min_gap[r], float(sc[r, wr - 1] - sc[r, wr]))
        out = {k: v[:, :n].copy() for k, v in ext.items()}
        if widths is not None:
            for r, wr in enumerate(widths):
                out["score"][r, wr:] = -np.inf
                for k in ("parent", "code", "node"):
                    out[k][r, wr:] = -1
        outs.append(out)
        bpp.append(out["parent"])
        bpc.append(out["code"])
        newp = np.full((R, n, t + 1), -1, dtype=np.int64)
        for r in range(R):
            for k in range(n):
                p = out["parent"][r, k]
                if p >= 0:
                    newp[r, k, :t] = prefixes[r, p]
                    newp[r, k, t] = out["code"][r, k]
        prefixes, scores, nodes, B_in = newp, out["score"].reshape(-1), out["node"].reshape(-1), n
    fin = oracle.beam_finalize(np.stack(bpp), np.stack(bpc), outs[-1]["score"], outs[-1]["node"])
    fin["min_gap"] = min_gap
    fin["steps"] = outs
    return fin
