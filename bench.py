"""Benchmark: catalog-constrained wide-beam expansion on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One timed step = one whole constrained beam search of the wide-beam workload
(16 requests x beam 512, depth 5, 4,096 codes per level, 8M-SID catalog with a
dense trie on levels 1-2 and CSR below, bf16 logits): five beam_step launches
plus beam_finalize. The per-step logits are the ones the search consumes (made
once by the seeded generator, keyed by prefix hash) and are resident in HBM
when the timed region starts; three rotating copies (3 x 256 MiB + step 0)
keep every step's reads out of L2.

Printed: one JSON line (rank 0). `value` = logits scored per second over all
ranks (live rows x V summed over the five steps, per search). Multi-GPU runs
are weak-scaled replicas: requests are independent, every rank searches its
own batch, nothing crosses GPUs in the data path.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "beam-step logits scored/sec & achieved HBM GB/s (% of B200 peak) at beam 512"
UNIT = "logits/s"
CFG = 4
COPIES = 3
SM_COUNT = 148      # B200 streaming multiprocessors
SM_MAX_MHZ = 1965   # clocks.max.sm of the B200s measured here


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _max_over_ranks(x: float, device) -> float:
    """The largest of every rank's x: a collective, so every rank calls it at
    the same point (one process: x itself)."""
    import torch
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _workload_config(w, extra=None):
    cfg = {
        "workload": w.name,
        "requests": w.R,
        "beam": w.n,
        "depth": w.depth,
        "codes_per_level": w.V,
        "catalog_sids": w.n_sids,
        "trie_layout": "dense bitmask levels 1-2, CSR levels 3-5",
        "logits_dtype": w.dtype,
        "l2": "inputs larger than L2: 3 rotating copies of the per-step logits (5 steps, 256 MiB + step 0 each)",
    }
    if extra:
        cfg.update(extra)
    return cfg


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, path):
        self.path = path
        self.proc = None
        try:
            self.f = open(path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        busy = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in busy),
                "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(busy), "reasons": reasons}


# ----------------------------------------------------------------- our arm
def run_ours(args, world, rank, local):
    import torch

    import trie_constrained_beam_b200 as tcb
    from sidgen import device as gdev
    from sidgen import host
    from sidgen.workloads import WORKLOADS
    from trie_constrained_beam_b200 import build as tbuild

    # The oracle's tries and a pool of worker processes over all host cores,
    # forked before the first CUDA call (a process forked after it cannot use
    # the parent's CUDA state and can hang); workers inherit the tries.
    pool = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pool = _start_oracle_pool(CFG, *(() if args.no_config_lines else (1, 2, 3)))
    torch.cuda.set_device(local)
    if rank == 0:
        tbuild.build()
        gdev.build()
    if world > 1:
        torch.distributed.barrier()
    w = WORKLOADS[CFG]
    dev = torch.device("cuda", local)
    cat = w.catalog()
    trie = tcb.sid_trie_build(cat, w.codes_per_level, w.layouts)
    search = tcb.BeamSearch(trie, w.R, w.n, w.V, depth=w.depth)
    stream = torch.cuda.current_stream()

    # 1. Generate the search's logits once (generator keyed by prefix hash).
    hashes = torch.from_numpy(host.request_roots(w.R).view(np.int64)).to(dev)
    base = []
    live_rows = []
    for t in range(w.depth):
        rows = search.rows(t)
        lg = torch.empty((rows, w.V), dtype=torch.bfloat16, device=dev)
        gdev.row_logits(w.logits_seed, hashes, w.V, w.sigma, lg)
        ps, pn, B_in = search.parents(t)
        live_rows.append(int(torch.isfinite(ps).sum().item()))
        search.step(t, lg)
        child = torch.empty((w.R * w.n,), dtype=torch.int64, device=dev)
        gdev.child_hash(hashes, w.R, B_in, search.bp_parent[t], search.bp_code[t], w.n, t + 1, child)
        hashes = child
        base.append(lg)
    search.finalize()
    ref_sids = search.sids.clone()
    assert tcb.sidbeam_get_device_status(search.workspace) == 0
    sets = [base] + [[x.clone() for x in base] for _ in range(args.copies - 1)]
    torch.cuda.synchronize()

    esize = 2
    logits_per_search = sum(r * w.V for r in live_rows)
    mask_row = ((w.V + 31) // 32 + 3) // 4 * 4 * 4
    step_bytes = []
    for t in range(w.depth):
        b = live_rows[t] * w.V * esize + live_rows[t] * 8 + w.R * w.n * 16
        if w.layouts[t] == 1:
            b += live_rows[t] * mask_row
        step_bytes.append(b)

    # 2. One CUDA graph per logits copy (five beam_step launches + finalize);
    #    the timed region replays them in rotation. A second set of graphs with
    #    events between the launches gives each step's device time.
    graphs = [search.capture(sets[i]) for i in range(len(sets))]
    ev_sets = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(w.depth + 2)]
               for _ in range(len(sets))]
    ev_graphs = [search.capture(sets[i], events=ev_sets[i]) for i in range(len(sets))]
    torch.cuda.synchronize()
    for i in range(args.warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    assert torch.equal(search.sids, ref_sids), "replay diverged from the generated search"

    K = args.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # Raw nvidia-smi samples go to --clocks-dir (kept) or a temporary file; the
    # JSON line carries their summary either way.
    clk_dir = args.clocks_dir or tempfile.gettempdir()
    clocks = ClockSampler(local, os.path.join(clk_dir, f"clocks_rank{rank}.csv"))
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        graphs[i % len(graphs)].replay()
    stop.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    elapsed_ms = start.elapsed_time(stop)
    if world > 1:
        elapsed_ms = _max_over_ranks(elapsed_ms, dev)
    assert torch.equal(search.sids, ref_sids)
    assert tcb.sidbeam_get_device_status(search.workspace) == 0

    # Per-step device times (graph replays with events, outside the timed region).
    reps = max(30, min(300, K // 4))
    acc = [[0.0] * (w.depth + 1) for _ in range(len(sets))]
    cnt = [0] * len(sets)
    for i in range(reps):
        j = i % len(sets)
        ev_graphs[j].replay()
        torch.cuda.synchronize()
        ev = ev_sets[j]
        for t in range(w.depth + 1):
            acc[j][t] += ev[t].elapsed_time(ev[t + 1])
        cnt[j] += 1
    per_step_us = [1e3 * sum(acc[j][t] for j in range(len(sets))) / sum(cnt) for t in range(w.depth)]
    finalize_us = 1e3 * sum(acc[j][w.depth] for j in range(len(sets))) / sum(cnt)
    steady = list(range(1, w.depth))
    dur_us = statistics.mean(per_step_us[t] for t in steady)
    bytes_launch = statistics.mean(step_bytes[t] for t in steady)
    peak, peak_kind = _peaks()
    achieved = bytes_launch / (dur_us * 1e-6) / 1e9
    value = world * K * logits_per_search / (elapsed_ms * 1e-3)

    # 3. End to end through the C ABI with host buffers: per search, copy every
    #    step's logits from pinned host memory, run, copy the results back.
    e2e = None
    if not args.no_e2e:
        pinned = [x.cpu().pin_memory() for x in base]
        dbuf = [torch.empty_like(x) for x in base]
        out_sids = torch.empty(search.sids.shape, dtype=torch.int32).pin_memory()
        out_leaf = torch.empty(search.leaf.shape, dtype=torch.int32).pin_memory()
        out_score = torch.empty((w.R, w.n), dtype=torch.float32).pin_memory()
        K2 = max(3, min(50, K // 20))

        def e2e_search():
            for t in range(w.depth):
                dbuf[t].copy_(pinned[t], non_blocking=True)
                search.step(t, dbuf[t], stream=stream)
            sids, leaf, scores = search.finalize(stream=stream)
            out_sids.copy_(sids, non_blocking=True)
            out_leaf.copy_(leaf, non_blocking=True)
            out_score.copy_(scores, non_blocking=True)

        for _ in range(2):
            e2e_search()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K2):
            e2e_search()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1)
        if world > 1:
            ems = _max_over_ranks(ems, dev)
        assert torch.equal(out_sids, ref_sids.cpu())
        h2d = sum(x.numel() * x.element_size() for x in pinned)
        d2h = out_sids.numel() * 4 + out_leaf.numel() * 4 + out_score.numel() * 4
        e2e = {"value": world * K2 * logits_per_search / (ems * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K2}

    cat_lines = None
    if not args.no_catalog:
        cat_lines = measure_catalog(tcb, trie, cat, w, dev)
    fused = None
    if not args.no_fused:
        fused = measure_fused(tcb, dev)
    gumbel = None
    if not args.no_gumbel:
        gumbel = measure_gumbel(tcb, trie, w, base, dev)
    widths = None
    if not args.no_widths:
        widths = measure_widths(tcb, trie, w, base, dev)

    configs = None
    if not args.no_config_lines:
        configs = {f"config{c}": measure_config(tcb, c, dev, pool, args.cpu_seconds / 3)
                   for c in (1, 2, 3)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, base, search, live_rows, budget_s=args.cpu_seconds, pool=pool)
    if pool is not None:
        pool.terminate()

    traffic, traffic_kernel = _profile_traffic()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": _workload_config(w, {"parallelism": f"replicas x{world} (requests sharded)"}),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "traffic_kernel": traffic_kernel,
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                     "kernel": "beam_step_kernel<bf16>, steady steps 1-4",
                     "bytes_per_launch": bytes_launch, "us_per_launch": dur_us},
        "step_us": per_step_us,
        "finalize_us": finalize_us,
        "timing": "CUDA graph replays of the whole search (5 beam_step + beam_finalize), "
                  "3 rotating logits copies; per-step times from events inside the graph",
        "logits_per_step": logits_per_search,
        "e2e": e2e,
        "catalog_score": cat_lines,
        "fused_lmhead": fused,
        "gumbel_top_k": gumbel,
        "per_request_widths": widths,
        "other_configs": configs,
        "cpu_baseline": cpu,
        "clocks": clk,
        "gpu_launches": K * (w.depth + 1),
    }
    return line


def measure_catalog(tcb, trie4, cat4, w4, dev):
    """catalog_score_topk throughput ((request, SID) pairs scored per second):
    the SPRINT-like workload (32 requests, 50,000 SIDs, 4 x 256, top-10) and the
    wide-beam catalog (8M SIDs, 5 x 4096) with 32 requests, top-10. Tables are
    seeded per-position log-softmax tables, resident in HBM."""
    import torch
    from sidgen import host
    from sidgen.workloads import WORKLOADS

    def run(trie, n_leaves, R, L, V, K, seed, sigma, reps=50, sim=None):
        table = torch.from_numpy(host.table_logits(seed, R, L, V, sigma)).to(dev).log_softmax(-1)
        table = table.contiguous()
        out_s = torch.empty((R, K), device=dev)
        out_l = torch.empty((R, K), dtype=torch.int32, device=dev)
        ws = torch.zeros(tcb.catalog_score_workspace_size(trie, R, K), dtype=torch.uint8, device=dev)
        if sim is not None:  # (user f32 [R, d], SID embeddings bf16 bits [N, d])
            u = torch.from_numpy(sim[0]).to(dev)
            e = torch.from_numpy(np.ascontiguousarray(sim[1]).view(np.int16)).to(dev)

            def call():
                tcb.catalog_score_topk_sim(trie, table, u, e, R, K, out_s, out_l, ws)
        else:
            def call():
                tcb.catalog_score_topk(trie, table, R, K, out_s, out_l, ws)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            call()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / reps
        assert tcb.sidbeam_get_device_status(ws) == 0
        out = {"us_per_call": us, "pairs_per_s": R * n_leaves / (us * 1e-6),
               "requests": R, "sids": n_leaves, "depth": L, "codes_per_level": V, "K": K}
        # Roofline: every (request, SID, level) is one 4-byte shared-memory table
        # lookup; the pipe serves one word per lane per clock on each SM.
        lookups = float(R) * n_leaves * L
        peak = SM_COUNT * 32 * SM_MAX_MHZ * 1e6
        out["roofline"] = {"bound": "alu", "unit": "lookups/s", "achieved": lookups / (us * 1e-6),
                           "peak": peak, "frac": lookups / (us * 1e-6) / peak,
                           "peak_source": f"{SM_COUNT} SMs x 32 lanes x {SM_MAX_MHZ} MHz "
                                          "(one shared-memory word per lane per clock)",
                           "code_bytes": n_leaves * L * 2, "table_bytes": R * L * V * 4}
        if sim is not None:
            out["similarity_dim"] = int(sim[0].shape[1])
        return out

    w2 = WORKLOADS[2]
    cat2 = w2.catalog()
    trie2 = tcb.sid_trie_build(cat2, w2.codes_per_level, w2.layouts)
    a = run(trie2, _n_leaves(cat2), w2.R, w2.depth, w2.V, w2.K, w2.logits_seed, w2.table_sigma)
    n2 = _n_leaves(cat2)
    sim2 = (host.user_vectors(w2.sim_seed, w2.R, w2.sim_dim, w2.user_sigma),
            host.sid_embeddings(w2.sim_seed, n2, w2.sim_dim, w2.emb_sigma))
    a2 = run(trie2, n2, w2.R, w2.depth, w2.V, w2.K, w2.logits_seed, w2.table_sigma, sim=sim2)
    b = run(trie4, _n_leaves(cat4), 32, w4.depth, w4.V, 10, w4.logits_seed + 7, 1.5, reps=10)
    return {"unit": "(request, SID) pairs/s", "sprint_opq_50k": a,
            "sprint_opq_50k_with_similarity": a2, "wide_beam_8M_x32": b}


def measure_gumbel(tcb, trie, w, base, dev, reps=10):
    """The wide-beam search with Gumbel top-k draws at temperature 1 (beam_step_gumbel)
    on the deterministic search's logits tensors (same shapes; the drawn beams
    differ): per-step device times from events between eager launches, and
    logits scored per second over the whole search."""
    import torch

    def steps_us(search):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(w.depth + 1)]

        def once(record):
            for t in range(w.depth):
                if record:
                    evs[t].record()
                search.step(t, base[t])
            if record:
                evs[w.depth].record()

        for _ in range(2):
            once(False)
        torch.cuda.synchronize()
        per = np.zeros(w.depth)
        for _ in range(reps):
            once(True)
            torch.cuda.synchronize()
            per += [evs[t].elapsed_time(evs[t + 1]) * 1e3 for t in range(w.depth)]
        assert tcb.sidbeam_get_device_status(search.workspace) == 0
        return per / reps

    search = tcb.BeamSearch(trie, w.R, w.n, w.V, depth=w.depth, temperature=1.0,
                            seed=0x5EED_0F_6B3E1)
    per = steps_us(search)
    det = steps_us(tcb.BeamSearch(trie, w.R, w.n, w.V, depth=w.depth))
    logits = sum(search.rows(t) * w.V for t in range(w.depth))
    return {"temperature": 1.0, "step_us": [float(x) for x in per],
            "deterministic_step_us": [float(x) for x in det],
            "ratio_to_deterministic": [float(x / y) for x, y in zip(per, det)],
            "logits_per_s": logits / (per.sum() * 1e-6),
            "timing": "eager launches, events between steps, 10 searches each (the "
                      "deterministic search timed the same way on the same logits)",
            "note": "rows of up to 8 KB in registers; one Philox draw per code that "
                    "could reach the threshold"}


def measure_widths(tcb, trie, w, base, dev, reps=50):
    """The wide-beam search with per-request widths 512, 384, 256, 128 (cycling
    over the 16 requests) in one launch per step, the whole search (5 steps +
    finalize) replayed as one CUDA graph on the deterministic search's logits;
    slots past a request's width are dead rows of the next step (not read)."""
    import torch
    widths = [(512, 384, 256, 128)[r % 4] for r in range(w.R)]
    search = tcb.BeamSearch(trie, w.R, w.n, w.V, depth=w.depth, widths=widths)
    for t in range(w.depth):
        search.step(t, base[t])
    search.finalize()
    torch.cuda.synchronize()
    g = search.capture(base)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    assert tcb.sidbeam_get_device_status(search.workspace) == 0
    live = w.R * w.V + sum(widths) * w.V * (w.depth - 1)   # rows scored: roots + kept beams
    return {"widths": "512/384/256/128 cycling over 16 requests", "us_per_search": us,
            "logits_per_s": live / (us * 1e-6),
            "timing": "CUDA graph of the whole search (5 beam_step + beam_finalize), 50 replays"}


def measure_fused(tcb, dev, reps=20):
    """The fused lm_head workload (32 requests x beam 128 = 4,096 rows, d = 2,048,
    V = 8,192, 1M-SID catalog): the tcgen05 GEMM alone (fp32 logits written) and
    the whole fused step 1 (child bitmaps + GEMM with the lse/child epilogue +
    selection; logits never written). Seeded inputs resident in HBM."""
    import torch
    from sidgen import host
    from sidgen.workloads import WORKLOADS

    w = WORKLOADS[5]
    M, V, d, R, B_in, n = w.R * w.n, w.V, w.hidden_dim, w.R, w.n, w.n
    rng = np.random.default_rng(5005)
    hashes = rng.integers(0, 2 ** 63, size=M, dtype=np.int64).view(np.uint64)
    h = torch.from_numpy(host.hidden_states(w.logits_seed, hashes, d, w.hidden_sigma)
                         .view(np.int16)).to(dev).view(torch.bfloat16)
    wt = torch.from_numpy(host.weight_matrix(w.weight_seed, V, d, w.weight_sigma)
                          .view(np.int16)).to(dev).view(torch.bfloat16)
    cat = w.catalog()
    trie = tcb.sid_trie_build(cat, w.codes_per_level, w.layouts)
    n1 = int(tcb.sid_trie_info(trie, 1)[0])
    pn = torch.from_numpy(np.concatenate([rng.choice(n1, size=B_in, replace=False)
                                          for _ in range(R)]).astype(np.int32)).to(dev)
    ps = torch.from_numpy(np.concatenate([np.sort(rng.uniform(-12, -2, size=B_in))[::-1]
                                          for _ in range(R)]).astype(np.float32)).to(dev)
    logits = torch.empty((M, V), dtype=torch.float32, device=dev)
    ws0 = torch.zeros(256, dtype=torch.uint8, device=dev)
    outs = [torch.empty(R * n, dtype=torch.float32, device=dev)] + \
        [torch.empty(R * n, dtype=torch.int32, device=dev) for _ in range(3)]
    ws = torch.zeros(tcb.fused_lmhead_workspace_size(R, B_in, n, V), dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / reps

    us_gemm = timed(lambda: tcb.lmhead_logits(h, wt, logits, ws0))
    us_step = timed(lambda: tcb.fused_lmhead_step(trie, 1, h, wt, ps, pn, R, B_in, n, *outs, ws))
    assert tcb.sidbeam_get_device_status(ws) == 0 and tcb.sidbeam_get_device_status(ws0) == 0
    flops = 2.0 * M * V * d
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peak = float(json.load(open(pk))["bf16_tflops"]) if os.path.exists(pk) else 1590.0
    return {"rows": M, "V": V, "d": d, "gflop_per_step": flops / 1e9,
            "gemm_us": us_gemm, "gemm_tflops": flops / (us_gemm * 1e-6) / 1e12,
            "gemm_frac_of_bf16_peak": flops / (us_gemm * 1e-6) / 1e12 / peak,
            "bf16_peak_tflops": peak, "fused_step_us": us_step,
            "fused_step_tflops": flops / (us_step * 1e-6) / 1e12}


def _n_leaves(cat):
    return int(np.asarray(cat).shape[0])  # the recipes draw distinct SIDs


def _profile_traffic():
    """DRAM bytes (read + write) per steady beam_step launch of the wide-beam
    search, from the committed ncu record ``profiles/beam_step_wide_beam.json``
    (written from the capture's raw counters), with the kernel name ncu printed
    and the source of the build it measured. None when there is no record or
    the record was taken on a different build of the kernel source."""
    p = os.path.join(ROOT, "profiles", "beam_step_wide_beam.json")
    if not os.path.exists(p):
        return None, None
    rec = json.load(open(p))
    src = os.path.join(ROOT, rec.get("source", ""))
    if not os.path.exists(src):
        return None, rec.get("kernel")
    import hashlib
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != rec.get("source_sha256"):
        return None, rec.get("kernel")
    v = rec.get("traffic_bytes_per_launch")
    return (None if v is None else float(v)), rec.get("kernel")


# ----------------------------------------------------------------- oracle timing
def _oracle_inputs(w, base, search, t):
    """Host copies of step t's inputs (bf16 bits, parent scores, nodes)."""
    import torch
    lg = base[t].view(torch.int16).cpu().numpy().view(np.uint16)
    ps, pn, B_in = search.parents(t)
    return lg, ps.cpu().numpy(), pn.cpu().numpy(), B_in


def _oracle_trie(w, cat=None):
    import oracle
    return oracle.OracleTrie(w.catalog() if cat is None else cat, w.codes_per_level)


# Oracle tries of the workloads the pool serves (filled before the fork).
_POOL_TRIES = {}


def _host_cpu():
    """(logical cores, CPU model) of this host."""
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def _start_oracle_pool(*cfgs):
    import multiprocessing as mp

    from sidgen.workloads import WORKLOADS
    for c in cfgs:
        if c not in _POOL_TRIES:
            _POOL_TRIES[c] = _oracle_trie(WORKLOADS[c])
    return mp.get_context("fork").Pool(os.cpu_count() or 1)


def _oracle_task(job):
    """One oracle beam step of one request (runs in a pool worker)."""
    import oracle
    cfg, t, lg, ps, pn, B_in, n, V = job
    oracle.beam_step(_POOL_TRIES[cfg], t, lg, ps, pn, 1, B_in, n, V)
    return int(np.isfinite(ps).sum()) * V


def _oracle_rates(cfg, jobs, budget_s, pool):
    """Logits scored per second by the oracle: on one thread (in this process),
    and on all cores (the pool, one request-step per task), each for about
    budget_s seconds over the jobs in turn."""
    import oracle
    trie = _POOL_TRIES[cfg]
    done, calls, t0 = 0, 0, time.perf_counter()
    while calls == 0 or time.perf_counter() - t0 < budget_s:
        _, t, lg, ps, pn, B_in, n, V = jobs[calls % len(jobs)]
        oracle.beam_step(trie, t, lg, ps, pn, 1, B_in, n, V)
        done += int(np.isfinite(ps).sum()) * V
        calls += 1
    single = done / (time.perf_counter() - t0)
    multi, mcalls = None, 0
    if pool is not None:
        per_call = (time.perf_counter() - t0) / calls
        ncores = os.cpu_count() or 1
        k = max(ncores, int(budget_s / per_call * ncores))
        batch = [jobs[i % len(jobs)] for i in range(k)]
        t1 = time.perf_counter()
        mdone = sum(pool.imap_unordered(_oracle_task, batch))
        multi = mdone / (time.perf_counter() - t1)
        mcalls = k
    return single, multi, calls, mcalls


def _request_jobs(cfg, w, base, search, steps):
    """Oracle inputs of whole requests (one request-step each) of the given steps."""
    import torch
    jobs = []
    for t in steps:
        lg = base[t].view(torch.int16).cpu().numpy().view(np.uint16) if base[t].dtype == torch.bfloat16 \
            else base[t].cpu().numpy()
        ps, pn, B_in = search.parents(t)
        ps, pn = ps.cpu().numpy(), pn.cpu().numpy()
        for r in range(w.R):
            sl = slice(r * B_in, (r + 1) * B_in)
            jobs.append((cfg, t, lg[sl], ps[sl], pn[sl], B_in, w.n, w.V))
    return jobs


def cpu_baseline(w, base, search, live_rows, budget_s=15.0, pool=None):
    """The oracle's beam step timed on a bounded sample of the same search:
    whole requests (512 rows x 4,096 bf16 logits) of steps 1-4 in turn, on one
    host thread and on all host cores (one process per core, one request-step
    per task)."""
    jobs = _request_jobs(CFG, w, base, search, range(1, w.depth))
    order = [jobs[(i % (w.depth - 1)) * w.R + (i // (w.depth - 1)) % w.R]
             for i in range(len(jobs))]          # steps in turn, request by request
    single, multi, calls, mcalls = _oracle_rates(CFG, order, budget_s, pool)
    cores, model = _host_cpu()
    line = {"value": single, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"oracle.beam_step on {calls} whole requests of steps 1-{w.depth - 1} "
                      f"(512 rows x {w.V} bf16 logits each, steps in turn), ~{budget_s:.0f} s, "
                      f"numpy float64, one thread",
            "host_cores": cores, "cpu_model": model}
    if multi is not None:
        line["all_cores"] = {"value": multi, "unit": UNIT, "cores": cores,
                             "sample": f"{mcalls} request-steps of the same sample over a pool "
                                       f"of {cores} processes"}
    return line


def measure_config(tcb, cfg, dev, pool, cpu_s):
    """One workload's whole search on the device (the search's own logits,
    resident in HBM, 3 rotating copies): per-step device times from events
    inside a CUDA graph replay, the search time from graph replays, and (for
    the HBM-bound flashrec-like workload) the steady steps' achieved HBM
    bandwidth; plus the oracle on a bounded sample of the same search, on one
    thread and on all cores."""
    import torch
    from sidgen import device as gdev
    from sidgen import host
    from sidgen.workloads import WORKLOADS

    w = WORKLOADS[cfg]
    cat = w.catalog()
    trie = tcb.sid_trie_build(cat, w.codes_per_level, w.layouts)
    search = tcb.BeamSearch(trie, w.R, w.n, w.V, depth=w.depth)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    esize = 2 if w.dtype == "bf16" else 4
    hashes = torch.from_numpy(host.request_roots(w.R).view(np.int64)).to(dev)
    base, live_rows = [], []
    for t in range(w.depth):
        lg = torch.empty((search.rows(t), w.V), dtype=tdt, device=dev)
        gdev.row_logits(w.logits_seed, hashes, w.V, w.sigma, lg)
        ps, pn, B_in = search.parents(t)
        live_rows.append(int(torch.isfinite(ps).sum().item()))
        search.step(t, lg)
        child = torch.empty((w.R * w.n,), dtype=torch.int64, device=dev)
        gdev.child_hash(hashes, w.R, B_in, search.bp_parent[t], search.bp_code[t], w.n, t + 1,
                        child)
        hashes = child
        base.append(lg)
    search.finalize()
    torch.cuda.synchronize()
    ref = search.sids.clone()
    sets = [base] + [[x.clone() for x in base] for _ in range(2)]
    graphs = [search.capture(x) for x in sets]
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(w.depth + 2)]
           for _ in sets]
    egraphs = [search.capture(sets[i], events=evs[i]) for i in range(len(sets))]
    for i in range(6):
        graphs[i % 3].replay()
    torch.cuda.synchronize()
    reps = 60
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(reps):
        graphs[i % 3].replay()
    e1.record()
    torch.cuda.synchronize()
    us_search = e0.elapsed_time(e1) * 1e3 / reps
    assert torch.equal(search.sids, ref)
    acc = np.zeros(w.depth + 1)
    for i in range(30):
        egraphs[i % 3].replay()
        torch.cuda.synchronize()
        acc += [evs[i % 3][t].elapsed_time(evs[i % 3][t + 1]) for t in range(w.depth + 1)]
    per = acc / 30 * 1e3
    assert tcb.sidbeam_get_device_status(search.workspace) == 0
    logits = sum(r * w.V for r in live_rows)
    out = {"workload": w.name, "us_per_search": us_search, "step_us": [float(x) for x in per[:-1]],
           "finalize_us": float(per[-1]), "logits_per_s": logits / (us_search * 1e-6),
           "timing": "CUDA graph replays of the whole search, 3 rotating logits copies; per-step "
                     "times from events inside the graph"}
    if cfg == 3:
        steady = list(range(1, w.depth))
        nbytes = [live_rows[t] * (w.V * esize + 8) + w.R * w.n * 16 for t in steady]
        dur = float(np.mean([per[t] for t in steady]))
        peak, kind = _peaks()
        gbs = float(np.mean(nbytes)) / (dur * 1e-6) / 1e9
        out["roofline"] = {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                           "frac": gbs / peak, "bytes_per_launch": float(np.mean(nbytes)),
                           "us_per_launch": dur, "peak_source": f"{kind} copy bandwidth"}
    if pool is not None:
        if cfg not in _POOL_TRIES:
            return out
        jobs = _request_jobs(cfg, w, base, search, range(1, w.depth))
        single, multi, calls, mcalls = _oracle_rates(cfg, jobs, cpu_s, pool)
        cores, model = _host_cpu()
        out["cpu_baseline"] = {"unit": UNIT, "kind": "oracle", "one_thread": single,
                               "all_cores": multi, "cores": cores, "cpu_model": model,
                               "sample": f"{calls} request-steps of steps 1-{w.depth - 1} on one "
                                         f"thread, {mcalls} on all cores"}
    return out


# ----------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle, as it stands, timed on the host cores on bounded samples of
    the same workload (steady step 2, slices of request 0's rows)."""
    import oracle
    from sidgen import host
    from sidgen.workloads import WORKLOADS

    w = WORKLOADS[CFG]
    # Inputs of step 2 come from the oracle's own search on host-generated logits
    # (the oracle needs no GPU): steps 0 and 1 are run once, untimed.
    trie = _oracle_trie(w)

    def fn(step, prefixes):
        return host.row_logits(w.logits_seed, host.prefix_hashes(prefixes), w.V, w.sigma, "bf16")

    R1 = 1
    scores = np.zeros(R1)
    nodes = np.zeros(R1, dtype=np.int64)
    prefixes = np.zeros((R1, 1, 0), dtype=np.int64)
    B_in = 1
    for t in range(2):
        z = fn(t, prefixes.reshape(R1 * B_in, t))
        out = oracle.beam_step(trie, t, z, scores, nodes, R1, B_in, w.n, w.V)
        newp = np.full((R1, w.n, t + 1), -1, dtype=np.int64)
        for k in range(w.n):
            p = out["parent"][0, k]
            if p >= 0:
                newp[0, k, :t] = prefixes[0, p]
                newp[0, k, t] = out["code"][0, k]
        prefixes, scores, nodes, B_in = newp, out["score"].reshape(-1), out["node"].reshape(-1), w.n
    t = 2
    z = fn(t, prefixes.reshape(B_in, t))
    # Calibrate the per-row cost, then size each step to fit the run in ~2 minutes.
    c0 = time.perf_counter()
    oracle.beam_step(trie, t, z[:8], scores[:8], nodes[:8], 1, 8, w.n, w.V)
    per_row = max((time.perf_counter() - c0) / 8, 1e-5)
    total_steps = max(1, args.steps + args.warmup)
    rows_per_step = int(max(1, min(B_in, 120.0 / total_steps / per_row)))
    pos = 0

    def one():
        nonlocal pos
        lo = pos % B_in
        hi = min(B_in, lo + rows_per_step)
        oracle.beam_step(trie, t, z[lo:hi], scores[lo:hi], nodes[lo:hi], 1, hi - lo, w.n, w.V)
        pos = hi % B_in
        return (hi - lo) * w.V

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += one()
    el = time.perf_counter() - t0
    value = done / el
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": _workload_config(w, {"parallelism": "single host thread"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"each step: oracle.beam_step on {rows_per_step} rows of "
                                   f"step 2 (x {w.V} bf16 logits), request 0 of the workload"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def record_traffic(csv_path, source):
    """Write profiles/beam_step_wide_beam.json from an ncu CSV of the wide-beam
    search's steady beam_step launches (steps 1-4), taken with
    --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum
    --csv: DRAM bytes read + written per launch (mean over the launches), the
    kernel name as ncu printed it, and the sha256 of the kernel source it
    measured (bench.py reports the traffic only while that source is unchanged)."""
    import csv
    import hashlib
    rows = [r for r in csv.reader(open(csv_path)) if r]
    hdr_i = next(i for i, r in enumerate(rows) if "Metric Name" in r)
    hdr = rows[hdr_i]
    col = {h: i for i, h in enumerate(hdr)}
    per = {}
    names = {}
    for r in rows[hdr_i + 1:]:
        if len(r) != len(hdr):
            continue
        lid = r[col["ID"]]
        m, v, u = r[col["Metric Name"]], r[col["Metric Value"]].replace(",", ""), r[col["Metric Unit"]]
        scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "nsecond": 1e-3,
                 "ns": 1e-3, "usecond": 1, "us": 1, "msecond": 1e3, "ms": 1e3}.get(u, 1)
        per.setdefault(lid, {})[m] = float(v) * scale
        names[lid] = r[col["Kernel Name"]]
    launches = [d for d in per.values() if "dram__bytes_read.sum" in d]
    traffic = [d["dram__bytes_read.sum"] + d.get("dram__bytes_write.sum", 0.0) for d in launches]
    rec = {"kernel": sorted(set(names.values())),
           "launches": len(launches),
           "traffic_bytes_per_launch": float(np.mean(traffic)),
           "traffic_bytes_each": traffic,
           "gpu_time_us_each": [d.get("gpu__time_duration.sum") for d in launches],
           "source": source,
           "source_sha256": hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest(),
           "how": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                  "--clock-control none -k regex:beam_step_kernel -s 1 -c 4 --csv on python "
                  "bench.py --steps 2 --warmup 1 --no-e2e --no-cpu-baseline --copies 1 --no-fused "
                  "--no-catalog --no-gumbel --no-widths --no-config-lines (the steady steps 1-4 "
                  "of the generating wide-beam search); cold-cache, serialised launches"}
    out = os.path.join(ROOT, "profiles", "beam_step_wide_beam.json")
    json.dump(rec, open(out, "w"), indent=1)
    print(out, rec["traffic_bytes_per_launch"])


def main():
    if len(sys.argv) >= 2 and sys.argv[1] == "--record-traffic":
        record_traffic(sys.argv[2], sys.argv[3])
        return
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fused", action="store_true",
                    help="skip the fused lm_head (tcgen05) lines")
    ap.add_argument("--clocks-dir", default=None,
                    help="directory for the raw clock samples (default: a temporary directory)")
    ap.add_argument("--no-widths", action="store_true",
                    help="skip the per-request widths line")
    ap.add_argument("--no-gumbel", action="store_true",
                    help="skip the Gumbel top-k search line")
    ap.add_argument("--no-catalog", action="store_true",
                    help="skip the catalog_score_topk throughput lines")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-config-lines", action="store_true",
                    help="skip the whole-search lines of the tiny, SPRINT-like and "
                         "flashrec-like workloads (configs 1-3)")
    ap.add_argument("--copies", type=int, default=COPIES,
                    help="rotating copies of the per-step logits (3 keeps reads out of L2)")
    args = ap.parse_args()
    world, rank, local = _dist()
    if args.gpus != world:
        # One process per GPU: N GPUs means N ranks launched by torch.distributed.run.
        print(json.dumps({"error": f"--gpus {args.gpus} but WORLD_SIZE is {world}: launch "
                                   f"{args.gpus} ranks with torch.distributed.run"}), flush=True)
        sys.exit(2)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        line = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
