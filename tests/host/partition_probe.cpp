// Test harness (host only): exposes the row partition of the launch geometry
// header to the CPU tests. Built by tests/test_partition_host.py with g++.
#include <stdint.h>

#include "launch.h"

// For every CTA c, writes each row of its sequence (rows(c, 0, 1)) into rows[]
// (CTA-major, `cap` slots per CTA, count in counts[c]); for every warp w < W,
// the warp's share (rows(c, w, W)) is checked to be the CTA entries w, w + W, ...
// Returns the grid size, or -1 when a warp share disagrees or a CTA has more
// than `cap` rows. maxG and the per-request contributor counts are returned too.
extern "C" int partition_probe(int R, int64_t B_in, int ctas, int W, int cap, int64_t* rows,
                               int* counts, int* maxG, int* first_cta, int* last_cta,
                               int* contributors) {
  const sidbeam::Partition p = sidbeam::make_partition(R, B_in, ctas);
  *maxG = p.maxG;
  for (int r = 0; r < R; ++r) {
    first_cta[r] = p.first_cta(r);
    last_cta[r] = p.last_cta(r);
    contributors[r] = p.contributors(r);
  }
  for (int c = 0; c < p.grid; ++c) {
    int64_t first, stride;
    int count;
    p.rows(c, 0, 1, first, stride, count);
    if (count > cap) return -1;
    counts[c] = count;
    for (int i = 0; i < count; ++i) rows[static_cast<int64_t>(c) * cap + i] = first + stride * i;
    for (int w = 0; w < W; ++w) {
      int64_t f2, s2;
      int n2;
      p.rows(c, w, W, f2, s2, n2);
      int expect = 0;
      for (int i = w; i < count; i += W) ++expect;
      if (n2 != expect) return -1;
      for (int k = 0; k < n2; ++k)
        if (f2 + s2 * k != first + stride * (w + static_cast<int64_t>(W) * k)) return -1;
    }
  }
  return p.grid;
}

// The workspace carve-up: offsets of status, tickets, request_thr, ghist,
// part_count, part_keys, part_vals and the total, in that order.
extern "C" void workspace_probe(int R, int maxG, int n, int64_t* out) {
  const sidbeam::WorkspaceLayout w = sidbeam::workspace_layout(R, maxG, n);
  const size_t v[8] = {w.status, w.tickets, w.request_thr, w.ghist, w.part_count,
                       w.part_keys, w.part_vals, w.total};
  for (int i = 0; i < 8; ++i) out[i] = static_cast<int64_t>(v[i]);
}

#include "step_plan.h"

// The beam_step shared-memory plan for one shape: returns whether one fits and
// writes W, S, Cw, stage_bytes, logits_copy_bytes, the ten region offsets
// (ctl, bars, meta, chist, whist, wprefix, wmask, stage, wkeys, wvals) and
// smem_bytes, in that order (17 ints).
extern "C" int plan_probe(int V, int esize, int extra, int prefix_words, int n, int reg,
                          int ctl_bytes, int* out) {
  sidbeam::StepConfig c{};
  if (!sidbeam::choose_step_config(V, esize, extra, prefix_words, n, reg != 0, ctl_bytes, &c))
    return 0;
  const int v[17] = {c.W, c.S, c.Cw, c.stage_bytes, c.logits_copy_bytes, c.off_ctl, c.off_bars,
                     c.off_meta, c.off_chist, c.off_whist, c.off_wprefix, c.off_wmask,
                     c.off_stage, c.off_wkeys, c.off_wvals, c.smem_bytes, c.reg};
  for (int i = 0; i < 17; ++i) out[i] = v[i];
  return 1;
}
