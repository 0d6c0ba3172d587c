// Shared-memory plan of the beam_step kernel (host only; the kernel and the
// CPU tests both include it).
#pragma once

#include <algorithm>

#include "launch.h"

namespace sidbeam {

// Rows of a CTA whose parent data fits the shared table: up to this many, the
// warps take rows from a shared counter instead of a fixed share each.
constexpr int kMetaRows = 256;
// Score-histogram bins (the rank merge's scratch is two of them per CTA).
constexpr int kPlanHistBins = 1024;

inline int plan_round_up(int x, int m) { return (x + m - 1) / m * m; }

// Shared-memory plan: [control | barriers | radix scratch | warp histograms
// (>= 2 x 1024 words: the rank merge's scratch) | dense prefix counts | mask
// copies | W x S stages | W top-n buffers], the parent table after the
// barriers. Register rows try 12 warps with one stage first; rows worked on in
// place want two stages per warp (one stage is the last resort). Small rows get
// more stages (up to kMaxStages). ctl_bytes: the control block, rounded to 128.
inline bool choose_step_config(int V, int esize, int extra_bytes, int prefix_words, int n,
                               bool reg, int ctl_bytes, StepConfig* cfg) {
  StepConfig c{};
  c.logits_copy_bytes = plan_round_up(V * esize, 16);
  c.extra_bytes = extra_bytes;
  c.stage_bytes = plan_round_up(c.logits_copy_bytes + extra_bytes, 128);
  c.prefix_words = prefix_words;
  c.reg = reg ? 1 : 0;
  int npow2 = 1;
  while (npow2 < n) npow2 <<= 1;
  // Register rows: 12 warps with one stage each (more warps hide more
  // latency; the stage is refilled as soon as the row is in registers).
  // Rows worked on in place: at least two stages per warp.
  struct Plan { int W, min_s; };
  static const Plan kRegPlans[] = {{12, 1}, {8, 2}, {8, 1}, {6, 1}, {4, 1}, {2, 1}, {1, 1}};
  static const Plan kSmemPlans[] = {{8, 2}, {6, 2}, {4, 2}, {8, 1}, {6, 1}, {4, 1}, {2, 1}, {1, 1}};
  const Plan* plans = reg ? kRegPlans : kSmemPlans;
  const int nplans = reg ? 7 : 8;
  for (int pi = 0; pi < nplans; ++pi) {
    {
      const int W = plans[pi].W, min_s = plans[pi].min_s;
      if (W > (reg ? kMaxStepWarpsReg : kMaxStepWarps)) continue;
      const int cw = std::max(plan_round_up(n, 32) + 32, plan_round_up((npow2 + W - 1) / W, 32));
      int o = 0;
      c.off_ctl = o;
      o += ctl_bytes;
      c.off_bars = o;
      o += plan_round_up(W * kMaxStages * 8, 128);
      c.off_meta = o;
      o += kMetaRows * 16;
      c.off_chist = o;
      o += 1024;
      c.off_whist = o;
      o += std::max(W * 1024, 2 * kPlanHistBins * 4);
      c.off_wprefix = o;
      o += W * c.prefix_words * 4;
      c.off_wmask = o;
      o += W * c.prefix_words * 4;
      o = plan_round_up(o, 128);
      const int warp_bytes = W * cw * 12 + 256;
      const int avail = kSmemBudget - o - warp_bytes;
      const int S = std::min(kMaxStages, avail / (W * c.stage_bytes));
      if (S < min_s) continue;
      c.W = W;
      c.S = S;
      c.Cw = cw;
      c.off_stage = o;
      o += W * S * c.stage_bytes;
      c.off_wkeys = plan_round_up(o, 128);
      o = c.off_wkeys + W * cw * 8;
      c.off_wvals = plan_round_up(o, 16);
      o = c.off_wvals + W * cw * 4;
      c.smem_bytes = plan_round_up(o, 128);
      if (c.smem_bytes > kSmemBudget) continue;
      *cfg = c;
      return true;
    }
  }
  return false;
}

}  // namespace sidbeam
