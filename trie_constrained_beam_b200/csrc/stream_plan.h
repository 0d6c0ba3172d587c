// Launch plan of the streaming step kernel (beam_stream.cu): warps, teams,
// per-warp stages and the shared-memory carve-up. Host code only; the kernel
// and the CPU tests both include it.
#pragma once

#include <algorithm>
#include <cstdint>

namespace sidbeam {

constexpr int kStreamMaxWarps = 12;   // warps per CTA
constexpr int kMaxStreamDepth = 4;    // rows a warp keeps in flight (stages per warp)
constexpr int kListStageCodes = 256;  // child codes staged behind a list row's chunk
constexpr int kRowChunkBytes = 8192;  // logits one warp holds in registers
constexpr int kTeamSlotBytes = 256;   // per team and parity: partial (max, sum) of each warp
constexpr int kMaxTeamWarps = 16;
constexpr int kStreamHistBins = 1024;

inline int sp_round_up(int x, int m) { return (x + m - 1) / m * m; }

struct StreamPlan {
  int W;             // warps (a multiple of K)
  int K;             // warps that share one row (a team): ceil(V * esize / 8 KB)
  int D;             // rows in flight per warp (stages per warp)
  int CW;            // codes per warp chunk of a row (a multiple of 16 / esize)
  int Cw;            // candidate slots per warp (>= n + 32)
  int chunk_bytes;   // logits bytes of one chunk: CW * esize (a multiple of 16)
  int extra_bytes;   // trie data staged behind a chunk
  int stage_bytes;
  int mcopy_bytes;   // per-warp copy of the chunk's child-bitmask bytes (0: no bitmask rows)
  int off_ctl, off_team, off_meta, off_chist, off_whist, off_wprefix, off_wmask, off_stage,
      off_wkeys, off_wvals;
  int smem_bytes;
};

// has_mask: some rows carry a child bitmask of mask_stride words (a dense
// level, or CSR nodes with many children); has_list: some rows carry CSR child
// codes. ctl_bytes: the selection control block, rounded to 128.
inline bool choose_stream_plan(int V, int esize, bool has_mask, int mask_stride, bool has_list,
                               int n, int ctl_bytes, int smem_budget, StreamPlan* out) {
  if (V < 1 || (esize != 2 && esize != 4) || n < 1) return false;
  const int per_vec = 16 / esize;
  const int kmin = (V * esize + kRowChunkBytes - 1) / kRowChunkBytes;
  if (kmin > kMaxTeamWarps) return false;
  int npow2 = 1;
  while (npow2 < n) npow2 <<= 1;
  static const int kWarpChoices[] = {12, 11, 10, 9, 8, 7, 6, 5, 4, 3, 2, 1};
  for (int D = kMaxStreamDepth; D >= 1; --D) {
    for (int W : kWarpChoices) {
      if (W > kStreamMaxWarps || W < kmin) continue;
      // Team size: fixed by the row size alone (so that a row's statistics
      // are summed in the same order whatever the batch); a CTA with fewer
      // rows than teams gives each row to several teams instead.
      if (W % kmin) continue;
      const int K = kmin;
      if (K > kMaxTeamWarps) continue;
      StreamPlan p{};
      p.W = W;
      p.K = K;
      p.D = D;
      p.CW = sp_round_up((V + K - 1) / K, per_vec);
      if (p.CW * esize > kRowChunkBytes) continue;
      p.chunk_bytes = p.CW * esize;
      p.mcopy_bytes = has_mask ? std::min(sp_round_up((p.CW + 7) / 8 + 16, 16), mask_stride * 4) : 0;
      int extra = p.mcopy_bytes;
      if (has_list) extra = std::max(extra, sp_round_up((kListStageCodes + 8) * 2, 16));
      p.extra_bytes = extra;
      p.stage_bytes = sp_round_up(p.chunk_bytes + extra, 128);
      p.Cw = std::max(sp_round_up(n, 32) + 32, sp_round_up((npow2 + W - 1) / W, 32));
      int o = 0;
      p.off_ctl = o;
      o += ctl_bytes;
      p.off_team = o;
      o += (W / K) * 2 * kTeamSlotBytes;
      p.off_meta = o;
      o += W * kMaxStreamDepth * 16;
      p.off_chist = o;
      o += 256 * 4;
      p.off_whist = o;
      o += std::max(W * 256 * 4, 2 * kStreamHistBins * 4);
      p.off_wprefix = o;
      o += W * p.mcopy_bytes;
      p.off_wmask = o;
      o += W * p.mcopy_bytes;
      o = sp_round_up(o, 128);
      p.off_stage = o;
      o += W * D * p.stage_bytes;
      p.off_wkeys = sp_round_up(o, 128);
      o = p.off_wkeys + W * p.Cw * 8;
      p.off_wvals = sp_round_up(o, 16);
      o = p.off_wvals + W * p.Cw * 4;
      p.smem_bytes = sp_round_up(o, 128);
      if (p.smem_bytes > smem_budget) continue;
      // More than one row in flight only with the full complement of warps,
      // and no more than about 16 KB of logits in flight per warp.
      if (D > 1 && (W < kStreamMaxWarps || D * p.chunk_bytes > 16384)) continue;
      *out = p;
      return true;
    }
  }
  return false;
}

}  // namespace sidbeam
