// Launch geometry shared by the host launchers and the kernels: the row
// partition over CTAs, the workspace carve-up and the shared-memory plan.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cstddef>

namespace sidbeam {

constexpr int kMaxStepWarpsReg = 12;   // register-row kernel: up to 12 warps (<= 168 registers)
constexpr int kMaxStepWarps = 12;      // shared-memory-row kernel
constexpr int kSmemBudget = 232448;    // 227 KiB of dynamic shared memory per CTA
constexpr int kMaxStages = 8;          // ring stages per warp

// Rows [0, total_rows) in request-major order (row = r * B_in + b) are split
// over CTAs. When there are at least as many CTAs as requests, each request
// gets its own group of G CTAs (no CTA touches two requests, so no request is
// merged while other rows of the same CTA still wait); otherwise the rows are
// cut into equal contiguous chunks that may span request boundaries.
struct Partition {
  int64_t total_rows;
  int64_t rows_per_cta;
  int grid;
  int B_in;     // rows per request
  int maxG;     // upper bound on contributors of any request
  int grouped;  // 1: request r owns CTAs r*G .. r*G+G-1 (its slots interleaved)
  int G;

  __host__ __device__ __forceinline__ void range(int cta, int64_t& lo, int64_t& hi) const {
    if (grouped) {
      const int r = cta / G, j = cta - r * G;
      const int64_t base = static_cast<int64_t>(r) * B_in;
      lo = base + static_cast<int64_t>(j) * rows_per_cta;
      hi = lo + rows_per_cta;
      if (hi > base + B_in) hi = base + B_in;
    } else {
      lo = static_cast<int64_t>(cta) * rows_per_cta;
      hi = lo + rows_per_cta;
      if (hi > total_rows) hi = total_rows;
    }
  }
  // The rows of a CTA as a strided sequence first + stride * i, i < count. A
  // request's group of CTAs interleaves its parent slots (CTA j takes slots
  // j, j+G, j+2G, ...), so that every CTA gets its share of the best parents
  // (the beam is ranked best-first) and the candidate work stays balanced.
  // `part` of `parts` (warps dealt rows round-robin) narrows it to one warp's
  // rows; parts = 1 gives the whole CTA's sequence.
  __host__ __device__ __forceinline__ void rows(int cta, int part, int parts, int64_t& first,
                                                int64_t& stride, int& count) const {
    int64_t f, st, n;
    if (grouped) {
      const int r = cta / G, j = cta - r * G;
      f = static_cast<int64_t>(r) * B_in + j;
      st = G;
      n = (B_in - j + G - 1) / G;
    } else {
      int64_t lo, hi;
      range(cta, lo, hi);
      f = lo;
      st = 1;
      n = hi - lo;
    }
    first = f + st * part;
    stride = st * parts;
    count = part < n ? static_cast<int>((n - part + parts - 1) / parts) : 0;
  }
  __host__ __device__ __forceinline__ int first_cta(int r) const {
    if (grouped) return r * G;
    return static_cast<int>(static_cast<int64_t>(r) * B_in / rows_per_cta);
  }
  __host__ __device__ __forceinline__ int last_cta(int r) const {
    if (grouped) return r * G + G - 1;
    return static_cast<int>((static_cast<int64_t>(r + 1) * B_in - 1) / rows_per_cta);
  }
  __host__ __device__ __forceinline__ int contributors(int r) const {
    return last_cta(r) - first_cta(r) + 1;
  }
};

inline Partition make_partition(int R, int64_t B_in, int ctas) {
  Partition p{};
  p.total_rows = static_cast<int64_t>(R) * B_in;
  p.B_in = static_cast<int>(B_in);
  if (ctas < 1) ctas = 1;
  if (R <= ctas) {
    int64_t G = ctas / R;
    if (G > B_in) G = B_in;
    if (G < 1) G = 1;
    p.rows_per_cta = (B_in + G - 1) / G;
    G = (B_in + p.rows_per_cta - 1) / p.rows_per_cta;
    p.grouped = 1;
    p.G = static_cast<int>(G);
    p.grid = R * p.G;
    p.maxG = p.G;
    return p;
  }
  int64_t g = ctas;
  if (g > p.total_rows) g = p.total_rows;
  if (g < 1) g = 1;
  p.rows_per_cta = (p.total_rows + g - 1) / g;
  if (p.rows_per_cta < 1) p.rows_per_cta = 1;
  p.grid = static_cast<int>((p.total_rows + p.rows_per_cta - 1) / p.rows_per_cta);
  int64_t mg = (B_in + p.rows_per_cta - 1) / p.rows_per_cta + 1;
  if (mg > p.grid) mg = p.grid;
  p.maxG = static_cast<int>(mg);
  p.grouped = 0;
  p.G = 0;
  return p;
}

// Workspace: [status | tickets[R] | request_thr[R] | score histograms[R][1024] |
//             part_count[R][maxG] | part_keys[R][maxG][2n] | part_vals[R][maxG][2n]],
// 256-byte aligned parts. Everything before part_keys must start at zero.
struct WorkspaceLayout {
  size_t status, tickets, request_thr, ghist, part_count, part_keys, part_vals, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Entries a CTA may leave in its partial list of a request: 2n, so that the
// survivors of a segment (the n best plus the slack of the histogram bound)
// are written without an exact cut in the common case.
__host__ __device__ __forceinline__ int partial_cap(int n) { return 2 * n; }

inline WorkspaceLayout workspace_layout(int R, int maxG, int n) {
  const int pcap = partial_cap(n);
  WorkspaceLayout w{};
  size_t o = 0;
  w.status = o;
  o = align256(o + 4);
  w.tickets = o;
  o = align256(o + static_cast<size_t>(R) * 4);
  w.request_thr = o;
  o = align256(o + static_cast<size_t>(R) * 8);
  w.ghist = o;
  o = align256(o + static_cast<size_t>(R) * 1024 * 4);
  w.part_count = o;
  o = align256(o + static_cast<size_t>(R) * maxG * 4);
  w.part_keys = o;
  o = align256(o + static_cast<size_t>(R) * maxG * pcap * 8);
  w.part_vals = o;
  o = align256(o + static_cast<size_t>(R) * maxG * pcap * 4);
  w.total = o;
  return w;
}

// Shared-memory plan of one beam_step CTA: every warp owns a ring of S
// stages (logits row + trie extra) that it fills itself with bulk copies.
struct StepConfig {
  int W;                  // warps
  int S;                  // ring stages per warp
  int Cw;                 // candidate slots per warp (>= n + 32)
  int stage_bytes;
  int logits_copy_bytes;  // V * sizeof(dtype) rounded up to 16
  int extra_bytes;        // per stage after the row: dense mask row or staged CSR codes
  int prefix_words;       // dense levels: mask words per warp (prefix counts, mask copy)
  int reg;                // rows held in registers (<= 8 KB per row)
  int off_ctl, off_bars, off_meta, off_chist, off_whist, off_wprefix, off_wmask, off_stage,
      off_wkeys, off_wvals;
  int smem_bytes;
};

}  // namespace sidbeam
