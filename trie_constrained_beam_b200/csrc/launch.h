// Launch geometry shared by the host launchers and the kernels: the row
// partition over CTAs, the workspace carve-up and the shared-memory plan.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cstddef>

namespace sidbeam {

constexpr int kMaxStepThreads = 288;         // 1 producer + up to 8 consumer warps
constexpr int kSmemBudget = 232448;          // 227 KiB of dynamic shared memory per CTA
constexpr int kMaxStages = 32;

// Rows [0, total_rows) in request-major order are cut into `grid` equal
// chunks of rows_per_cta; the CTAs that touch request r are
// first_cta(r) .. last_cta(r).
struct Partition {
  int64_t total_rows;
  int64_t rows_per_cta;
  int grid;
  int B_in;   // rows per request
  int maxG;   // upper bound on contributors of any request

  __host__ __device__ __forceinline__ int first_cta(int r) const {
    return static_cast<int>(static_cast<int64_t>(r) * B_in / rows_per_cta);
  }
  __host__ __device__ __forceinline__ int last_cta(int r) const {
    return static_cast<int>((static_cast<int64_t>(r + 1) * B_in - 1) / rows_per_cta);
  }
  __host__ __device__ __forceinline__ int contributors(int r) const {
    return last_cta(r) - first_cta(r) + 1;
  }
};

inline Partition make_partition(int R, int64_t B_in, int ctas) {
  Partition p{};
  p.total_rows = static_cast<int64_t>(R) * B_in;
  int64_t g = ctas < 1 ? 1 : ctas;
  if (g > p.total_rows) g = p.total_rows;
  if (g < 1) g = 1;
  p.rows_per_cta = (p.total_rows + g - 1) / g;
  if (p.rows_per_cta < 1) p.rows_per_cta = 1;
  p.grid = static_cast<int>((p.total_rows + p.rows_per_cta - 1) / p.rows_per_cta);
  p.B_in = static_cast<int>(B_in);
  int64_t mg = (B_in + p.rows_per_cta - 1) / p.rows_per_cta + 1;
  if (mg > p.grid) mg = p.grid;
  p.maxG = static_cast<int>(mg);
  return p;
}

// Workspace: [status | tickets[R] | request_thr[R] | part_count[R][maxG] |
//             part_keys[R][maxG][n] | part_vals[R][maxG][n]], 256-byte aligned parts.
struct WorkspaceLayout {
  size_t status, tickets, request_thr, part_count, part_keys, part_vals, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline WorkspaceLayout workspace_layout(int R, int maxG, int n) {
  WorkspaceLayout w{};
  size_t o = 0;
  w.status = o;
  o = align256(o + 4);
  w.tickets = o;
  o = align256(o + static_cast<size_t>(R) * 4);
  w.request_thr = o;
  o = align256(o + static_cast<size_t>(R) * 8);
  w.part_count = o;
  o = align256(o + static_cast<size_t>(R) * maxG * 4);
  w.part_keys = o;
  o = align256(o + static_cast<size_t>(R) * maxG * n * 8);
  w.part_vals = o;
  o = align256(o + static_cast<size_t>(R) * maxG * n * 4);
  w.total = o;
  return w;
}

// Shared-memory plan of one beam_step CTA.
struct StepConfig {
  int W;                  // consumer warps
  int S;                  // ring stages
  int Cw;                 // candidate slots per consumer warp (>= n + 32)
  int stage_bytes;
  int logits_copy_bytes;  // V * sizeof(dtype) rounded up to 16
  int mask_copy_bytes;    // dense levels: one bitmask row
  int off_bars, off_ctl, off_meta, off_chist, off_whist, off_stage, off_wkeys, off_wvals;
  int smem_bytes;
};

bool choose_step_config(int V, int esize, int mask_stride_words, int n, StepConfig* cfg);

}  // namespace sidbeam
