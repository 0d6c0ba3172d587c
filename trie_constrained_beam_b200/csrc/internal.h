// Host-side internals of libsidbeam: the trie object and error reporting.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <string>

#include "sidbeam.h"

namespace sidbeam {

// One expansion structure: level-t nodes (parents) -> level-(t+1) codes.
struct StepTrie {
  int layout = 0;               // SIDBEAM_LAYOUT_DENSE or SIDBEAM_LAYOUT_CSR
  int V = 0;                    // codes at level t+1
  int64_t n_parent = 0;         // P_t
  int64_t n_child = 0;          // P_{t+1}
  uint32_t* off = nullptr;      // [P_t + 1]: children of p are ids off[p] .. off[p+1]-1
  uint32_t* mask = nullptr;     // dense: [P_t][mask_stride] bit c of row p = child code c
  int mask_words = 0;           // ceil(V / 32)
  int mask_stride = 0;          // mask_words rounded up to a multiple of 4 (16-byte rows)
  uint16_t* codes = nullptr;    // CSR: [P_{t+1} + 8]: code of child id q (padded for 16-B loads)
  size_t bytes = 0;
};

}  // namespace sidbeam

struct sidbeam_trie {
  int depth = 0;
  int device = 0;
  int V[SIDBEAM_MAX_DEPTH] = {};
  int64_t n_nodes[SIDBEAM_MAX_DEPTH + 1] = {};
  sidbeam::StepTrie steps[SIDBEAM_MAX_DEPTH];
  int64_t n_leaves = 0;
  int32_t* leaf_rows = nullptr;    // [n_leaves]
  uint16_t* leaf_codes = nullptr;  // [depth][leaf_codes_stride], SoA (stride: n_leaves rounded up to 8, plus 8)
  int64_t leaf_codes_stride = 0;   // n_leaves + 8
  size_t leaf_bytes = 0;
};

namespace sidbeam {

int set_error(int status, const char* fmt, ...);
int cuda_error(cudaError_t e, const char* what);
int device_sm_count();

// The deterministic step behind every host check of beam_step_ex; with
// clear_bytes > 0 the first clear_bytes of the workspace are zeroed on the
// stream right before the launch (nothing is enqueued when a check fails).
int beam_step_checked(const sidbeam_trie* trie, int step, const void* logits, sidbeam_dtype dtype,
                      int64_t ld, const float* parent_scores, const int32_t* parent_nodes, int R,
                      int B_in, int n_out, int V, float* out_scores, int32_t* out_parent,
                      int32_t* out_code, int32_t* out_node, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream, unsigned flags,
                      const int32_t* out_width, size_t clear_bytes);

// Device status word bits (first 4 bytes of a workspace).
constexpr uint32_t kStatusBadNode = 1u;
constexpr uint32_t kStatusTimeout = 2u;
// Byte offset, inside the workspace's first 256-byte block (after the status
// word), of the counter of rows beam_step did not read (row skipping).
constexpr size_t kSkippedRowsOffset = 8;
// ... and of max_j ||e_j|| for catalog_score_topk_sim (written each call).
constexpr size_t kEmbNormOffset = 16;

}  // namespace sidbeam
