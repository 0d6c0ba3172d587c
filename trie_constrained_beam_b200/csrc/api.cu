// C ABI entry points of libsidbeam: argument checks, workspace sizes,
// beam_finalize, device status and error strings. Argument errors are found
// here, on the host, before anything is launched.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include <cstdio>
#include <cstring>

#include "internal.h"
#include "launch.h"

namespace sidbeam {

static thread_local char g_last_error[512] = "";

int set_error(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

int cuda_error(cudaError_t e, const char* what) {
  return set_error(SIDBEAM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int device_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 1;
  return sms > 0 ? sms : 1;
}

int launch_beam_step(const sidbeam_trie* trie, int step, const void* logits, int dtype, int64_t ld,
                     const float* parent_scores, const int32_t* parent_nodes, int R, int B_in,
                     int n_out, int V, float* out_scores, int32_t* out_parent, int32_t* out_code,
                     int32_t* out_node, void* workspace, size_t workspace_bytes,
                     cudaStream_t stream, unsigned flags, float gumbel_T, uint64_t gumbel_seed,
                     float* row_lse, const int32_t* out_width, size_t clear_bytes);

namespace {

__global__ void finalize_kernel(int depth, int R, int n, const int32_t* __restrict__ bp_parent,
                                const int32_t* __restrict__ bp_code,
                                const int32_t* __restrict__ last_node,
                                int32_t* __restrict__ out_sids, int32_t* __restrict__ out_leaf) {
  const int64_t total = static_cast<int64_t>(R) * n;
  const int64_t plane = total;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / n;
    int32_t* sid = out_sids + i * depth;
    const bool live = bp_code[(depth - 1) * plane + i] >= 0;
    int slot = static_cast<int>(i - r * n);
    bool ok = live;
    for (int t = depth - 1; t >= 0; --t) {
      if (!ok || slot < 0 || slot >= n) {
        ok = false;
        sid[t] = -1;
        continue;
      }
      const int64_t at = t * plane + r * n + slot;
      sid[t] = bp_code[at];
      slot = bp_parent[at];
      if (t > 0 && slot < 0) ok = false;
    }
    if (!ok)
      for (int t = 0; t < depth; ++t) sid[t] = -1;
    out_leaf[i] = ok ? last_node[i] : -1;
  }
}

}  // namespace
}  // namespace sidbeam

using namespace sidbeam;

extern "C" const char* sidbeam_last_error(void) { return g_last_error; }

extern "C" const char* sidbeam_version(void) { return "0.1.0"; }

extern "C" size_t beam_step_workspace_size(int R, int B_in, int n_out, int V) {
  if (R < 1 || B_in < 1 || n_out < 1 || n_out > SIDBEAM_MAX_BEAM || V < 1 || V > SIDBEAM_MAX_V)
    return 0;
  const Partition p = make_partition(R, B_in, std::min(device_sm_count(), 640));
  return workspace_layout(R, p.maxG, n_out).total;
}

extern "C" int beam_step(const sidbeam_trie* trie, int step, const void* logits,
                         sidbeam_dtype dtype, int64_t ld, const float* parent_scores,
                         const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                         float* out_scores, int32_t* out_parent, int32_t* out_code,
                         int32_t* out_node, void* workspace, size_t workspace_bytes,
                         void* stream) {
  return beam_step_ex(trie, step, logits, dtype, ld, parent_scores, parent_nodes, R, B_in, n_out,
                      V, out_scores, out_parent, out_code, out_node, workspace, workspace_bytes,
                      stream, 0u, nullptr);
}

namespace sidbeam {

// The host checks every step entry point shares (shapes, pointers, alignment).
int check_step_args(const sidbeam_trie* trie, int step, const void* logits,
                           sidbeam_dtype dtype, int64_t ld, const float* parent_scores,
                           const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                           const float* out_scores, const int32_t* out_parent,
                           const int32_t* out_code, const int32_t* out_node,
                           const void* workspace) {
  if (!logits || !parent_scores || !out_scores || !out_parent || !out_code || !out_node)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: NULL pointer argument");
  if (trie && !parent_nodes)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: parent_nodes is NULL with a trie");
  if (dtype != SIDBEAM_F32 && dtype != SIDBEAM_BF16)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: unknown dtype %d", static_cast<int>(dtype));
  if (R < 1 || B_in < 1)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: R=%d B_in=%d must be >= 1", R, B_in);
  if (n_out < 1 || n_out > SIDBEAM_MAX_BEAM)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: n_out=%d outside [1, %d]", n_out,
                     SIDBEAM_MAX_BEAM);
  const int esize = dtype == SIDBEAM_BF16 ? 2 : 4;
  if (V < 1 || V > SIDBEAM_MAX_V || static_cast<int64_t>(V) * esize > 65536)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: V=%d unsupported for this dtype", V);
  if (static_cast<uint64_t>(B_in) * static_cast<uint64_t>(V) > 0xFFFFFFFFull)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: B_in*V = %lld must be < 2^32",
                     static_cast<long long>(B_in) * V);
  if (static_cast<int64_t>(R) * B_in > 0x7FFFFFFFll || static_cast<int64_t>(R) * n_out > 0x7FFFFFFFll)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: too many rows");
  if (ld < V) return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: ld=%lld < V=%d",
                               static_cast<long long>(ld), V);
  if ((reinterpret_cast<uintptr_t>(logits) & 15u) != 0 || (ld * esize) % 16 != 0)
    return set_error(SIDBEAM_ERR_ALIGNMENT,
                     "beam_step: logits must be 16-byte aligned with ld*sizeof(dtype) %% 16 == 0");
  if (trie) {
    if (step < 0 || step >= trie->depth)
      return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: step %d outside [0, %d)", step,
                       trie->depth);
    if (trie->V[step] != V)
      return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: V=%d but the trie has V=%d at level %d",
                       V, trie->V[step], step + 1);
  }
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return set_error(SIDBEAM_ERR_WORKSPACE, "beam_step: workspace must be 256-byte aligned");
  return SIDBEAM_OK;
}

// The deterministic step after every host check; clear_bytes > 0 zeroes the
// head of the workspace on the stream right before the launch (after every
// check, so that a rejected call enqueues nothing).
int beam_step_checked(const sidbeam_trie* trie, int step, const void* logits, sidbeam_dtype dtype,
                      int64_t ld, const float* parent_scores, const int32_t* parent_nodes, int R,
                      int B_in, int n_out, int V, float* out_scores, int32_t* out_parent,
                      int32_t* out_code, int32_t* out_node, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream, unsigned flags,
                      const int32_t* out_width, size_t clear_bytes) {
  if (flags & ~static_cast<unsigned>(SIDBEAM_STEP_SKIP_ROWS))
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: unknown flags 0x%x", flags);
  const int rc = check_step_args(trie, step, logits, dtype, ld, parent_scores, parent_nodes, R,
                                 B_in, n_out, V, out_scores, out_parent, out_code, out_node,
                                 workspace);
  if (rc != SIDBEAM_OK) return rc;
  return launch_beam_step(trie, step, logits, dtype, ld, parent_scores, parent_nodes, R, B_in,
                          n_out, V, out_scores, out_parent, out_code, out_node, workspace,
                          workspace_bytes, stream, flags, 0.f, 0ull, nullptr, out_width,
                          clear_bytes);
}

}  // namespace sidbeam

extern "C" int beam_step_ex(const sidbeam_trie* trie, int step, const void* logits,
                            sidbeam_dtype dtype, int64_t ld, const float* parent_scores,
                            const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                            float* out_scores, int32_t* out_parent, int32_t* out_code,
                            int32_t* out_node, void* workspace, size_t workspace_bytes,
                            void* stream, unsigned flags, const int32_t* out_width) {
  return sidbeam::beam_step_checked(trie, step, logits, dtype, ld, parent_scores, parent_nodes,
                                    R, B_in, n_out, V, out_scores, out_parent, out_code,
                                    out_node, workspace, workspace_bytes,
                                    static_cast<cudaStream_t>(stream), flags, out_width, 0);
}

// Gumbel steps keep every row's lse after the beam_step workspace.
static size_t gumbel_lse_offset(int R, int B_in, int n_out, int V) {
  return (beam_step_workspace_size(R, B_in, n_out, V) + 255) & ~static_cast<size_t>(255);
}

extern "C" size_t beam_step_gumbel_workspace_size(int R, int B_in, int n_out, int V) {
  const size_t base = beam_step_workspace_size(R, B_in, n_out, V);
  if (base == 0) return 0;
  return gumbel_lse_offset(R, B_in, n_out, V) + static_cast<size_t>(R) * B_in * sizeof(float);
}

extern "C" int beam_step_gumbel(const sidbeam_trie* trie, int step, const void* logits,
                                sidbeam_dtype dtype, int64_t ld, const float* parent_scores,
                                const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                                float temperature, uint64_t seed, float* out_scores,
                                int32_t* out_parent, int32_t* out_code, int32_t* out_node,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!(temperature >= 0.f) || temperature > 1e30f)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step_gumbel: temperature must be finite, >= 0");
  if (temperature == 0.f)  // the deterministic step
    return beam_step_ex(trie, step, logits, dtype, ld, parent_scores, parent_nodes, R, B_in,
                        n_out, V, out_scores, out_parent, out_code, out_node, workspace,
                        workspace_bytes, stream, 0u, nullptr);
  const size_t need = beam_step_gumbel_workspace_size(R, B_in, n_out, V);
  if (need == 0 || workspace_bytes < need)
    return set_error(SIDBEAM_ERR_WORKSPACE, "beam_step_gumbel: workspace of %zu bytes, need %zu",
                     workspace_bytes, need);
  // The shape checks of beam_step, then the Gumbel launch.
  const int rc = check_step_args(trie, step, logits, dtype, ld, parent_scores, parent_nodes, R,
                                 B_in, n_out, V, out_scores, out_parent, out_code, out_node,
                                 workspace);
  if (rc != SIDBEAM_OK) return rc;
  float* row_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                            gumbel_lse_offset(R, B_in, n_out, V));
  return launch_beam_step(trie, step, logits, dtype, ld, parent_scores, parent_nodes, R, B_in,
                          n_out, V, out_scores, out_parent, out_code, out_node, workspace,
                          workspace_bytes, static_cast<cudaStream_t>(stream), 0u, temperature,
                          seed, row_lse, nullptr, 0);
}

extern "C" int beam_finalize(int depth, int R, int n, const int32_t* bp_parent,
                             const int32_t* bp_code, const int32_t* last_node, int32_t* out_sids,
                             int32_t* out_leaf, void* stream) {
  if (!bp_parent || !bp_code || !last_node || !out_sids || !out_leaf)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_finalize: NULL pointer argument");
  if (depth < 1 || depth > SIDBEAM_MAX_DEPTH || R < 1 || n < 1)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_finalize: bad shape depth=%d R=%d n=%d",
                     depth, R, n);
  const int64_t total = static_cast<int64_t>(R) * n;
  int64_t g = (total + 255) / 256;
  if (g > 148 * 8) g = 148 * 8;
  finalize_kernel<<<static_cast<unsigned>(g), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      depth, R, n, bp_parent, bp_code, last_node, out_sids, out_leaf);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SIDBEAM_OK : cuda_error(e, "beam_finalize: launch");
}

extern "C" int beam_step_skipped_rows(void* workspace, uint32_t* count, void* stream) {
  if (!workspace || !count)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step_skipped_rows: NULL argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace) + kSkippedRowsOffset;
  uint32_t c = 0;
  cudaError_t e = cudaMemcpyAsync(&c, w, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && c) {
    const uint32_t zero = 0;
    e = cudaMemcpyAsync(w, &zero, 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return cuda_error(e, "beam_step_skipped_rows");
  *count = c;
  return SIDBEAM_OK;
}

extern "C" int sidbeam_get_device_status(void* workspace, void* stream) {
  if (!workspace) return set_error(SIDBEAM_ERR_INVALID_ARG, "sidbeam_get_device_status: NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "sidbeam_get_device_status");
  if (word) {
    const uint32_t zero = 0;
    e = cudaMemcpyAsync(workspace, &zero, 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_error(e, "sidbeam_get_device_status");
  }
  if (word & kStatusTimeout)
    return set_error(SIDBEAM_ERR_TIMEOUT, "a bounded wait inside a kernel gave up");
  if (word & kStatusBadNode)
    return set_error(SIDBEAM_ERR_DEVICE_CHECK, "a parent node id was outside the trie level");
  return SIDBEAM_OK;
}
