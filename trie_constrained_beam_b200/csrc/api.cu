// C ABI entry points of libsidbeam: argument checks, workspace sizes,
// beam_finalize, device status and error strings. Argument errors are found
// here, on the host, before anything is launched.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

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

// One CTA per request. The parent slots of the inner levels 1 .. depth-2 go
// to shared memory as 16-bit slots (kNoSlot: outside [0, n)), so that each
// beam's chain of parent lookups runs there; the codes of all levels are then
// read from global memory together (one independent gather per level).
constexpr int kFinalizeThreads = 512;
constexpr uint16_t kNoSlot = 0xFFFFu;

__global__ void __launch_bounds__(kFinalizeThreads)
    finalize_kernel(int depth, int n, int64_t plane, const int32_t* __restrict__ bp_parent,
                    const int32_t* __restrict__ bp_code, const int32_t* __restrict__ last_node,
                    int32_t* __restrict__ out_sids, int32_t* __restrict__ out_leaf) {
  extern __shared__ uint16_t inner_slot[];  // [depth - 2][n]
  // Launched as a programmatic dependent of the last step: nothing is read
  // before that grid has completed and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t base = static_cast<int64_t>(blockIdx.x) * n;
  for (int t = 1; t < depth - 1; ++t)
    for (int k = threadIdx.x; k < n; k += blockDim.x) {
      const int32_t p = bp_parent[t * plane + base + k];
      inner_slot[(t - 1) * n + k] = (p >= 0 && p < n) ? static_cast<uint16_t>(p) : kNoSlot;
    }
  __syncthreads();
  constexpr int kD = SIDBEAM_MAX_DEPTH;
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const int64_t i = base + k;
    const int64_t top = (depth - 1) * plane + i;
    const int32_t code_top = bp_code[top];
    const int32_t leaf = last_node[i];
    int s = depth > 1 ? bp_parent[top] : 0;
    bool ok = code_top >= 0;  // a padded beam has no code at the last step
    // Slots of levels depth-2 .. 0, each in [0, n) for a valid beam.
    int slot[kD - 1];
#pragma unroll
    for (int t = kD - 2; t >= 0; --t) {
      slot[t] = 0;
      if (t < depth - 1) {
        if (s < 0 || s >= n) ok = false;
        if (ok) slot[t] = s;
        if (t >= 1) s = ok ? static_cast<int>(inner_slot[(t - 1) * n + s]) : -1;
      }
    }
    int32_t code[kD - 1];
#pragma unroll
    for (int t = 0; t < kD - 1; ++t)
      code[t] = (t < depth - 1 && ok) ? bp_code[t * plane + base + slot[t]] : -1;
    int32_t* sid = out_sids + i * depth;
#pragma unroll
    for (int t = 0; t < kD; ++t)
      if (t < depth) sid[t] = !ok ? -1 : (t == depth - 1 ? code_top : code[t]);
    out_leaf[i] = ok ? leaf : -1;
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

// Opt the finalize kernel into its largest shared-memory use once per device.
static cudaError_t finalize_opt_in() {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  constexpr int kMax = (SIDBEAM_MAX_DEPTH - 2) * SIDBEAM_MAX_BEAM * 2;
  if (dev < 0 || dev >= 64)
    return cudaFuncSetAttribute(finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMax);
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMax);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

extern "C" int beam_finalize(int depth, int R, int n, const int32_t* bp_parent,
                             const int32_t* bp_code, const int32_t* last_node, int32_t* out_sids,
                             int32_t* out_leaf, void* stream) {
  if (!bp_parent || !bp_code || !last_node || !out_sids || !out_leaf)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_finalize: NULL pointer argument");
  if (depth < 1 || depth > SIDBEAM_MAX_DEPTH || R < 1 || n < 1 || n > SIDBEAM_MAX_BEAM)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_finalize: bad shape depth=%d R=%d n=%d",
                     depth, R, n);
  const size_t smem = static_cast<size_t>(depth > 2 ? depth - 2 : 0) * n * sizeof(uint16_t);
  cudaError_t e = cudaSuccess;
  if (smem > 48 * 1024) {
    e = finalize_opt_in();
    if (e != cudaSuccess) return cuda_error(e, "beam_finalize: cudaFuncSetAttribute");
  }
  const int threads = std::min(kFinalizeThreads, (n + 31) / 32 * 32);
  // A programmatic dependent of the previous kernel on the stream (the last
  // beam_step): its launch overlaps that kernel's tail.
  cudaLaunchConfig_t lc{};
  lc.gridDim = dim3(static_cast<unsigned>(R));
  lc.blockDim = dim3(static_cast<unsigned>(threads));
  lc.dynamicSmemBytes = smem;
  lc.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  e = cudaLaunchKernelEx(&lc, finalize_kernel, depth, n, static_cast<int64_t>(R) * n, bp_parent,
                         bp_code, last_node, out_sids, out_leaf);
  if (e == cudaSuccess) e = cudaGetLastError();
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
