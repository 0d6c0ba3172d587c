// beam_step_noalloc: beam_step without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run a
// step: a plugin whose host application owns every device allocation (or
// enforces a fixed memory budget), a serving loop that plans all memory up
// front and treats any later cudaMalloc as a failure, or code on a path where
// allocating would synchronise the device. For them this entry point takes
// its scratch space from a fixed array compiled into the library instead of
// from a caller-supplied workspace.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds SIDBEAM_NOALLOC_SCRATCH_BYTES of it until the process exits.
// Its host-side name is only a stand-in, so the device address is looked up
// once per device (cudaGetSymbolAddress, with that device current) and passed
// to the kernel like any workspace.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include <mutex>

#include "internal.h"
#include "launch.h"

namespace sidbeam {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SIDBEAM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "beam_step_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step_noalloc: device %d not supported", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_error(e, "beam_step_noalloc: cudaGetSymbolAddress");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SIDBEAM_OK;
}

}  // namespace
}  // namespace sidbeam

using namespace sidbeam;

extern "C" int beam_step_noalloc(const sidbeam_trie* trie, int step, const void* logits,
                                 sidbeam_dtype dtype, int64_t ld, const float* parent_scores,
                                 const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                                 float* out_scores, int32_t* out_parent, int32_t* out_code,
                                 int32_t* out_node, void* stream) {
  const size_t need = beam_step_workspace_size(R, B_in, n_out, V);
  if (need == 0)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step_noalloc: invalid shape R=%d B_in=%d n=%d V=%d",
                     R, B_in, n_out, V);
  if (need > SIDBEAM_NOALLOC_SCRATCH_BYTES)
    return set_error(SIDBEAM_ERR_WORKSPACE,
                     "beam_step_noalloc: this shape needs %zu bytes of scratch; the built-in "
                     "array holds %d bytes (use beam_step with a workspace)",
                     need, SIDBEAM_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != SIDBEAM_OK) return rc;
  // The counters at the head of the scratch must start at zero (status word,
  // per-request tickets and bounds, histograms, partial-list sizes); the step
  // clears them on the stream after all of its argument checks have passed,
  // right before its kernel, so a rejected call enqueues nothing.
  const Partition p = make_partition(R, B_in, std::min(device_sm_count(), 640));
  const WorkspaceLayout ws = workspace_layout(R, p.maxG, n_out);
  return beam_step_checked(trie, step, logits, dtype, ld, parent_scores, parent_nodes, R, B_in,
                           n_out, V, out_scores, out_parent, out_code, out_node, scratch,
                           SIDBEAM_NOALLOC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream), 0u,
                           nullptr, ws.part_keys);
}
