// SID-range lm_head on the 5th-generation tensor cores (tcgen05), and the
// fused step it feeds.
//
// flashrec 0.1.0 (PyPI page), Features > Decoding ("SID constraint"): the
// lm_head is evaluated only over the SID token range and feeds the
// constrained step directly.
//
// logits[row][c] = sum_k H[row][k] * W[c][k] (H bf16 [M][d], W bf16 [V][d],
// both row-major: a "TN" GEMM, K-major on both sides), fp32 accumulation.
//
// Kernel (sm_100a, one CTA per SM, persistent over 128 x 256 output tiles):
//  * warp 0, one lane: TMA (cp.async.bulk.tensor.2d, 128-byte swizzle, no
//    multicast) of the H and W k-slices (64 wide) of a tile into a ring of 4
//    shared-memory stages (mbarrier complete_tx);
//  * warp 1: allocates 512 TMEM columns (two 128 x 256 fp32 accumulators) and,
//    from one lane, issues tcgen05.mma (M=128, N=256, K=16; bf16 in, fp32
//    accumulate in TMEM); tcgen05.commit frees a stage when its MMAs are done
//    and signals a finished accumulator;
//  * warps 2-5 (one per TMEM lane quarter: thread = output row): read the
//    accumulator with tcgen05.ld 32 columns at a time and either store the
//    logits (plain mode) or keep, per (row, 256-column tile), the partial max
//    and sum of exp and write the logits of the row's valid children only
//    (fused mode). Two accumulators let the epilogue of one tile overlap the
//    MMAs of the next.
// Every mbarrier wait is bounded; on expiry the status word records a timeout
// and the CTA finishes without further work.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "device_utils.cuh"
#include "internal.h"
#include "lmhead.h"

namespace sidbeam {
namespace {

using namespace dev;

constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kTileK = 64;                       // bf16: 128 bytes, one swizzle row
constexpr int kStages = 4;
constexpr int kABytes = kTileM * kTileK * 2;     // 16 KiB
constexpr int kBBytes = kTileN * kTileK * 2;     // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;   // 48 KiB
constexpr int kTmemCols = 512;                   // two accumulators of 256 columns
constexpr int kGemmThreads = 192;                // 6 warps
constexpr int kGemmSmem = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

// ------------------------------------------------------------ descriptors
// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, bf16 A
// and B, both K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4)            // D format: f32
                            | (1u << 7)          // A format: bf16
                            | (1u << 10)         // B format: bf16
                            | ((kTileN >> 3) << 17)
                            | ((kTileM >> 4) << 24);

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row swizzle atoms of 1024 bytes
// (stride byte offset 1024), leading byte offset unused (16), version 1,
// layout "swizzle 128B" (2). `addr` must lie in a 1024-byte aligned tile.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Wait for phase `parity` of `bar`, at most kWaitTimeoutNs; gives up early if
// *abort is set. Returns false when it gave up (and then sets *abort and the
// status word's timeout bit itself on expiry).
__device__ __forceinline__ bool gemm_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint32_t* status) {
  return bounded_wait(bar, parity, abort, status, kStatusTimeout);
}

}  // namespace

namespace {

__global__ void __launch_bounds__(kGemmThreads, 1)
    lmhead_gemm_kernel(const __grid_constant__ CUtensorMap map_h,
                       const __grid_constant__ CUtensorMap map_w, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // Stages on a 1024-byte boundary (the swizzle atom), barriers after them.
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;    // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;         // MMA completion before teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (a.M + kTileM - 1) / kTileM;
  const int n_tiles = (a.N + kTileN - 1) / kTileN;
  const int tiles = m_tiles * n_tiles;
  const int k_steps = (a.K + kTileK - 1) / kTileK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {  // the whole warp allocates; the address lands in shared memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_map(&map_h);
      prefetch_map(&map_w);
      uint32_t it = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int mt = t / n_tiles, nt = t - mt * n_tiles;
        for (int k = 0; k < k_steps; ++k, ++it) {
          const int s = static_cast<int>(it % kStages);
          if (it >= static_cast<uint32_t>(kStages) &&
              !gemm_wait(&empty[s], ((it / kStages) - 1) & 1u, abort_flag, a.status))
            goto producer_done;
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(st, &map_h, k * kTileK, mt * kTileM, &full[s]);
          tma_load_2d(st + kABytes, &map_w, k * kTileK, nt * kTileN, &full[s]);
        }
      }
    producer_done:
      // Copies still in flight land before the CTA goes away (normally they
      // have all been consumed already).
      for (uint32_t j = it > static_cast<uint32_t>(kStages) ? it - kStages : 0u; j < it; ++j)
        drain_wait(&full[j % kStages], (j / kStages) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, local = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
        const uint32_t ab = local & 1u;
        if (local >= 2 && !gemm_wait(&acc_empty[ab], ((local >> 1) - 1) & 1u, abort_flag,
                                     a.status))
          break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * kTileN;
        bool ok = true;
        for (int k = 0; k < k_steps; ++k, ++it) {
          const int s = static_cast<int>(it % kStages);
          if (!gemm_wait(&full[s], (it / kStages) & 1u, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + s * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk)  // 16 bf16 = 32 bytes per MMA
            umma_f16(d, smem_desc(sa + kk * 32), smem_desc(sb + kk * 32), kIdesc,
                     (k > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);  // the accumulator is complete
      }
      // Every MMA issued has completed before TMEM is freed.
      umma_commit(drain);
      drain_wait(drain, 0u);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int ew = warp - 2;                 // epilogue warp 0..3
    (void)ew;
    uint32_t local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const int mt = t / n_tiles, nt = t - mt * n_tiles;
      const uint32_t ab = local & 1u;
      if (!gemm_wait(&acc_full[ab], (local >> 1) & 1u, abort_flag, a.status)) break;
      tc_fence_after();
      const int row = mt * kTileM + quarter * 32 + lane;
      const uint32_t taddr = tmem_base + ab * kTileN + (static_cast<uint32_t>(quarter * 32) << 16);
      const int n0 = nt * kTileN;
      if (a.mode == kLmheadPlain) {
        for (int j = 0; j < kTileN / 32; ++j) {
          uint32_t v[32];
          tmem_ld32(taddr + j * 32, v);
          if (row < a.M) {
            float* out = a.logits + static_cast<int64_t>(row) * a.ld_out + n0 + j * 32;
            if (n0 + j * 32 + 32 <= a.N) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(out + e) =
                    make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (n0 + j * 32 + e < a.N) out[e] = __uint_as_float(v[e]);
            }
          }
        }
      } else {
        // Fused: partial max, then partial sum of exp, over this tile's valid
        // columns (all V codes: the normaliser is over the full codebook), and
        // the logits of the row's valid children.
        constexpr float kL2e = 1.4426950408889634f;
        float m = __int_as_float(0xFF800000);
        for (int j = 0; j < kTileN / 32; ++j) {
          uint32_t v[32];
          tmem_ld32(taddr + j * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (n0 + j * 32 + e < a.N) m = fmaxf(m, __uint_as_float(v[e]));
        }
        float s = 0.f;
        const float mL = m * kL2e;
        for (int j = 0; j < kTileN / 32; ++j) {
          uint32_t v[32];
          tmem_ld32(taddr + j * 32, v);
          const int c0 = n0 + j * 32;
          uint32_t bits = 0u;
          if (row < a.M && c0 < a.N)
            bits = a.bitmap ? a.bitmap[static_cast<int64_t>(row) * a.words + (c0 >> 5)] : ~0u;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (c0 + e < a.N) {
              const float z = __uint_as_float(v[e]);
              s += ex2_approx(fmaf(z, kL2e, -mL));
              if ((bits >> e) & 1u)
                a.logits[static_cast<int64_t>(row) * a.N + c0 + e] = z;
            }
          }
        }
        if (row < a.M) a.partial[static_cast<int64_t>(row) * n_tiles + nt] = make_float2(m, s);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }

  // Teardown: every warp is done with TMEM (the epilogue's last reads finished
  // before its arrivals; the MMA warp's last commit has fired before the
  // epilogue could read), then the allocating warp frees it.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
}

// ------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix, box [box_rows][64].
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int launch_lmhead_gemm(const void* hidden, const void* w_sid, const GemmArgs& args,
                       cudaStream_t stream) {
  CUtensorMap mh, mw;
  if (!make_map(&mh, hidden, args.M, args.K, kTileM) ||
      !make_map(&mw, w_sid, args.N, args.K, kTileN))
    return set_error(SIDBEAM_ERR_CUDA, "lm_head: tensor map encoding failed");
  static std::mutex mu;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "lm_head: cudaGetDevice");
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
      e = cudaFuncSetAttribute(lmhead_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kGemmSmem);
      if (e != cudaSuccess) return cuda_error(e, "lm_head: cudaFuncSetAttribute");
      if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
  }
  const int tiles = ((args.M + kTileM - 1) / kTileM) * ((args.N + kTileN - 1) / kTileN);
  int grid = device_sm_count();
  if (grid > tiles) grid = tiles;
  if (grid < 1) grid = 1;
  lmhead_gemm_kernel<<<grid, kGemmThreads, kGemmSmem, stream>>>(mh, mw, args);
  e = cudaGetLastError();
  return e == cudaSuccess ? SIDBEAM_OK : cuda_error(e, "lm_head: launch");
}

}  // namespace sidbeam

using namespace sidbeam;

extern "C" int lmhead_logits(const void* hidden, const void* w_sid, int M, int V, int d,
                             float* logits, int64_t ld, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!hidden || !w_sid || !logits)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "lmhead_logits: NULL pointer argument");
  if (M < 1 || V < 1 || d < 1 || V > SIDBEAM_MAX_V)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "lmhead_logits: bad shape M=%d V=%d d=%d", M, V, d);
  if (ld < V || (ld & 3) != 0)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "lmhead_logits: ld=%lld must be >= V and a multiple of 4",
                     static_cast<long long>(ld));
  if ((d & 7) != 0 || (reinterpret_cast<uintptr_t>(hidden) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(w_sid) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(logits) & 15u) != 0)
    return set_error(SIDBEAM_ERR_ALIGNMENT,
                     "lmhead_logits: hidden, w_sid and logits must be 16-byte aligned, d %% 8 == 0");
  if (!workspace || workspace_bytes < 256 || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return set_error(SIDBEAM_ERR_WORKSPACE, "lmhead_logits: workspace of >= 256 bytes, 256-byte aligned");
  GemmArgs a{};
  a.M = M;
  a.N = V;
  a.K = d;
  a.mode = kLmheadPlain;
  a.logits = logits;
  a.ld_out = ld;
  a.status = static_cast<uint32_t*>(workspace);
  return launch_lmhead_gemm(hidden, w_sid, a, static_cast<cudaStream_t>(stream));
}

namespace sidbeam {
int launch_fused_lmhead(const sidbeam_trie* trie, int step, const void* hidden,
                        const void* w_sid, int d, const float* parent_scores,
                        const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                        float* out_scores, int32_t* out_parent, int32_t* out_code,
                        int32_t* out_node, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);
size_t fused_lmhead_workspace(int R, int B_in, int n_out, int V);
}  // namespace sidbeam

extern "C" size_t fused_lmhead_workspace_size(int R, int B_in, int n_out, int V) {
  if (R < 1 || B_in < 1 || n_out < 1 || n_out > SIDBEAM_MAX_BEAM || V < 1 || V > SIDBEAM_MAX_V)
    return 0;
  return fused_lmhead_workspace(R, B_in, n_out, V);
}

extern "C" int sidbeam_fused_lmhead_step(const sidbeam_trie* trie, int step, const void* hidden,
                                         const void* w_sid, int d, const float* parent_scores,
                                         const int32_t* parent_nodes, int R, int B_in, int n_out,
                                         int V, float* out_scores, int32_t* out_parent,
                                         int32_t* out_code, int32_t* out_node, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  if (!hidden || !w_sid || !parent_scores || !out_scores || !out_parent || !out_code || !out_node)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "fused_lmhead_step: NULL pointer argument");
  if (trie && !parent_nodes)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "fused_lmhead_step: parent_nodes is NULL with a trie");
  if (R < 1 || B_in < 1 || d < 1)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "fused_lmhead_step: R=%d B_in=%d d=%d", R, B_in, d);
  if (n_out < 1 || n_out > SIDBEAM_MAX_BEAM)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "fused_lmhead_step: n_out=%d outside [1, %d]", n_out,
                     SIDBEAM_MAX_BEAM);
  if (V < 1 || V > SIDBEAM_MAX_V)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "fused_lmhead_step: V=%d unsupported", V);
  if (static_cast<uint64_t>(B_in) * static_cast<uint64_t>(V) > 0xFFFFFFFFull ||
      static_cast<int64_t>(R) * B_in > 0x7FFFFFFFll || static_cast<int64_t>(R) * n_out > 0x7FFFFFFFll)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "fused_lmhead_step: shape too large");
  if ((d & 7) != 0 || (reinterpret_cast<uintptr_t>(hidden) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(w_sid) & 15u) != 0)
    return set_error(SIDBEAM_ERR_ALIGNMENT,
                     "fused_lmhead_step: hidden and w_sid 16-byte aligned, d %% 8 == 0");
  if (trie) {
    if (step < 0 || step >= trie->depth)
      return set_error(SIDBEAM_ERR_INVALID_ARG, "fused_lmhead_step: step %d outside [0, %d)", step,
                       trie->depth);
    if (trie->V[step] != V)
      return set_error(SIDBEAM_ERR_INVALID_ARG,
                       "fused_lmhead_step: V=%d but the trie has V=%d at level %d", V,
                       trie->V[step], step + 1);
  }
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return set_error(SIDBEAM_ERR_WORKSPACE, "fused_lmhead_step: workspace must be 256-byte aligned");
  return launch_fused_lmhead(trie, step, hidden, w_sid, d, parent_scores, parent_nodes, R, B_in,
                             n_out, V, out_scores, out_parent, out_code, out_node, workspace,
                             workspace_bytes, static_cast<cudaStream_t>(stream));
}
