// The SID-range lm_head GEMM (tcgen05) shared by the C ABI and the fused step.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sidbeam {

constexpr int kLmheadPlain = 0;  // write the fp32 logits
constexpr int kLmheadFused = 1;  // per-tile (max, sum exp) + the valid children's logits

struct GemmArgs {
  int M, N, K;              // rows, codes (V), hidden size d
  int mode;                 // kLmheadPlain or kLmheadFused
  float* logits;            // plain: [M][ld_out] fp32; fused: child logits, [M][N]
  int64_t ld_out;
  float2* partial;          // fused: [M][ntiles] (max, sum exp) per 256-column tile
  const uint32_t* bitmap;   // fused: [M][words] valid-child bits per row (null: every code)
  int words;
  uint32_t* status;         // device status word
};

constexpr int kLmheadTileN = 256;

// Launches the GEMM on `stream` (host arguments already checked).
int launch_lmhead_gemm(const void* hidden, const void* w_sid, const GemmArgs& args,
                       cudaStream_t stream);

}  // namespace sidbeam
