// Device twin of sidgen/host.py: seeded synthetic inputs made on the GPU.
//
// Bit-identical to the numpy twin: Philox4x32-10 (Salmon et al., SC'11),
// the SplitMix64 finaliser (Steele et al., OOPSLA'14), an integer Irwin-Hall
// sum of eight 16-bit uniforms, and one correctly rounded fp32 multiply
// (__fmul_rn) per normal draw. No beam-search arithmetic lives here.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

struct U4 { uint32_t x, y, z, w; };

__device__ __forceinline__ U4 philox10(U4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) { k0 += kPhiloxW0; k1 += kPhiloxW1; }
    const uint32_t hi0 = __umulhi(kPhiloxM0, c.x), lo0 = kPhiloxM0 * c.x;
    const uint32_t hi1 = __umulhi(kPhiloxM1, c.z), lo1 = kPhiloxM1 * c.z;
    c = U4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
  }
  return c;
}

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_draw(U4 r, float ksig) {
  int s = 0;
  s += (int)(r.x & 0xFFFFu) + (int)(r.x >> 16);
  s += (int)(r.y & 0xFFFFu) + (int)(r.y >> 16);
  s += (int)(r.z & 0xFFFFu) + (int)(r.z >> 16);
  s += (int)(r.w & 0xFFFFu) + (int)(r.w >> 16);
  const int centred = 2 * s - 8 * 65535;          // |centred| < 2^24: exact in fp32
  return __fmul_rn((float)centred, ksig);
}

__device__ __forceinline__ uint16_t to_bf16_rne(float x) {
  const uint32_t u = __float_as_uint(x);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

__global__ void philox_kernel(uint64_t seed, const uint32_t* __restrict__ ctr,
                              uint32_t* __restrict__ out, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    U4 c{ctr[4 * i], ctr[4 * i + 1], ctr[4 * i + 2], ctr[4 * i + 3]};
    U4 r = philox10(c, (uint32_t)seed, (uint32_t)(seed >> 32));
    out[4 * i] = r.x; out[4 * i + 1] = r.y; out[4 * i + 2] = r.z; out[4 * i + 3] = r.w;
  }
}

// One CTA-stride loop over (row, code); element (row, c) at counter
// (h lo, h hi, c, stream).
__global__ void row_logits_kernel(uint64_t seed, const uint64_t* __restrict__ hashes,
                                  int64_t rows, int V, int64_t ld, float ksig, int bf16,
                                  uint32_t stream, void* __restrict__ out) {
  const int64_t total = rows * (int64_t)V;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / V;
    const int c = (int)(i - row * V);
    const uint64_t h = hashes[row];
    const float x = normal_draw(
        philox10(U4{(uint32_t)h, (uint32_t)(h >> 32), (uint32_t)c, stream},
                 (uint32_t)seed, (uint32_t)(seed >> 32)),
        ksig);
    if (bf16) static_cast<uint16_t*>(out)[row * ld + c] = to_bf16_rne(x);
    else      static_cast<float*>(out)[row * ld + c] = x;
  }
}

__global__ void child_hash_kernel(const uint64_t* __restrict__ parent_hash, int R, int B_in,
                                  const int32_t* __restrict__ out_parent,
                                  const int32_t* __restrict__ out_code, int n, int level,
                                  uint64_t* __restrict__ child) {
  const int64_t total = (int64_t)R * n;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / n;
    const int p = out_parent[i];
    const int c = out_code[i];
    if (p < 0 || c < 0) { child[i] = 0; continue; }
    const uint64_t tag = ((uint64_t)level << 48) | (uint64_t)(uint32_t)c;
    child[i] = mix64(parent_hash[r * B_in + p] ^ tag);
  }
}

// Generic "counter = (a, b, c, stream)" fill: element (i, j, k) of an
// [A, B, C] array; used for score tables (r, l, c) and weights (c, k, 0).
__global__ void grid3_kernel(uint64_t seed, int64_t A, int64_t B, int64_t C, float ksig,
                             int bf16, uint32_t stream, int swap_bc, void* __restrict__ out) {
  const int64_t total = A * B * C;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t a = i / (B * C);
    const int64_t rem = i - a * B * C;
    const int64_t b = rem / C;
    const int64_t c = rem - b * C;
    U4 ctr = swap_bc ? U4{(uint32_t)a, (uint32_t)c, 0u, stream}
                     : U4{(uint32_t)a, (uint32_t)b, (uint32_t)c, stream};
    const float x = normal_draw(philox10(ctr, (uint32_t)seed, (uint32_t)(seed >> 32)), ksig);
    if (bf16) static_cast<uint16_t*>(out)[i] = to_bf16_rne(x);
    else      static_cast<float*>(out)[i] = x;
  }
}

// Hidden states [rows, d]: element (row, k) at counter (h lo, h hi, k, stream).
__global__ void hidden_kernel(uint64_t seed, const uint64_t* __restrict__ hashes, int64_t rows,
                              int d, float ksig, uint32_t stream, uint16_t* __restrict__ out) {
  const int64_t total = rows * (int64_t)d;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / d;
    const int k = (int)(i - row * d);
    const uint64_t h = hashes[row];
    out[i] = to_bf16_rne(normal_draw(
        philox10(U4{(uint32_t)h, (uint32_t)(h >> 32), (uint32_t)k, stream},
                 (uint32_t)seed, (uint32_t)(seed >> 32)),
        ksig));
  }
}

inline int grid_for(int64_t total) {
  int64_t g = (total + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  if (g < 1) g = 1;
  return (int)g;
}

inline int finish() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? 0 : (int)e;
}

}  // namespace

extern "C" {

int sidgen_philox(uint64_t seed, const uint32_t* ctr, uint32_t* out, int64_t n,
                  cudaStream_t stream) {
  if (n <= 0) return 0;
  philox_kernel<<<grid_for(n), 256, 0, stream>>>(seed, ctr, out, n);
  return finish();
}

int sidgen_row_logits(uint64_t seed, const uint64_t* hashes, int64_t rows, int V, int64_t ld,
                      float ksig, int bf16, int stream_id, void* out, cudaStream_t stream) {
  if (rows <= 0 || V <= 0) return 0;
  if (ld < V) return -1;
  row_logits_kernel<<<grid_for(rows * V), 256, 0, stream>>>(seed, hashes, rows, V, ld, ksig,
                                                            bf16, (uint32_t)stream_id, out);
  return finish();
}

int sidgen_child_hash(const uint64_t* parent_hash, int R, int B_in, const int32_t* out_parent,
                      const int32_t* out_code, int n, int level, uint64_t* child,
                      cudaStream_t stream) {
  if ((int64_t)R * n <= 0) return 0;
  child_hash_kernel<<<grid_for((int64_t)R * n), 256, 0, stream>>>(parent_hash, R, B_in,
                                                                  out_parent, out_code, n,
                                                                  level, child);
  return finish();
}

int sidgen_table(uint64_t seed, int R, int L, int V, float ksig, float* out,
                 cudaStream_t stream) {
  const int64_t total = (int64_t)R * L * V;
  if (total <= 0) return 0;
  grid3_kernel<<<grid_for(total), 256, 0, stream>>>(seed, R, L, V, ksig, 0, 1u, 0, out);
  return finish();
}

int sidgen_weight(uint64_t seed, int V, int d, float ksig, uint16_t* out, cudaStream_t stream) {
  const int64_t total = (int64_t)V * d;
  if (total <= 0) return 0;
  grid3_kernel<<<grid_for(total), 256, 0, stream>>>(seed, V, 1, d, ksig, 1, 3u, 1, out);
  return finish();
}

int sidgen_hidden(uint64_t seed, const uint64_t* hashes, int64_t rows, int d, float ksig,
                  uint16_t* out, cudaStream_t stream) {
  if (rows * (int64_t)d <= 0) return 0;
  hidden_kernel<<<grid_for(rows * d), 256, 0, stream>>>(seed, hashes, rows, d, ksig, 2u, out);
  return finish();
}

}  // extern "C"
