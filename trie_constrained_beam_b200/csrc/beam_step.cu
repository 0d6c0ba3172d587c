// beam_step: one catalog-constrained expansion step for all beam rows.
//
// flashrec 0.1.0 (PyPI page), Features > Decoding ("SID constraint"): a fused
// kernel restricts every continuation to the catalog trie (dense or CSR);
// Features > Serving ("API"): deterministic top-k at temperature 0.
//
// Design (sm_100a):
//  * One CTA per SM; the rows of a CTA are dealt to its warps (row i of the
//    CTA to warp i mod W). When a CTA has fewer rows than warps, every warp
//    takes every row and the candidate walk is split between them.
//  * Every warp streams its own rows: it owns a ring of S shared-memory
//    stages and, from one lane, issues untiled bulk copies (cp.async.bulk,
//    the TMA engine; no multicast) of the logits row and of the node's trie
//    data (the dense bitmask row, or the first child codes at CSR levels)
//    into a stage that completes on the stage's mbarrier. The first copies go
//    out before the row's parent score and node have even been read.
//  * A row of up to 8 KB is copied into registers (plus the trie data its
//    candidate walk needs) and the stage is refilled at once with the warp's
//    row S places ahead; larger rows are worked on in place.
//  * Row max and the full-codebook log-normaliser lse = m + log(sum exp(z-m))
//    in fp32 (packed f32x2 arithmetic, ex2.approx, warp shuffles); then the
//    node's children are walked twice, above a threshold that is always a
//    valid lower bound on the request's n-th best key: first counted in the
//    CTA's score histogram, then offered as key(score = s + (z_c - lse),
//    idx = b*V + c) to the warp's top-n buffer.
//  * At the end of a request segment the warps hand their candidates over
//    (topn.cuh): a CTA that holds a whole request ranks them itself, else the
//    last of the request's CTAs ranks everyone's partial lists.
// The logits are read exactly once from HBM.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"
#include "launch.h"
#include "step_plan.h"
#include "topn.cuh"

namespace sidbeam {
namespace {

using namespace dev;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kRegVecs = 16;  // 16-byte vectors per lane held in registers (8 KB rows)
// A register row with more hits than this is walked in two passes (count,
// raise the threshold, offer).
constexpr int kOnePassHits = 64;
constexpr uint32_t kFull = 0xFFFFFFFFu;
// Dense rows with more children than this, when every warp of the CTA takes
// the row, are walked in place in their stage.
constexpr uint32_t kHugeDense = 2048;

// f(I) for I = 0 .. N-1 with I a compile-time constant (keeps register arrays
// indexed statically).
template <int I> struct Idx { static constexpr int value = I; };
template <int N>
struct Unrolled {
  template <class F>
  __device__ __forceinline__ static void run(F&& f) {
    Unrolled<N - 1>::run(f);
    f(Idx<N - 1>{});
  }
};
template <>
struct Unrolled<0> {
  template <class F>
  __device__ __forceinline__ static void run(F&&) {}
};

struct StepArgs {
  const uint8_t* logits;
  int64_t row_bytes;  // ld * sizeof(dtype)
  int bf16;
  int V;
  const float* parent_scores;
  const int32_t* parent_nodes;
  int R, B_in, n;
  int layout;  // 0 = none (unconstrained), SIDBEAM_LAYOUT_DENSE, SIDBEAM_LAYOUT_CSR
  const uint32_t* off;
  const uint32_t* mask;
  int mask_words, mask_stride;
  const uint16_t* codes;
  int64_t n_parent;
  float* out_scores;
  int32_t* out_parent;
  int32_t* out_code;
  int32_t* out_node;
  uint32_t* status;
  uint32_t* tickets;
  unsigned long long* request_thr;
  uint32_t* part_count;
  unsigned long long* part_keys;
  int32_t* part_vals;
  uint32_t* ghist;
  Partition part;
  StepConfig cfg;
  int coop;  // 1: every warp takes every row of the CTA (fewer rows than warps)
  int skip_rows;     // 1: rows whose parent score is below the request's bound are not read
  uint32_t* skipped; // counter of rows not read for that reason
  // Gumbel top-k (temperature gumbel_T > 0; the kernel instantiation with GUM = 1)
  float gumbel_T;
  uint32_t gseed0, gseed1;  // Philox key (seed lo, hi)
  int gstep;                // counter word 3
  float* row_lse;           // [R * B_in]: every live row's lse (the writer needs it)
  const int32_t* out_width; // [R] beams kept per request (<= n), or null (n for all)
};

// ------------------------------------------------------------ Gumbel top-k
// Temperature T > 0 (flashrec 0.1.0, Features > Serving, "API": Gumbel top-k
// without replacement above temperature 0): candidate c of parent slot b in
// request r gets the key of s + (z_c + T*G - lse), G a standard Gumbel
// variate for (r, b, c, step); the n largest keys are a draw of n candidates
// without replacement in proportion to exp(score / T), and the beams keep
// the unperturbed score (written out from the row's logits and lse).
// G = -log(-log U), U = (v + 1/2) 2^-23 exact in fp32, v = the top 23 bits of
// the first word of Philox4x32-10 (Salmon et al., SC'11) on counter
// (r, b, c, step), key = the seed. G <= kGumbelMax for every U.
constexpr float kGumbelMax = 16.7f;

__device__ __forceinline__ uint32_t philox_word0(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    if (i > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

// T * G for candidate (r, b, code).
__device__ __forceinline__ float gumbel_noise(const StepArgs& a, int r, uint32_t b, int code) {
  const uint32_t v = philox_word0(static_cast<uint32_t>(r), b, static_cast<uint32_t>(code),
                                  static_cast<uint32_t>(a.gstep), a.gseed0, a.gseed1) >> 9;
  const float U = (static_cast<float>(v) + 0.5f) * 1.1920928955078125e-07f;  // 2^-23
  return a.gumbel_T * -logf(-logf(U));
}

// The writer of a Gumbel step: the ranks follow the perturbed keys; the score
// written is the unperturbed s + (z - lse), recomputed from the row exactly as
// the deterministic step computes it.
struct GumbelWriter {
  float* scores;
  int32_t* parent;
  int32_t* code;
  int32_t* node;
  int n;
  uint32_t V;
  const uint8_t* logits;
  int64_t row_bytes;
  int bf16;
  const float* parent_scores;
  const float* row_lse;
  int B_in;
  const int32_t* width;
  __device__ __forceinline__ void operator()(int r, int i, uint64_t key, int32_t val,
                                             bool valid) const {
    const size_t o = static_cast<size_t>(r) * n + i;
    if (valid && (!width || i < width[r])) {
      const uint32_t idx = key_idx(key);
      const int32_t b = static_cast<int32_t>(idx / V), c = static_cast<int32_t>(idx % V);
      const int64_t row = static_cast<int64_t>(r) * B_in + b;
      const uint8_t* zr = logits + row * row_bytes;
      const float z = bf16 ? __uint_as_float(static_cast<uint32_t>(
                                 reinterpret_cast<const uint16_t*>(zr)[c]) << 16)
                           : reinterpret_cast<const float*>(zr)[c];
      scores[o] = parent_scores[row] + (z - row_lse[row]);
      parent[o] = b;
      code[o] = c;
      node[o] = val;
    } else {
      scores[o] = __int_as_float(0xFF800000);
      parent[o] = -1;
      code[o] = -1;
      node[o] = -1;
    }
  }
};

// Ranks at or past a request's width (out_width) are written as padding: the
// top-w of a request are the first w ranks of its top-n.
struct StepWriter {
  float* scores;
  int32_t* parent;
  int32_t* code;
  int32_t* node;
  int n;
  uint32_t V;
  const int32_t* width;
  __device__ __forceinline__ void operator()(int r, int i, uint64_t key, int32_t val,
                                             bool valid) const {
    const size_t o = static_cast<size_t>(r) * n + i;
    if (valid && (!width || i < width[r])) {
      const uint32_t idx = key_idx(key);
      scores[o] = key_score(key);
      parent[o] = static_cast<int32_t>(idx / V);
      code[o] = static_cast<int32_t>(idx % V);
      node[o] = val;
    } else {
      scores[o] = __int_as_float(0xFF800000);  // -inf
      parent[o] = -1;
      code[o] = -1;
      node[o] = -1;
    }
  }
};

// --------------------------------------------------------------- row math
template <int BF16>
__device__ __forceinline__ float elem(const uint8_t* row, int c) {
  if (BF16) {
    const uint32_t u = static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(row)[c]) << 16;
    return __uint_as_float(u);
  }
  return reinterpret_cast<const float*>(row)[c];
}

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Packed fp32 pairs (sm_100 f32x2 arithmetic).
__device__ __forceinline__ uint64_t pk(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float pk_lo(uint64_t p) { return __uint_as_float(static_cast<uint32_t>(p)); }
__device__ __forceinline__ float pk_hi(uint64_t p) { return __uint_as_float(static_cast<uint32_t>(p >> 32)); }
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t ex2_pair(uint64_t p) {
  return pk(ex2_approx(pk_lo(p)), ex2_approx(pk_hi(p)));
}

// Max of the 16 bytes `q` (8 bf16 or 4 fp32 values).
template <int BF16>
__device__ __forceinline__ float vec_max(const uint4& q) {
  if (BF16) {
    const uint32_t w = bmax2(bmax2(q.x, q.y), bmax2(q.z, q.w));
    return fmaxf(bf_lo(w), bf_hi(w));
  }
  return fmaxf(fmaxf(__uint_as_float(q.x), __uint_as_float(q.y)),
               fmaxf(__uint_as_float(q.z), __uint_as_float(q.w)));
}

// Pairwise sums of 2^(z*log2e - m*log2e) over the 16 bytes `q`, as a packed pair.
template <int BF16>
__device__ __forceinline__ uint64_t vec_sumexp2(const uint4& q, uint64_t l2e, uint64_t nml) {
  if (BF16) {
    const uint64_t e0 = ex2_pair(ffma2(pk(bf_lo(q.x), bf_hi(q.x)), l2e, nml));
    const uint64_t e1 = ex2_pair(ffma2(pk(bf_lo(q.y), bf_hi(q.y)), l2e, nml));
    const uint64_t e2 = ex2_pair(ffma2(pk(bf_lo(q.z), bf_hi(q.z)), l2e, nml));
    const uint64_t e3 = ex2_pair(ffma2(pk(bf_lo(q.w), bf_hi(q.w)), l2e, nml));
    return fadd2(fadd2(e0, e1), fadd2(e2, e3));
  }
  const uint64_t e0 = ex2_pair(ffma2(pk(__uint_as_float(q.x), __uint_as_float(q.y)), l2e, nml));
  const uint64_t e1 = ex2_pair(ffma2(pk(__uint_as_float(q.z), __uint_as_float(q.w)), l2e, nml));
  return fadd2(e0, e1);
}

// Row max m and full-codebook log-normaliser lse = m + log(sum_c exp(z_c - m))
// of one row in shared memory (warp-collective, fp32).
template <int BF16>
__device__ __forceinline__ void row_stats(const uint8_t* row, int V, int lane, float& m_out,
                                          float& lse_out) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  const int nvec = V / kPerVec;  // full 16-byte vectors
  const int tail0 = nvec * kPerVec;
  const uint4* q = reinterpret_cast<const uint4*>(row);
  float m;
  if (BF16) {
    uint32_t r = 0xFF80FF80u;  // (-inf, -inf)
    for (int v = lane; v < nvec; v += 32) {
      const uint4 x = q[v];
      r = bmax2(r, bmax2(bmax2(x.x, x.y), bmax2(x.z, x.w)));
    }
    m = fmaxf(bf_lo(r), bf_hi(r));
  } else {
    m = __int_as_float(0xFF800000);
    for (int v = lane; v < nvec; v += 32) m = fmaxf(m, vec_max<0>(q[v]));
  }
  if (lane < V - tail0) m = fmaxf(m, elem<BF16>(row, tail0 + lane));
  // Each lane sums exp(z - m_lane) against its own max, so the exponentials
  // start without waiting for a warp-wide reduction; the lanes are combined
  // once at the end (sum * 2^((m_lane - m) * log2e)).
  const float mL = m * kLog2e;
  const uint64_t l2e = pk(kLog2e, kLog2e);
  const uint64_t nml = pk(-mL, -mL);
  uint64_t a0 = 0, a1 = 0;  // packed (0.f, 0.f)
  int v = lane;
  for (; v + 32 < nvec; v += 64) {
    a0 = fadd2(a0, vec_sumexp2<BF16>(q[v], l2e, nml));
    a1 = fadd2(a1, vec_sumexp2<BF16>(q[v + 32], l2e, nml));
  }
  if (v < nvec) a0 = fadd2(a0, vec_sumexp2<BF16>(q[v], l2e, nml));
  const uint64_t a = fadd2(a0, a1);
  float sum = pk_lo(a) + pk_hi(a);
  if (lane < V - tail0) sum += ex2_approx(fmaf(elem<BF16>(row, tail0 + lane), kLog2e, -mL));
  const float mw = warp_max(m);
  sum = (m > __int_as_float(0xFF800000)) ? sum * ex2_approx((m - mw) * kLog2e) : 0.f;
  sum = warp_sum(sum);
  m = mw;
  m_out = m;
  lse_out = m + logf(sum);
}


// --------------------------------------------------------------- register rows
// Element j of a 16-byte vector (8 bf16 or 4 fp32), j warp-divergent.
template <int BF16>
__device__ __forceinline__ float vec_elem(const uint4& x, int j) {
  if (BF16) {
    const uint32_t w = (j < 4) ? ((j < 2) ? x.x : x.y) : ((j < 6) ? x.z : x.w);
    return (j & 1) ? bf_hi(w) : bf_lo(w);
  }
  const uint32_t w = (j < 2) ? ((j < 1) ? x.x : x.y) : ((j < 3) ? x.z : x.w);
  return __uint_as_float(w);
}

// Elements j >= keep of a vector become -inf (they lie past V).
__device__ __forceinline__ uint32_t cut_word_bf16(uint32_t w, int first, int keep) {
  if (first >= keep) return 0xFF80FF80u;
  if (first + 1 >= keep) return (w & 0x0000FFFFu) | 0xFF800000u;
  return w;
}
template <int BF16>
__device__ __forceinline__ void vec_cut(uint4& x, int keep) {
  if (BF16) {
    x.x = cut_word_bf16(x.x, 0, keep);
    x.y = cut_word_bf16(x.y, 2, keep);
    x.z = cut_word_bf16(x.z, 4, keep);
    x.w = cut_word_bf16(x.w, 6, keep);
  } else {
    if (1 >= keep) x.y = 0xFF800000u;
    if (2 >= keep) x.z = 0xFF800000u;
    if (3 >= keep) x.w = 0xFF800000u;
  }
}

// Row max and log-normaliser of a row held in registers (vector lane + 32k in
// x[k]; entries past V are -inf and contribute exp(-inf) = 0).
// FULL: every lane holds kRegVecs real vectors (a full 8 KB row); the loops
// are then straight-line code the compiler can interleave freely.
template <int BF16, bool FULL = false>
__device__ __forceinline__ void row_stats_reg(const uint4 (&x)[kRegVecs], int nvec, int lane,
                                              float& m_out, float& lse_out) {
  float m;
  if (BF16) {
    uint32_t r = 0xFF80FF80u;
    Unrolled<kRegVecs>::run([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      if (FULL || 32 * k < nvec) r = bmax2(r, bmax2(bmax2(x[k].x, x[k].y), bmax2(x[k].z, x[k].w)));
    });
    m = fmaxf(bf_lo(r), bf_hi(r));
  } else {
    m = __int_as_float(0xFF800000);
    Unrolled<kRegVecs>::run([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      if (FULL || 32 * k < nvec) m = fmaxf(m, vec_max<0>(x[k]));
    });
  }
  // Lane-local max for the exponentials; lanes combined once at the end.
  const float mL = m * kLog2e;
  const uint64_t l2e = pk(kLog2e, kLog2e);
  const uint64_t nml = pk(-mL, -mL);
  uint64_t a0 = 0, a1 = 0;
  Unrolled<kRegVecs>::run([&](auto kc) {
    constexpr int k = decltype(kc)::value;
    if (FULL || 32 * k < nvec) {
      if (k & 1) a1 = fadd2(a1, vec_sumexp2<BF16>(x[k], l2e, nml));
      else a0 = fadd2(a0, vec_sumexp2<BF16>(x[k], l2e, nml));
    }
  });
  const uint64_t a = fadd2(a0, a1);
  float sum = pk_lo(a) + pk_hi(a);
  const float mw = warp_max(m);
  sum = (m > __int_as_float(0xFF800000)) ? sum * ex2_approx((m - mw) * kLog2e) : 0.f;
  sum = warp_sum(sum);
  m = mw;
  m_out = m;
  lse_out = m + logf(sum);
}

// Node id of dense child code c: first child id + rank of c among the node's
// set bits. `prefix` holds the set-bit counts before each mask word.
__device__ __forceinline__ int32_t dense_child(const uint32_t* mrow, const uint32_t* prefix,
                                               uint32_t o0, int c) {
  const uint32_t w = mrow[c >> 5];
  return static_cast<int32_t>(o0 + prefix[c >> 5] + __popc(w & ((1u << (c & 31)) - 1u)));
}

// Set-bit counts before every word of a dense mask row (warp-collective).
__device__ __forceinline__ void dense_prefix(const uint32_t* mrow, int words, uint32_t* prefix,
                                             int lane) {
  uint32_t carry = 0;
  for (int k0 = 0; k0 < words; k0 += 32) {
    const int k = k0 + lane;
    const uint32_t p = k < words ? static_cast<uint32_t>(__popc(mrow[k])) : 0u;
    uint32_t incl = p;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    if (k < words) prefix[k] = carry + incl - p;
    carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  __syncwarp();
}


// --------------------------------------------------------------- warp rings
// The rows a warp takes, in order: row(i) for i < count.
struct RowSeq {
  int64_t first;
  int64_t stride;
  int count;
  __device__ __forceinline__ int64_t row(int i) const { return first + stride * i; }
};

// Parent data of 32 consecutive entries of a warp's row sequence, one per lane.
struct MetaBatch {
  int base;         // sequence index of lane 0's row (a multiple of 32)
  float s;          // parent score
  int32_t p;        // parent node
  uint32_t o0, o1;  // children of p: ids o0 .. o1-1 (trie levels only)
  unsigned live;    // lanes whose row is expanded
};

// A row is dead (skipped, its logits never used) when its parent score is
// -inf or, with a trie, its node is negative; a node past the level's end is
// also skipped and reported in the status word.
__device__ __forceinline__ void load_meta(const StepArgs& a, const RowSeq& q, int base, int lane,
                                          MetaBatch& m) {
  const int i = base + lane;
  const bool in = i < q.count;
  float s = __int_as_float(0xFF800000);
  int32_t p = -1;
  if (in) {
    const int64_t row = q.row(i);
    s = a.parent_scores[row];
    p = a.layout ? a.parent_nodes[row] : 0;
  }
  bool live = in && s != __int_as_float(0xFF800000);
  if (a.layout) {
    if (p < 0) {
      live = false;
    } else if (static_cast<int64_t>(p) >= a.n_parent) {
      if (live) atomicOr(a.status, kStatusBadNode);
      live = false;
    }
  }
  uint32_t o0 = 0, o1 = 0;
  if (live && a.layout) {
    o0 = a.off[p];
    o1 = a.off[p + 1];
  }
  m.base = base;
  m.s = s;
  m.p = p;
  m.o0 = o0;
  m.o1 = o1;
  m.live = __ballot_sync(kFull, live);
}

// CSR: child codes staged behind the row start at id a0 = o0 rounded down to
// a multiple of 8 (a 16-byte boundary); at most extra_bytes / 2 of them.
__device__ __forceinline__ uint32_t csr_staged(const StepArgs& a, uint32_t o0, uint32_t o1) {
  if (o1 <= o0) return 0u;
  const uint32_t n = o1 - (o0 & ~7u);
  const uint32_t cap = static_cast<uint32_t>(a.cfg.extra_bytes / 2);
  return n < cap ? n : cap;
}

// Bytes of trie data staged behind a live row.
__device__ __forceinline__ uint32_t extra_bytes(const StepArgs& a, uint32_t o0, uint32_t o1) {
  if (a.layout == SIDBEAM_LAYOUT_DENSE) return static_cast<uint32_t>(a.mask_stride) * 4u;
  if (a.layout == SIDBEAM_LAYOUT_CSR) return (csr_staged(a, o0, o1) * 2u + 15u) & ~15u;
  return 0u;
}

// Copy of the trie data of node p behind the row (one lane; bytes > 0).
__device__ __forceinline__ void copy_extra(const StepArgs& a, uint8_t* stage, uint64_t* bar,
                                           int32_t p, uint32_t o0, uint32_t bytes,
                                           uint64_t pol) {
  const void* src = a.layout == SIDBEAM_LAYOUT_DENSE
                        ? static_cast<const void*>(a.mask + static_cast<size_t>(p) * a.mask_stride)
                        : static_cast<const void*>(a.codes + (o0 & ~7u));
  bulk_copy_g2s(stage + a.cfg.logits_copy_bytes, src, bytes, bar, pol);
}

// One warp's ring. Entry k of the warp's ring traffic goes to stage k % S; the
// parent data of the row in stage j is kept in lane j (st_*).
struct Ring {
  uint8_t* stages;
  uint64_t* full;
  int S;
  int consumed;  // rows taken out of the ring (warp-uniform)
  int issued;    // rows put into the ring (warp-uniform)
  int ip;        // next sequence index to look at for issuing (warp-uniform)
  int st_seq;
  int st_live;
  float st_s;
  int32_t st_p;
  uint32_t st_o0, st_o1;
};

// Puts the next live row of the sequence into the stage just released (the
// ring is full whenever this succeeds, so that stage is issued % S). The
// stage's earlier contents were read by this warp's lanes: __syncwarp orders
// those reads before lane 0, and the proxy fence before the async copy.
// Returns false when the sequence has no live row left. Warp-collective.
// Row skipping (optional). Every child score s + (z - lse) is at most the
// parent score s in fp32 (z <= lse, so z - lse <= 0 after rounding, and
// adding a non-positive number does not raise s), so the largest key a child
// of the row can have is key(s, lowest index). When that is below a valid
// lower bound on the request's n-th best key, no child of the row can be
// selected and its logits need not be read: the result is the same.
__device__ __forceinline__ bool row_skippable(float s, uint64_t bound) {
  return bound != 0ull && make_key(s, 0u) < bound;
}

// Issues row `row` (sequence entry seq, parent data s, p, o0..o1) into the
// stage just released: its logits and, behind them, its trie data.
__device__ __forceinline__ void ring_issue(const StepArgs& a, Ring& g, int lane, uint64_t pol,
                                           int seq, int64_t row, float s, int32_t p, uint32_t o0,
                                           uint32_t o1) {
  const int stage = g.issued % g.S;
  if (lane == stage) {
    g.st_seq = seq;
    g.st_live = 1;
    g.st_s = s;
    g.st_p = p;
    g.st_o0 = o0;
    g.st_o1 = o1;
  }
  __syncwarp();
  if (lane == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    uint8_t* dst = g.stages + static_cast<size_t>(stage) * a.cfg.stage_bytes;
    const uint32_t ex = extra_bytes(a, o0, o1);
    mbar_arrive_expect_tx(&g.full[stage], static_cast<uint32_t>(a.cfg.logits_copy_bytes) + ex);
    bulk_copy_g2s(dst, a.logits + row * a.row_bytes,
                  static_cast<uint32_t>(a.cfg.logits_copy_bytes), &g.full[stage], pol);
    if (ex) copy_extra(a, dst, &g.full[stage], p, o0, ex, pol);
  }
  ++g.issued;
}

// Puts the next live row of the warp's own sequence into the stage just
// released (parent data read 32 entries at a time). Returns false when the
// sequence is exhausted. Rows that row_skippable rules out against `bound`
// (0: none) are passed over and counted.
__device__ __forceinline__ bool ring_refill(const StepArgs& a, const RowSeq& q, MetaBatch& mb,
                                           Ring& g, int lane, uint64_t pol, uint64_t bound) {
  while (g.ip < q.count) {
    if (g.ip >= mb.base + 32) load_meta(a, q, g.ip & ~31, lane, mb);
    const unsigned m = mb.live & (~0u << (g.ip - mb.base));
    if (m == 0u) {
      g.ip = mb.base + 32;
      continue;
    }
    const int j = __ffs(m) - 1;
    const float s = __shfl_sync(kFull, mb.s, j);
    const int32_t p = __shfl_sync(kFull, mb.p, j);
    const uint32_t o0 = __shfl_sync(kFull, mb.o0, j);
    const uint32_t o1 = __shfl_sync(kFull, mb.o1, j);
    const int seq = mb.base + j;
    g.ip = seq + 1;
    if (row_skippable(s, bound)) {
      if (lane == 0) atomicAdd(a.skipped, 1u);
      continue;
    }
    ring_issue(a, g, lane, pol, seq, q.row(seq), s, p, o0, o1);
    return true;
  }
  return false;
}

// The same from the CTA's shared row table: the next entry of the CTA's
// sequence goes to whichever warp asks first, so that a warp held up by a
// heavy row takes fewer rows. Dead entries (score -inf in the table) are
// skipped. cq: the CTA's whole sequence.
__device__ __forceinline__ bool ring_refill_shared(const StepArgs& a, const RowSeq& cq,
                                                  const uint4* meta, int* next, Ring& g, int lane,
                                                  uint64_t pol, uint64_t bound) {
  for (;;) {
    int j = 0;
    if (lane == 0) j = atomicAdd(next, 1);
    j = __shfl_sync(kFull, j, 0);
    if (j >= cq.count) return false;
    const uint4 m = meta[j];
    const float s = __uint_as_float(m.x);
    if (s == __int_as_float(0xFF800000)) continue;
    if (row_skippable(s, bound)) {
      if (lane == 0) atomicAdd(a.skipped, 1u);
      continue;
    }
    ring_issue(a, g, lane, pol, j, cq.row(j), s, static_cast<int32_t>(m.y), m.z, m.w);
    return true;
  }
}

// --------------------------------------------------------------- row walks
// What the walks need to know about a row.
struct RowCtx {
  float s;        // parent score
  float lse;      // log-normaliser over the full codebook
  float C;        // histogram reference of the request
  uint32_t idx0;  // b * V (key index of code 0)
  uint32_t o0;    // first child id
  uint32_t o1;    // one past the last child id
  int r;          // request (Gumbel counters)
  uint32_t b;     // parent slot in the request
};

// Code of CSR child id k: from the stage when it was staged, else from HBM/L2.
__device__ __forceinline__ int csr_code(const StepArgs& a, const uint8_t* zrow, uint32_t o0,
                                        uint32_t nst, uint32_t k) {
  const uint32_t i = k - (o0 & ~7u);
  if (i < nst) return reinterpret_cast<const uint16_t*>(zrow + a.cfg.logits_copy_bytes)[i];
  return a.codes[k];
}

// Warp threshold at the start of a row: the CTA-wide and request-wide bounds.
__device__ __forceinline__ void row_thresholds(WarpBuf& wb, SelCtl* ctl, unsigned long long req) {
  const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
  if (c > wb.thr) wb.thr = c;
  if (req > wb.thr) wb.thr = req;
}

// Copies a row of up to 8 KB from its stage into registers (vector lane + 32k
// in x[k]); entries past V become -inf.
template <int BF16>
__device__ __forceinline__ void copy_row_regs(const uint8_t* zrow, int V, int lane,
                                              uint4 (&x)[kRegVecs]) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  const int nvec = (V + kPerVec - 1) / kPerVec;
  const uint4* q = reinterpret_cast<const uint4*>(zrow);
  const uint4 ninf = BF16 ? make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u)
                          : make_uint4(0xFF800000u, 0xFF800000u, 0xFF800000u, 0xFF800000u);
  if (nvec == 32 * kRegVecs && V % kPerVec == 0) {  // a full 8 KB row: plain loads
    Unrolled<kRegVecs>::run([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      x[k] = q[lane + 32 * k];
    });
    return;
  }
  const int tail = V % kPerVec;
  const int vt = tail ? nvec - 1 : -1;
  Unrolled<kRegVecs>::run([&](auto kc) {
    constexpr int k = decltype(kc)::value;
    const int v = lane + 32 * k;
    x[k] = v < nvec ? q[v] : ninf;
    if (v == vt) vec_cut<BF16>(x[k], tail);
  });
}

// Children at or above the threshold in a register row (dense level or no
// trie): byte k of the packed hits holds the bits of this lane's vector k
// (lane + 32k) whose code is a valid child with z >= zthr. Only vectors whose
// largest logit reaches the threshold look at the mask. Returns whether any
// lane of the warp has a hit.
// GUM: a hit is a candidate whose perturbed logit z + T*G reaches zthr; the
// draw is made only for codes whose z + T*kGumbelMax does (r, b: the row's
// request and parent slot, the draw's counter).
template <int BF16, bool FULL, int GUM = 0>
__device__ __forceinline__ bool reg_hits(const StepArgs& a, const uint4 (&x)[kRegVecs], int nvec,
                                         float zthr, const uint32_t* wmask, int lane, int part,
                                         int nparts, uint32_t (&hp)[kRegVecs / 4], int r = 0,
                                         uint32_t b = 0) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  const bool dense = wmask != nullptr;
  const float gm = GUM ? a.gumbel_T * kGumbelMax : 0.f;
  auto hit = [&](float z, int code) -> bool {
    if constexpr (GUM) return z + gm >= zthr && z + gumbel_noise(a, r, b, code) >= zthr;
    return z >= zthr;
  };
  auto bulk = [&](float vmax) -> bool {  // may a code of the vector reach zthr?
    if constexpr (GUM) return vmax + gm >= zthr;
    return vmax >= zthr;
  };
#pragma unroll
  for (int i = 0; i < kRegVecs / 4; ++i) hp[i] = 0u;
  if (dense) {
    // Masked rows: most vectors hold no valid child, so the mask decides
    // first (one shared byte per vector), and only the valid codes of the
    // remaining vectors are compared.
    unsigned vm[kRegVecs];
#pragma unroll
    for (int k = 0; k < kRegVecs; ++k) {
      const int v = lane + 32 * k;
      const bool mine = FULL || (32 * k < nvec && (k % nparts) == part && v < nvec);
      vm[k] = !mine ? 0u
                    : BF16 ? static_cast<unsigned>(reinterpret_cast<const uint8_t*>(wmask)[v])
                           : (wmask[v >> 3] >> ((v & 7) * 4)) & 0xFu;
      if (!FULL && a.V - v * kPerVec < kPerVec) vm[k] &= (1u << (a.V - v * kPerVec)) - 1u;
    }
    Unrolled<kRegVecs>::run([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      unsigned valid = vm[k];
      if (valid && bulk(vec_max<BF16>(x[k]))) {
        unsigned bits = 0u;
        while (valid) {
          const int j = __ffs(valid) - 1;
          valid &= valid - 1u;
          if (hit(vec_elem<BF16>(x[k], j), (lane + 32 * k) * kPerVec + j)) bits |= 1u << j;
        }
        hp[k >> 2] |= bits << ((k & 3) * 8);
      }
    });
  } else {
    Unrolled<kRegVecs>::run([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      const int v = lane + 32 * k;
      const bool mine = FULL || (32 * k < nvec && (k % nparts) == part && v < nvec);
      if (mine && bulk(vec_max<BF16>(x[k]))) {
        const int cb = v * kPerVec;
        unsigned valid = (1u << kPerVec) - 1u;
        if (!FULL && a.V - cb < kPerVec) valid &= (1u << (a.V - cb)) - 1u;
        unsigned bits = 0u;
#pragma unroll
        for (int j = 0; j < kPerVec; ++j)
          if (((valid >> j) & 1u) && hit(vec_elem<BF16>(x[k], j), cb + j)) bits |= 1u << j;
        hp[k >> 2] |= bits << ((k & 3) * 8);
      }
    });
  }
  return __any_sync(kFull, (hp[0] | hp[1] | hp[2] | hp[3]) != 0u);
}

// Counts the hits in the CTA histogram and/or offers them to the warp buffer
// (mode); when offering, a hit that falls below a threshold raised meanwhile
// is dropped. The logits of the hits are read from zrow: the row in global
// memory (or its stage, while that is held). One body out of line for the
// three modes: these
// paths run for a minority of rows, so their code is shared (it stays warm in
// the instruction cache) and the caller hands over no register copy of the
// row (the hit bits are all it needs). The warp buffer goes in by value and
// its new state comes back.
enum TakeMode { kTakeBinOffer = 0, kTakeBin = 1, kTakeOffer = 2 };

struct TakeOut {
  uint64_t thr;
  int count;
  int binned;
};

// GUM: every hit's logit is perturbed by its own draw before it is tested and
// keyed (the same draw as in reg_hits).
template <int BF16, int GUM = 0>
__device__ __noinline__ TakeOut take_hits(const StepArgs& a, const uint8_t* zrow, uint32_t h0,
                                          uint32_t h1, uint32_t h2, uint32_t h3,
                                          const uint32_t* wmask, uint32_t* wprefix, RowCtx c,
                                          float zthr, WarpBuf wb, SelCtl* ctl, ThrSinks sinks,
                                          int lane, int mode) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  constexpr int kBatch = 4;
  const bool dense = wmask != nullptr;  // node ids by rank in the child bitmap
  if (dense && mode != kTakeBin)
    dense_prefix(wmask, a.layout == SIDBEAM_LAYOUT_DENSE ? a.mask_words : (a.V + 31) / 32,
                 wprefix, lane);
  uint32_t hb[kRegVecs / 4] = {h0, h1, h2, h3};
  while (__any_sync(kFull, (hb[0] | hb[1] | hb[2] | hb[3]) != 0u)) {
    int code[kBatch];
    float z[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      int bit = -1;
#pragma unroll
      for (int w = kRegVecs / 4 - 1; w >= 0; --w)  // lowest set bit over the 128
        if (hb[w]) bit = 32 * w + __ffs(hb[w]) - 1;
      if (bit >= 0) hb[bit >> 5] &= hb[bit >> 5] - 1u;
      code[u] = bit < 0 ? -1 : (lane + 32 * (bit >> 3)) * kPerVec + (bit & 7);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) z[u] = code[u] >= 0 ? elem<BF16>(zrow, code[u]) : 0.f;
    if constexpr (GUM) {
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (code[u] >= 0) z[u] += gumbel_noise(a, c.r, c.b, code[u]);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const bool has = code[u] >= 0 && (mode == kTakeBin || z[u] >= zthr);
      if (!__any_sync(kFull, has)) continue;
      const float score = c.s + (z[u] - c.lse);
      if (mode != kTakeOffer)
        warp_bin(ctl->hist, has, score_bin(score, c.C), wb.binned, &ctl->hist_total);
      if (mode != kTakeBin) {
        const int32_t node = (has && dense) ? dense_child(wmask, wprefix, c.o0, code[u]) : -1;
        warp_offer_nc(wb, has, make_key(score, c.idx0 + static_cast<uint32_t>(code[u])), node,
                      static_cast<uint32_t>(a.n), lane, sinks);
        zthr = zthreshold(wb.thr, c.s, c.lse);
      }
    }
  }
  return TakeOut{wb.thr, wb.count, wb.binned};
}


// Child bitmap of a CSR node in the warp's mask copy: bit c set for every
// child code c (child ids o0 .. o1-1, codes ascending, so the rank of a code
// among the set bits is its id minus o0). Codes are read 16 bytes at a time
// from an 8-aligned start (the code array is padded), four loads per lane
// in flight. Warp-collective.
__device__ __forceinline__ void csr_bitmap(const StepArgs& a, uint32_t o0, uint32_t o1,
                                           int words, uint32_t* wmask, int lane) {
  for (int i = lane; i < words; i += 32) wmask[i] = 0u;
  __syncwarp();
  const uint32_t a0 = o0 & ~7u;
  const uint32_t nv = (o1 - a0 + 7u) / 8u;
  const uint4* src = reinterpret_cast<const uint4*>(a.codes + a0);
  for (uint32_t v0 = lane; v0 < nv; v0 += 32u * 4u) {
    uint4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t v = v0 + 32u * u;
      q[u] = v < nv ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t v = v0 + 32u * u;
      const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t id = a0 + v * 8u + e;
        if (v < nv && id >= o0 && id < o1) {
          const uint32_t code = (w[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu;
          atomicOr(&wmask[code >> 5], 1u << (code & 31));
        }
      }
    }
  }
  __syncwarp();
}

// Candidate walk of a row in place in its stage (rows over 8 KB, CSR rows with
// more children than one 32-lane batch per warp, dense rows with very many
// children). wmask: the warp's mask copy (room for a V-bit row).
constexpr uint32_t kCsrBitmapMin = 192;  // CSR rows with more children use a bitmap
// Counts a CTA keeps before it moves them to the request's histogram.
constexpr unsigned kPushAfter = 64;
__device__ __noinline__ uint64_t push_histogram(const StepArgs& a, SelCtl* ctl, int r, float C,
                                                uint64_t thr, ThrSinks sinks, int lane);
// r: the row's request; multi: the request is split over several CTAs (the
// count pass then also pushes, so that the offer pass sees their counts).
// GUM: Gumbel top-k (see gumbel_noise): every candidate's logit is replaced
// by z + T*G before its key is formed, and the bulk tests (row max, vector
// max) allow for the largest possible T*G.
template <int BF16, int GUM = 0>
__device__ void smem_walk(const StepArgs& a, const uint8_t* zrow, const RowCtx& c, float rmax,
                          float zthr, WarpBuf& wb, SelCtl* ctl, uint32_t* wprefix,
                          uint32_t* wmask, const ThrSinks& sinks, int lane, int part,
                          int nparts, int r, bool multi) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  const float gm = GUM ? a.gumbel_T * kGumbelMax : 0.f;  // bound on T*G
  auto zeff = [&](float z, int code) -> float {
    if constexpr (GUM) return z + gumbel_noise(a, c.r, c.b, code);
    return z;
  };
  if (rmax + gm < zthr) return;  // even the row's largest logit cannot reach the threshold
  const uint32_t* mrow = nullptr;  // valid-child bitmap (null: every code is valid)
  int words = 0;
  if (a.layout == SIDBEAM_LAYOUT_CSR) {
    if (c.o1 - c.o0 <= kCsrBitmapMin) {  // all codes are staged behind the row
      const uint32_t nst = csr_staged(a, c.o0, c.o1);
      const uint32_t k_step = static_cast<uint32_t>(32 * nparts);
      for (uint32_t k0 = c.o0 + static_cast<uint32_t>(part * 32); k0 < c.o1; k0 += k_step) {
        const uint32_t k = k0 + lane;
        const bool in = k < c.o1;
        const int code = in ? csr_code(a, zrow, c.o0, nst, k) : 0;
        const float z = in ? zeff(elem<BF16>(zrow, code), code) : 0.f;
        const bool ok = in && z >= zthr;
        if (!__any_sync(kFull, ok)) continue;
        const float score = c.s + (z - c.lse);
        warp_bin(ctl->hist, ok, score_bin(score, c.C), wb.binned, &ctl->hist_total);
        warp_offer_nc(wb, ok, make_key(score, c.idx0 + static_cast<uint32_t>(code)),
                      static_cast<int32_t>(k), static_cast<uint32_t>(a.n), lane, sinks);
        zthr = zthreshold(wb.thr, c.s, c.lse);
      }
      return;
    }
    words = (a.V + 31) / 32;
    csr_bitmap(a, c.o0, c.o1, words, wmask, lane);
    mrow = wmask;
  } else if (a.layout == SIDBEAM_LAYOUT_DENSE) {
    mrow = reinterpret_cast<const uint32_t*>(zrow + a.cfg.logits_copy_bytes);
    words = a.mask_words;
  }
  // Many children: two passes. Count every child at or above the threshold,
  // raise the threshold from the histogram, then offer only what still
  // reaches it.
  const int nvec_all = (a.V + kPerVec - 1) / kPerVec;
  const uint4* q = reinterpret_cast<const uint4*>(zrow);
  bool have_prefix = false;
  for (int pass = 0; pass < 2; ++pass) {
    for (int v0 = part * 32; v0 < nvec_all; v0 += 32 * nparts) {
      const int v = v0 + lane;
      unsigned bits = 0u;
      float zp[kPerVec];  // effective logits of the hits (GUM)
      const uint4 x = v < nvec_all ? q[v] : make_uint4(0u, 0u, 0u, 0u);
      if (v < nvec_all && vec_max<BF16>(x) + gm >= zthr) {
        const int cb = v * kPerVec;
        unsigned valid = (1u << kPerVec) - 1u;
        if (mrow) valid = (mrow[cb >> 5] >> (cb & 31)) & ((1u << kPerVec) - 1u);
        if (a.V - cb < kPerVec) valid &= (1u << (a.V - cb)) - 1u;
#pragma unroll
        for (int j = 0; j < kPerVec; ++j) {
          if constexpr (GUM) {
            zp[j] = 0.f;
            if (((valid >> j) & 1u) && vec_elem<BF16>(x, j) + gm >= zthr) {
              zp[j] = zeff(vec_elem<BF16>(x, j), cb + j);
              if (zp[j] >= zthr) bits |= 1u << j;
            }
          } else {
            if (((valid >> j) & 1u) && vec_elem<BF16>(x, j) >= zthr) bits |= 1u << j;
          }
        }
      }
      if (pass == 0) {  // count the hits of this vector in one go
#pragma unroll
        for (int j = 0; j < kPerVec; ++j)
          if ((bits >> j) & 1u) {
            const float z = GUM ? zp[j] : vec_elem<BF16>(x, j);
            atomicAdd(&ctl->hist[score_bin(c.s + (z - c.lse), c.C)], 1u);
          }
        const int cnt = static_cast<int>(__reduce_add_sync(kFull, __popc(bits)));
        wb.binned += cnt;
        if (lane == 0 && cnt) atomicAdd(&ctl->hist_total, static_cast<unsigned>(cnt));
        continue;
      }
      if (!__any_sync(kFull, bits != 0u)) continue;
      if (mrow && !have_prefix) {
        dense_prefix(mrow, words, wprefix, lane);
        have_prefix = true;
      }
      while (__any_sync(kFull, bits != 0u)) {
        const int j = bits ? __ffs(bits) - 1 : 0;
        const int code = v * kPerVec + j;
        const float z = (GUM && bits) ? zeff(vec_elem<BF16>(x, j), code) : vec_elem<BF16>(x, j);
        const bool has = bits != 0u && z >= zthr;
        bits &= bits - 1u;
        const float score = c.s + (z - c.lse);
        const int32_t node = (has && mrow) ? dense_child(mrow, wprefix, c.o0, code) : -1;
        warp_offer_nc(wb, has, make_key(score, c.idx0 + static_cast<uint32_t>(code)), node,
                      static_cast<uint32_t>(a.n), lane, sinks);
        zthr = zthreshold(wb.thr, c.s, c.lse);
      }
    }
    if (pass == 0) {
      __syncwarp();
      refresh_thr(wb, ctl, static_cast<uint32_t>(a.n), c.C, lane, sinks);
      if (multi && *reinterpret_cast<volatile unsigned*>(&ctl->hist_total) >= kPushAfter)
        wb.thr = push_histogram(a, ctl, r, c.C, wb.thr, sinks, lane);
      zthr = zthreshold(wb.thr, c.s, c.lse);
    }
  }
}

// Moves this CTA's histogram counts into request r's global histogram and
// raises the shared bounds from the global one, which holds every CTA's
// pushed counts (warp-collective; one warp of the CTA at a time, the others
// skip). Counts move by atomic exchange, so each candidate stays counted
// exactly once; the segment end pushes what is left. Only for requests split
// over several CTAs (a CTA that holds a whole request keeps its histogram).
__device__ __noinline__ uint64_t push_histogram(const StepArgs& a, SelCtl* ctl, int r, float C,
                                                uint64_t thr, ThrSinks sinks, int lane) {
  int got = 0;
  if (lane == 0) got = atomicCAS(&ctl->push_lock, 0, 1) == 0 ? 1 : 0;
  if (!__shfl_sync(kFull, got, 0)) return thr;
  uint32_t* gh = a.ghist + static_cast<size_t>(r) * kHistBins;
  for (int b = lane; b < kHistBins; b += 32) {
    const uint32_t c = atomicExch(&ctl->hist[b], 0u);
    if (c) atomicAdd(gh + b, c);
  }
  if (lane == 0) atomicExch(&ctl->hist_total, 0u);
  __threadfence();
  uint4 h[8];
  const uint4* g4 = reinterpret_cast<const uint4*>(gh) + lane * 8;
#pragma unroll
  for (int j = 0; j < 8; ++j) h[j] = __ldcg(g4 + j);
  const uint64_t hb = hist_bound_regs(h, static_cast<uint32_t>(a.n), C, lane);
  if (hb > thr) {
    thr = hb;
    publish_thr(hb, lane, sinks);
  }
  __syncwarp();
  if (lane == 0) atomicExch(&ctl->push_lock, 0);
  return thr;
}

// refresh_thr with the histogram scan out of line (the scan runs for a
// minority of rows; the cheap test stays inline).
__device__ __noinline__ uint64_t refresh_scan(SelCtl* ctl, uint32_t n, float C, uint64_t thr,
                                              ThrSinks sinks, int lane) {
  WarpBuf wb{nullptr, nullptr, nullptr, 0, 0, thr, kRefreshAfter};
  refresh_thr(wb, ctl, n, C, lane, sinks);
  return wb.thr;
}
__device__ __forceinline__ void refresh_row(WarpBuf& wb, SelCtl* ctl, uint32_t n, float C,
                                            int lane, const ThrSinks& sinks) {
  if ((wb.binned < kRefreshAfter && wb.thr != 0ull) ||
      *reinterpret_cast<volatile unsigned*>(&ctl->hist_total) < n) {
    const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
    if (c > wb.thr) wb.thr = c;
    return;
  }
  wb.binned = 0;
  wb.thr = refresh_scan(ctl, n, C, wb.thr, sinks, lane);
}

// Histogram reference of request r: the largest finite parent score of the
// request (every child score is at most its parent's score), the same value
// in every CTA. Two slots alternate so that one can be cleared while the
// other is read. All team threads call it.
__device__ __forceinline__ float finite_or_ninf(float x) {
  return (x > __int_as_float(0xFF800000) && x < __int_as_float(0x7F800000))
             ? x
             : __int_as_float(0xFF800000);
}
// The reduction of the per-thread maxima m over the team.
__device__ __forceinline__ float segment_ref_finish(const Team& t, SelCtl* ctl, int slot, float m) {
  m = warp_max(m);
  if (t.lane == 0 && m > __int_as_float(0xFF800000)) atomicMax(&ctl->ref_ord[slot], ord_f32(m));
  team_sync(t);
  const unsigned o = *reinterpret_cast<volatile unsigned*>(&ctl->ref_ord[slot]);
  if (t.tid == 0) ctl->ref_ord[slot ^ 1] = 0u;
  return o ? unord_f32(o) : 0.f;
}
__device__ __forceinline__ float segment_ref(const StepArgs& a, const Team& t, SelCtl* ctl, int r,
                                             int slot) {
  float m = __int_as_float(0xFF800000);
  const float* ps = a.parent_scores + static_cast<int64_t>(r) * a.B_in;
  for (int i = t.tid; i < a.B_in; i += t.T) m = fmaxf(m, finite_or_ninf(ps[i]));
  return segment_ref_finish(t, ctl, slot, m);
}

// --------------------------------------------------------------- segment end
// Once per segment, out of line (away from the per-row loop). The warp buffer
// goes in by value so that the caller's copy stays in registers; the caller
// empties its own copy afterwards.
template <int GUM>
__device__ __noinline__ bool segment_end(const StepArgs& a, Team team, WarpBuf wb, SelCtl* ctl,
                                         uint64_t* wkeys, int32_t* wvals, uint32_t* whist,
                                         uint32_t* cta_hist, uint8_t* stages, int direct_cap,
                                         int cur_r, int r_last, float C) {
  const StepConfig& cfg = a.cfg;
  FlushArgs f;
  f.n = a.n;
  f.r = cur_r;
  f.k = static_cast<int>(blockIdx.x) - a.part.first_cta(cur_r);
  f.G = a.part.contributors(cur_r);
  f.maxG = a.part.maxG;
  f.pcap = partial_cap(a.n);
  f.part_keys = a.part_keys;
  f.part_vals = a.part_vals;
  f.part_count = a.part_count;
  f.tickets = a.tickets;
  f.request_thr = a.request_thr;
  f.ghist = a.ghist;
  f.C = C;
  f.wkeys = wkeys;
  f.cw = cfg.Cw;
  f.sort_keys = wkeys;
  f.sort_vals = wvals;
  f.sort_cap = cfg.W * cfg.Cw;
  f.radix_hist = cta_hist;
  f.wvals = wvals;
  f.rank_P = whist;
  f.rank_cur = whist + kHistBins;
  // The stages are idle only at the CTA's last segment (every ring is empty).
  const bool last = cur_r == r_last;
  f.direct_keys = last ? reinterpret_cast<uint64_t*>(stages) : nullptr;
  f.direct_vals =
      last ? reinterpret_cast<int32_t*>(stages + static_cast<size_t>(direct_cap) * 8) : nullptr;
  f.direct_cap = last ? direct_cap : 0;
  if constexpr (GUM) {
    const GumbelWriter writer{a.out_scores, a.out_parent, a.out_code, a.out_node, a.n,
                              static_cast<uint32_t>(a.V), a.logits, a.row_bytes, a.bf16,
                              a.parent_scores, a.row_lse, a.B_in, a.out_width};
    return segment_flush(team, wb, ctl, f, writer);
  } else {
    const StepWriter writer{a.out_scores, a.out_parent, a.out_code, a.out_node, a.n,
                            static_cast<uint32_t>(a.V), a.out_width};
    return segment_flush(team, wb, ctl, f, writer);
  }
}

// --------------------------------------------------------------- threshold seeding
// The first row of every warp starts without a threshold, and together these
// rows hold most of a step's candidates at levels where nodes have many
// children. So before the per-row loop each warp counts every valid child of
// its first row into a scratch histogram (exact scores, all lanes busy: no
// per-candidate warp work); once all have counted, the n-th best of these
// candidates bounds the request's n-th best from below and becomes the CTA's
// and the request's first threshold. The scratch is not the segment
// histogram, whose counts must match the candidates offered. Warp-collective;
// zrow: the row's stage.
// GUM: the scores counted are the perturbed ones (each child's own draw; r, b:
// the row's request and parent slot), so the bound holds for perturbed keys.
template <int BF16, int GUM = 0>
__device__ void seed_count(const StepArgs& a, const uint8_t* zrow, float s, float lse, uint32_t o0,
                           uint32_t o1, float C, uint32_t* shist, int lane, int r = 0,
                           uint32_t b = 0) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  auto zeff = [&](float z, int code) -> float {
    if constexpr (GUM) return z + gumbel_noise(a, r, b, code);
    return z;
  };
  if (a.layout == SIDBEAM_LAYOUT_CSR) {
    const uint32_t nst = csr_staged(a, o0, o1);
    for (uint32_t k = o0 + lane; k < o1; k += 32u) {
      const int code = csr_code(a, zrow, o0, nst, k);
      const float z = zeff(elem<BF16>(zrow, code), code);
      atomicAdd(&shist[score_bin(s + (z - lse), C)], 1u);
    }
    return;
  }
  const uint32_t* mrow = a.layout == SIDBEAM_LAYOUT_DENSE
                             ? reinterpret_cast<const uint32_t*>(zrow + a.cfg.logits_copy_bytes)
                             : nullptr;
  const uint4* q = reinterpret_cast<const uint4*>(zrow);
  const int nvec = (a.V + kPerVec - 1) / kPerVec;
  for (int v = lane; v < nvec; v += 32) {
    const uint4 x = q[v];
    const int cb = v * kPerVec;
    unsigned valid = (1u << kPerVec) - 1u;
    if (mrow) valid = (mrow[cb >> 5] >> (cb & 31)) & ((1u << kPerVec) - 1u);
    if (a.V - cb < kPerVec) valid &= (1u << (a.V - cb)) - 1u;
#pragma unroll
    for (int j = 0; j < kPerVec; ++j)
      if ((valid >> j) & 1u)
        atomicAdd(&shist[score_bin(s + (zeff(vec_elem<BF16>(x, j), cb + j) - lse), C)], 1u);
  }
}

// The Gumbel count out of line (the draws' registers stay out of the kernel's
// own allocation).
template <int BF16>
__device__ __noinline__ void seed_count_gumbel(const StepArgs& a, const uint8_t* zrow, float s,
                                               float lse, uint32_t o0, uint32_t o1, float C,
                                               uint32_t* shist, int lane, int r, uint32_t b) {
  seed_count<BF16, 1>(a, zrow, s, lse, o0, o1, C, shist, lane, r, b);
}

// --------------------------------------------------------------- kernel
template <int BF16, int REG, int GUM = 0>
__global__ void __launch_bounds__(REG ? kMaxStepWarpsReg * 32 : kMaxStepWarps * 32, 1)
    beam_step_kernel(const __grid_constant__ StepArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kPerVec = BF16 ? 8 : 4;
  const StepConfig& cfg = a.cfg;
  SelCtl* ctl = reinterpret_cast<SelCtl*>(smem + cfg.off_ctl);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + cfg.off_bars);
  uint32_t* cta_hist = reinterpret_cast<uint32_t*>(smem + cfg.off_chist);
  uint32_t* whist = reinterpret_cast<uint32_t*>(smem + cfg.off_whist);
  uint32_t* wprefix = reinterpret_cast<uint32_t*>(smem + cfg.off_wprefix);
  uint32_t* wmask = reinterpret_cast<uint32_t*>(smem + cfg.off_wmask);
  uint8_t* stages = smem + cfg.off_stage;
  uint64_t* wkeys = reinterpret_cast<uint64_t*>(smem + cfg.off_wkeys);
  int32_t* wvals = reinterpret_cast<int32_t*>(smem + cfg.off_wvals);

  const int W = cfg.W, S = cfg.S;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Team team{static_cast<int>(threadIdx.x), W * 32, warp, lane, W};

  int64_t lo, hi;
  a.part.range(static_cast<int>(blockIdx.x), lo, hi);
  RowSeq q;
  a.part.rows(static_cast<int>(blockIdx.x), a.coop ? 0 : warp, a.coop ? 1 : W, q.first, q.stride,
              q.count);
  const int part = a.coop ? warp : 0;
  const int nparts = a.coop ? W : 1;

  Ring g{};
  g.stages = stages + static_cast<size_t>(warp) * S * cfg.stage_bytes;
  g.full = bars + warp * S;
  g.S = S;
  const uint64_t pol = policy_evict_first();

  // 0. Programmatic dependent launch: the next launch on the stream may start
  //    its own set-up now; this grid touches no global memory before the grid
  //    it depends on (the previous step, which wrote the parents and cleared
  //    the workspace counters) has completed and its writes are visible.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // 1. This warp's barriers, and the logits of its first S rows, before any
  //    parent data is known (the rest of each stage follows below).
  if (lane == 0) {
    for (int k = 0; k < S; ++k) mbar_init(&g.full[k], 1);
    fence_mbar_init();
  }
  __syncwarp();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int spec = q.count < S ? q.count : S;
  if (lane == 0) {
    for (int k = 0; k < spec; ++k) {
      mbar_expect_tx(&g.full[k], static_cast<uint32_t>(cfg.logits_copy_bytes));
      bulk_copy_g2s(g.stages + static_cast<size_t>(k) * cfg.stage_bytes,
                    a.logits + q.row(k) * a.row_bytes,
                    static_cast<uint32_t>(cfg.logits_copy_bytes), &g.full[k], pol);
    }
  }
  MetaBatch mb;
  load_meta(a, q, 0, lane, mb);
  // Rows handed out from a shared table (the CTA's sequence; entries below
  // W * S are the warps' first rows, issued above).
  RowSeq cq;
  a.part.rows(static_cast<int>(blockIdx.x), 0, 1, cq.first, cq.stride, cq.count);
  const bool shared_rows = !a.coop && cq.count <= kMetaRows;
  uint4* meta = reinterpret_cast<uint4*>(smem + cfg.off_meta);

  // 2. Trie data of the first rows, now that their parents are known.
  for (int k = 0; k < spec; ++k) {
    const int live = (mb.live >> k) & 1u;
    const float s = __shfl_sync(kFull, mb.s, k);
    const int32_t p = __shfl_sync(kFull, mb.p, k);
    const uint32_t o0 = __shfl_sync(kFull, mb.o0, k);
    const uint32_t o1 = __shfl_sync(kFull, mb.o1, k);
    if (lane == k) {
      g.st_seq = shared_rows ? warp + W * k : k;
      g.st_live = live;
      g.st_s = s;
      g.st_p = p;
      g.st_o0 = o0;
      g.st_o1 = o1;
    }
    if (lane == 0) {
      const uint32_t ex = live ? extra_bytes(a, o0, o1) : 0u;
      mbar_arrive_expect_tx(&g.full[k], ex);
      if (ex) copy_extra(a, g.stages + static_cast<size_t>(k) * cfg.stage_bytes, &g.full[k], p, o0,
                         ex, pol);
    }
  }
  g.issued = spec;
  g.ip = spec;

  // 3. CTA state, the shared row table, and the first segment's histogram
  //    reference.
  if (threadIdx.x == 0) {
    ctl->cta_thr = 0ull;
    ctl->abort_flag = 0;
    ctl->counter = 0;
    ctl->ref_ord[0] = 0u;
    ctl->ref_ord[1] = 0u;
    ctl->hist_total = 0u;
    ctl->push_lock = 0;
    ctl->next_row = W * S;
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) {
    ctl->hist[i] = 0u;
    whist[i] = 0u;  // seeding scratch (the warps' select scratch later)
  }
  __syncthreads();
  const int r_first = static_cast<int>(lo / a.B_in);
  const int r_last = static_cast<int>((hi - 1) / a.B_in);
  int ref_slot = 0;
  // The shared table (parent data of every row, as load_meta reads it; dead
  // rows get score -inf) and the first segment's reference, their loads in
  // flight together; the reference's barrier also publishes the table.
  float mref = __int_as_float(0xFF800000);
  {
    const float* ps = a.parent_scores + static_cast<int64_t>(r_first) * a.B_in;
    const int T = static_cast<int>(blockDim.x);
    const int nt = shared_rows ? cq.count : 0;
    for (int i0 = threadIdx.x; i0 < (nt > a.B_in ? nt : a.B_in); i0 += T) {
      float sj = __int_as_float(0xFF800000);
      int32_t pj = 0;
      int64_t row = 0;
      if (i0 < nt) {
        row = cq.row(i0);
        sj = a.parent_scores[row];
        if (a.layout) pj = a.parent_nodes[row];
      }
      if (i0 < a.B_in) mref = fmaxf(mref, finite_or_ninf(ps[i0]));
      if (i0 < nt) {
        uint32_t o0 = 0u, o1 = 0u;
        if (a.layout && (pj < 0 || static_cast<int64_t>(pj) >= a.n_parent)) {
          if (pj >= 0 && sj != __int_as_float(0xFF800000)) atomicOr(a.status, kStatusBadNode);
          sj = __int_as_float(0xFF800000);
        } else if (a.layout && sj != __int_as_float(0xFF800000)) {
          o0 = a.off[pj];
          o1 = a.off[pj + 1];
        }
        meta[i0] = make_uint4(__float_as_uint(sj), static_cast<uint32_t>(pj), o0, o1);
      }
    }
  }
  float C = segment_ref_finish(team, ctl, ref_slot, mref);
  if constexpr (GUM) C += a.gumbel_T * kGumbelMax;  // perturbed scores reach this high
  if (shared_rows) q = cq;  // sequence entries are CTA entries from here on

  // 3b. Threshold seeding from the first row of every warp that belongs to
  //     the first request, when those rows have more than n children in all
  //     (read from the shared table). Gumbel steps count perturbed scores.
  if (shared_rows) {
    const int64_t end_first = static_cast<int64_t>(r_first + 1) * a.B_in;  // rows of r_first
    const int nfirst = cq.count < W ? cq.count : W;
    uint32_t nch = 0u;
    for (int j = lane; j < nfirst; j += 32) {
      const uint4 m = meta[j];
      if (m.x != 0xFF800000u && cq.row(j) < end_first)
        nch += a.layout ? m.w - m.z : static_cast<uint32_t>(a.V);
    }
    if (warp_sum_u(nch) > static_cast<uint32_t>(a.n)) {  // the same in every warp
      if (warp < cq.count && meta[warp].x != 0xFF800000u && cq.row(warp) < end_first &&
          bounded_wait(&g.full[0], 0u, &ctl->abort_flag, a.status, kStatusTimeout)) {
        const uint4 m = meta[warp];  // the warp's first row: CTA entry `warp`, stage 0
        int r0 = 0;
        uint32_t b0 = 0u;
        if constexpr (GUM) {  // the draws' counter
          const int64_t row0 = cq.row(warp);
          r0 = static_cast<int>(row0 / a.B_in);
          b0 = static_cast<uint32_t>(row0 - static_cast<int64_t>(r0) * a.B_in);
        }
        float rmax0, lse0;
        row_stats<BF16>(g.stages, a.V, lane, rmax0, lse0);
        if constexpr (GUM)
          seed_count_gumbel<BF16>(a, g.stages, __uint_as_float(m.x), lse0, m.z, m.w, C, whist,
                                  lane, r0, b0);
        else
          seed_count<BF16>(a, g.stages, __uint_as_float(m.x), lse0, m.z, m.w, C, whist, lane);
      }
      team_sync(team);
      if (warp == 0) {
        const uint64_t hb = hist_bound(whist, static_cast<uint32_t>(a.n), C, lane);
        if (lane == 0 && hb) {
          atomicMax(&ctl->cta_thr, static_cast<unsigned long long>(hb));
          atomicMax(a.request_thr + r_first, static_cast<unsigned long long>(hb));
        }
      }
      team_sync(team);  // the scratch goes back to the warps
    }
  }

  WarpBuf wb{wkeys + static_cast<size_t>(warp) * cfg.Cw,
             wvals + static_cast<size_t>(warp) * cfg.Cw, whist + warp * 256, cfg.Cw, 0, 0ull, 0};
  uint32_t* my_prefix = wprefix + warp * cfg.prefix_words;
  uint32_t* my_mask = wmask + warp * cfg.prefix_words;
  const int direct_cap = (W * S * cfg.stage_bytes / 12) & ~1;

  // The request's shared bound as last read (after each row is issued).
  unsigned long long req_pref = 0ull;
  int req_pref_r = -1;
  // Row skipping needs a bound of the rows' own request: CTAs that hold rows
  // of one request only.
  const bool skipping = !GUM && a.skip_rows && a.part.grouped;
  auto refill = [&]() {
    uint64_t bound = 0ull;
    if (skipping) {
      bound = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
      if (req_pref_r >= 0 && req_pref > bound) bound = req_pref;
    }
    if (shared_rows)
      ring_refill_shared(a, q, meta, &ctl->next_row, g, lane, pol, bound);
    else
      ring_refill(a, q, mb, g, lane, pol, bound);
  };

  // End of the segment of request cur_r (all warps, in the same order).
  int cur_r = r_first;
  auto flush = [&]() -> bool {
    const bool stop = segment_end<GUM>(a, team, wb, ctl, wkeys, wvals, whist, cta_hist, stages,
                                  direct_cap, cur_r, r_last, C);
    wb.count = 0;
    wb.thr = 0ull;
    if (stop) return true;
    if (cur_r < r_last)
      C = segment_ref(a, team, ctl, cur_r + 1, ref_slot ^= 1) +
          (GUM ? a.gumbel_T * kGumbelMax : 0.f);
    ++cur_r;
    return false;
  };

  bool wait_failed = false, stopped = false;
  while (g.consumed < g.issued) {
    const int stage = g.consumed % S;
    if (!bounded_wait(&g.full[stage], (g.consumed / S) & 1u, &ctl->abort_flag, a.status,
                      kStatusTimeout)) {
      wait_failed = true;
      break;
    }
    const int seq = __shfl_sync(kFull, g.st_seq, stage);
    const int live = __shfl_sync(kFull, g.st_live, stage);
    const float s = __shfl_sync(kFull, g.st_s, stage);
    const uint32_t o0 = __shfl_sync(kFull, g.st_o0, stage);
    const uint32_t o1 = __shfl_sync(kFull, g.st_o1, stage);
    const uint8_t* zrow = g.stages + static_cast<size_t>(stage) * cfg.stage_bytes;
    if (!live) {
      ++g.consumed;
      refill();
      continue;
    }
    const int64_t row = q.row(seq);
    const int r = static_cast<int>(row) / a.B_in;  // rows number < 2^31
    while (r > cur_r && !stopped) stopped = flush();
    if (stopped) break;

    const uint32_t b = static_cast<uint32_t>(row - static_cast<int64_t>(r) * a.B_in);
    const bool multi = a.part.contributors(r) > 1;
    RowCtx c{s, 0.f, C, b * static_cast<uint32_t>(a.V), o0, o1, r, b};
    const ThrSinks sinks{&ctl->cta_thr, a.request_thr + r};
    const unsigned long long req_now = req_pref_r == r ? req_pref : 0ull;
    const bool csr = a.layout == SIDBEAM_LAYOUT_CSR;
    const uint32_t nchild = o1 - o0;
    // Register rows: all but CSR nodes with more children than one 32-lane
    // batch per warp, and, when every warp takes every row (a CTA with fewer
    // rows than warps), dense nodes with very many children; those are walked
    // in place in their stage.
    const bool reg_row =
        REG && (csr ? nchild <= static_cast<uint32_t>(32 * nparts)
                    : (a.layout != SIDBEAM_LAYOUT_DENSE || nparts == 1 || nchild <= kHugeDense));
    if (reg_row) {
      uint4 x[kRegVecs];
      copy_row_regs<BF16>(zrow, a.V, lane, x);
      if (a.layout == SIDBEAM_LAYOUT_DENSE) {  // mask_stride is a multiple of 4 words
        const uint4* mrow = reinterpret_cast<const uint4*>(zrow + cfg.logits_copy_bytes);
        for (int i = lane; i < (a.mask_stride >> 2); i += 32)
          reinterpret_cast<uint4*>(my_mask)[i] = mrow[i];
      }
      const uint32_t ck = o0 + static_cast<uint32_t>(part * 32 + lane);
      const bool cin = csr && ck < o1;
      int ccode = 0;
      float cz = 0.f;
      if (cin) {
        ccode = csr_code(a, zrow, o0, csr_staged(a, o0, o1), ck);
        cz = elem<BF16>(zrow, ccode);
      }
      // Everything the row needs from its stage is now in registers or in the
      // warp's mask copy: the stage goes back at once, so that the next row's
      // copy overlaps this row's arithmetic (the few hit logits a walk needs
      // are read back from the row in global memory, still in L2).
      __syncwarp();
      ++g.consumed;
      refill();
      req_pref = *reinterpret_cast<volatile unsigned long long*>(a.request_thr + r);
      req_pref_r = r;

      const int nvec = (a.V + kPerVec - 1) / kPerVec;
      const bool full = nvec == 32 * kRegVecs && a.V % kPerVec == 0;
      float rmax;
      if (full)
        row_stats_reg<BF16, true>(x, nvec, lane, rmax, c.lse);
      else
        row_stats_reg<BF16>(x, nvec, lane, rmax, c.lse);
      if (GUM && lane == 0) a.row_lse[row] = c.lse;  // the writer recomputes scores from it
      row_thresholds(wb, ctl, req_now);
      float zthr = zthreshold(wb.thr, c.s, c.lse);
      if constexpr (GUM) {  // perturbed logits reach at most z + T * kGumbelMax
        if (rmax + a.gumbel_T * kGumbelMax < zthr) continue;
      } else {
        if (rmax < zthr) continue;
      }
      if (csr) {
        bool ok = cin && cz >= zthr;
        if constexpr (GUM) {
          ok = cin && cz + a.gumbel_T * kGumbelMax >= zthr;
          if (ok) cz += gumbel_noise(a, r, b, ccode);
          ok = ok && cz >= zthr;
        }
        if (!__any_sync(kFull, ok)) continue;
        const float score = c.s + (cz - c.lse);
        warp_bin(ctl->hist, ok, score_bin(score, C), wb.binned, &ctl->hist_total);
        warp_offer_nc(wb, ok, make_key(score, c.idx0 + static_cast<uint32_t>(ccode)),
                      static_cast<int32_t>(ck), static_cast<uint32_t>(a.n), lane, sinks);
      } else {
        const uint32_t* hmask = a.layout == SIDBEAM_LAYOUT_DENSE ? my_mask : nullptr;
        uint32_t hp[kRegVecs / 4];
        const bool any =
            (full && nparts == 1)
                ? reg_hits<BF16, true, GUM>(a, x, nvec, zthr, hmask, lane, part, nparts, hp, r, b)
                : reg_hits<BF16, false, GUM>(a, x, nvec, zthr, hmask, lane, part, nparts, hp, r,
                                             b);
        if (!any) continue;
        const int nhits = static_cast<int>(
            __reduce_add_sync(kFull, __popc(hp[0]) + __popc(hp[1]) + __popc(hp[2]) + __popc(hp[3])));
        const uint8_t* zg = a.logits + row * a.row_bytes;
        auto take = [&](int mode) {
          const TakeOut o = take_hits<BF16, GUM>(a, zg, hp[0], hp[1], hp[2], hp[3], hmask,
                                                 my_prefix, c, zthr, wb, ctl, sinks, lane, mode);
          wb.thr = o.thr;
          wb.count = o.count;
          wb.binned = o.binned;
        };
        if (nhits <= kOnePassHits) {
          take(kTakeBinOffer);
        } else {
          // Many hits: count them all, raise the threshold (this CTA's histogram,
          // then the request's), and offer only the hits that still reach it.
          take(kTakeBin);
          __syncwarp();
          refresh_row(wb, ctl, static_cast<uint32_t>(a.n), C, lane, sinks);
          if (multi && *reinterpret_cast<volatile unsigned*>(&ctl->hist_total) >= kPushAfter)
            wb.thr = push_histogram(a, ctl, r, C, wb.thr, sinks, lane);
          const float zthr1 = zthreshold(wb.thr, c.s, c.lse);
          if (zthr1 > zthr) zthr = zthr1;
          take(kTakeOffer);
        }
      }
      __syncwarp();
      refresh_row(wb, ctl, static_cast<uint32_t>(a.n), C, lane, sinks);
      if (multi && *reinterpret_cast<volatile unsigned*>(&ctl->hist_total) >= kPushAfter)
        wb.thr = push_histogram(a, ctl, r, C, wb.thr, sinks, lane);
    } else {
      float rmax;
      row_stats<BF16>(zrow, a.V, lane, rmax, c.lse);
      if (GUM && lane == 0) a.row_lse[row] = c.lse;  // the writer recomputes scores from it
      row_thresholds(wb, ctl, req_now);
      smem_walk<BF16, GUM>(a, zrow, c, rmax, zthreshold(wb.thr, c.s, c.lse), wb, ctl, my_prefix,
                      my_mask, sinks, lane, part, nparts, r, multi);
      __syncwarp();
      refresh_row(wb, ctl, static_cast<uint32_t>(a.n), C, lane, sinks);
      if (multi && *reinterpret_cast<volatile unsigned*>(&ctl->hist_total) >= kPushAfter)
        wb.thr = push_histogram(a, ctl, r, C, wb.thr, sinks, lane);
      ++g.consumed;
      refill();
      req_pref = *reinterpret_cast<volatile unsigned long long*>(a.request_thr + r);
      req_pref_r = r;
    }
  }

  // 4. Remaining segment ends. A warp whose wait gave up has set the abort
  //    flag; the next flush sees it in every warp and all of them stop.
  if (!stopped) {
    if (wait_failed) {
      flush();
    } else {
      while (cur_r <= r_last)
        if (flush()) break;
    }
  }
  // Copies still in flight land before the CTA's shared memory goes away.
  if (lane == 0)
    for (int k = g.consumed; k < g.issued; ++k) drain_wait(&g.full[k % S], (k / S) & 1u);
}

}  // namespace

// ------------------------------------------------------------------ host side

static int round_up(int x, int m) { return (x + m - 1) / m * m; }
static_assert(dev::kHistBins == kPlanHistBins, "the plan sizes the rank-merge scratch");

// Raise the kernel's dynamic shared-memory limit to the full budget once per
// device (kept out of the per-call path, and out of any stream capture that
// follows a first eager call).
static cudaError_t opt_in_smem(const void* fn, int which) {
  static std::mutex mu;
  static bool done[8][64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64)
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
  std::lock_guard<std::mutex> lock(mu);
  if (done[which][dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
  if (e == cudaSuccess) done[which][dev] = true;
  return e;
}

int launch_beam_step(const sidbeam_trie* trie, int step, const void* logits, int dtype, int64_t ld,
                     const float* parent_scores, const int32_t* parent_nodes, int R, int B_in,
                     int n_out, int V, float* out_scores, int32_t* out_parent, int32_t* out_code,
                     int32_t* out_node, void* workspace, size_t workspace_bytes,
                     cudaStream_t stream, unsigned flags, float gumbel_T, uint64_t gumbel_seed,
                     float* row_lse, const int32_t* out_width, size_t clear_bytes) {
  StepArgs a{};
  a.logits = static_cast<const uint8_t*>(logits);
  a.bf16 = dtype == SIDBEAM_BF16;
  const int esize = a.bf16 ? 2 : 4;
  a.row_bytes = ld * esize;
  a.V = V;
  a.parent_scores = parent_scores;
  a.parent_nodes = parent_nodes;
  a.R = R;
  a.B_in = B_in;
  a.n = n_out;
  if (trie) {
    const StepTrie& st = trie->steps[step];
    a.layout = st.layout;
    a.off = st.off;
    a.mask = st.mask;
    a.mask_words = st.mask_words;
    a.mask_stride = st.mask_stride;
    a.codes = st.codes;
    a.n_parent = st.n_parent;
  }
  a.out_scores = out_scores;
  a.out_parent = out_parent;
  a.out_code = out_code;
  a.out_node = out_node;

  a.part = make_partition(R, B_in, std::min(device_sm_count(), 640));
  const WorkspaceLayout ws = workspace_layout(R, a.part.maxG, n_out);
  if (workspace == nullptr || workspace_bytes < ws.total)
    return set_error(SIDBEAM_ERR_WORKSPACE, "beam_step: workspace of %zu bytes, need %zu",
                     workspace_bytes, ws.total);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<uint32_t*>(w + ws.status);
  a.skipped = reinterpret_cast<uint32_t*>(w + ws.status + kSkippedRowsOffset);
  a.skip_rows = (flags & SIDBEAM_STEP_SKIP_ROWS) ? 1 : 0;
  const bool gum = gumbel_T > 0.f;
  a.gumbel_T = gum ? gumbel_T : 0.f;
  a.gseed0 = static_cast<uint32_t>(gumbel_seed);
  a.gseed1 = static_cast<uint32_t>(gumbel_seed >> 32);
  a.gstep = step;
  a.row_lse = row_lse;
  a.out_width = out_width;
  a.tickets = reinterpret_cast<uint32_t*>(w + ws.tickets);
  a.request_thr = reinterpret_cast<unsigned long long*>(w + ws.request_thr);
  a.part_count = reinterpret_cast<uint32_t*>(w + ws.part_count);
  a.part_keys = reinterpret_cast<unsigned long long*>(w + ws.part_keys);
  a.part_vals = reinterpret_cast<int32_t*>(w + ws.part_vals);
  a.ghist = reinterpret_cast<uint32_t*>(w + ws.ghist);

  const bool dense = a.layout == SIDBEAM_LAYOUT_DENSE;
  const int extra = dense ? a.mask_stride * 4 : (a.layout == SIDBEAM_LAYOUT_CSR ? 512 : 0);
  // Per-warp bitmap + prefix counts: dense mask rows, and CSR nodes with many
  // children (turned into a bitmap).
  const int prefix_words = dense ? a.mask_stride
                                 : (a.layout == SIDBEAM_LAYOUT_CSR ? ((V + 31) / 32 + 3) / 4 * 4 : 0);
  const bool reg = static_cast<int64_t>(V) * esize <= 16 * 32 * kRegVecs;
  const int ctl_bytes = round_up(static_cast<int>(sizeof(dev::SelCtl)), 128);
  if (!choose_step_config(V, esize, extra, prefix_words, n_out, reg, ctl_bytes, &a.cfg) &&
      !(reg && choose_step_config(V, esize, extra, prefix_words, n_out, false, ctl_bytes,
                                  &a.cfg)))
    return set_error(SIDBEAM_ERR_INVALID_ARG,
                     "beam_step: V=%d with n_out=%d does not fit in shared memory", V, n_out);
  if (a.cfg.W > (a.cfg.reg ? kMaxStepWarpsReg : kMaxStepWarps))
    return set_error(SIDBEAM_ERR_INVALID_ARG, "beam_step: internal warp plan out of range");
  a.coop = a.part.rows_per_cta < a.cfg.W ? 1 : 0;

  const void* fns[8] = {reinterpret_cast<const void*>(&beam_step_kernel<0, 0>),
                        reinterpret_cast<const void*>(&beam_step_kernel<1, 0>),
                        reinterpret_cast<const void*>(&beam_step_kernel<0, 1>),
                        reinterpret_cast<const void*>(&beam_step_kernel<1, 1>),
                        reinterpret_cast<const void*>(&beam_step_kernel<0, 0, 1>),
                        reinterpret_cast<const void*>(&beam_step_kernel<1, 0, 1>),
                        reinterpret_cast<const void*>(&beam_step_kernel<0, 1, 1>),
                        reinterpret_cast<const void*>(&beam_step_kernel<1, 1, 1>)};
  const int which = (gum ? 4 : 0) + (a.cfg.reg ? 2 : 0) + (a.bf16 ? 1 : 0);
  cudaError_t e = opt_in_smem(fns[which], which);
  if (e != cudaSuccess) return cuda_error(e, "beam_step: cudaFuncSetAttribute");
  const dim3 grid(static_cast<unsigned>(a.part.grid));
  const dim3 block(static_cast<unsigned>(32 * a.cfg.W));
  if (clear_bytes) {  // every check has passed: the caller's counters start at zero
    e = cudaMemsetAsync(workspace, 0, clear_bytes, stream);
    if (e != cudaSuccess) return cuda_error(e, "beam_step: cudaMemsetAsync");
  }
  // Launched as a programmatic dependent of the previous kernel on the stream
  // (its launch and set-up overlap that kernel's tail; see the kernel's step 0).
  cudaLaunchConfig_t lc{};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = static_cast<size_t>(a.cfg.smem_bytes);
  lc.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  switch (which) {
    case 0: e = cudaLaunchKernelEx(&lc, beam_step_kernel<0, 0>, a); break;
    case 1: e = cudaLaunchKernelEx(&lc, beam_step_kernel<1, 0>, a); break;
    case 2: e = cudaLaunchKernelEx(&lc, beam_step_kernel<0, 1>, a); break;
    case 3: e = cudaLaunchKernelEx(&lc, beam_step_kernel<1, 1>, a); break;
    case 4: e = cudaLaunchKernelEx(&lc, beam_step_kernel<0, 0, 1>, a); break;
    case 5: e = cudaLaunchKernelEx(&lc, beam_step_kernel<1, 0, 1>, a); break;
    case 6: e = cudaLaunchKernelEx(&lc, beam_step_kernel<0, 1, 1>, a); break;
    default: e = cudaLaunchKernelEx(&lc, beam_step_kernel<1, 1, 1>, a); break;
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "beam_step: launch");
  return SIDBEAM_OK;
}

}  // namespace sidbeam
