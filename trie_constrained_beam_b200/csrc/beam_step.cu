// beam_step: one catalog-constrained expansion step for all beam rows.
//
// flashrec 0.1.0 (PyPI page), Features > Decoding ("SID constraint"): a fused
// kernel restricts every continuation to the catalog trie (dense or CSR);
// Features > Serving ("API"): deterministic top-k at temperature 0.
//
// Design (sm_100a):
//  * One CTA per SM. Rows are split evenly over CTAs; a CTA's rows may span
//    request boundaries (one "segment" per request it touches).
//  * Warp 0 is the producer: it reads each row's parent score / node and, for
//    live rows only, issues untiled bulk copies (cp.async.bulk, TMA engine) of
//    the logits row and of the node's trie data -- the bitmask row at dense
//    levels, the child-code range at CSR levels -- into a ring of S
//    shared-memory stages that complete on mbarriers.
//  * Warps 1..W are consumers. They claim ring items in order. A row of up to
//    8 KB is copied into registers together with what the candidate walk needs
//    from the stage, and the stage goes back to the producer at once; larger
//    rows are worked on in place. The row max and sum of exp over the FULL
//    codebook give lse = m + log(sum) (fp32, packed f32x2 arithmetic, warp
//    shuffles); then the node's children are walked twice: first counted in
//    the CTA's score histogram, then, above the raised threshold, offered as
//    key(score = s + (z_c - lse), idx = b*V + c) to the warp's top-n buffer.
//  * At the end of each segment the consumer warps run the CTA merge and, in
//    the last contributing CTA of the request, the request merge (topn.cuh).
// The logits are read exactly once from HBM.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"
#include "launch.h"
#include "topn.cuh"

namespace sidbeam {
namespace {

using namespace dev;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kRegVecs = 16;  // 16-byte vectors per lane held in registers (8 KB rows)

enum ItemKind : int32_t { kItemRow = 0, kItemSegmentEnd = 1, kItemExit = 2 };

// f(I) for I = 0 .. N-1 with I a compile-time constant (keeps register arrays
// indexed statically even where the compiler would not unroll a loop).
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

struct __align__(16) Meta {
  int32_t kind;
  int32_t req;
  int64_t row;
  float score;     // parent score s
  int32_t node;    // parent node p
  uint32_t o0;     // children of p: ids o0 .. o1-1
  uint32_t o1;
  uint32_t seq;    // ring item number; written before the full-barrier arrive
  uint32_t a0;     // CSR: first staged child id (o0 rounded down to a multiple of 8)
  uint32_t nst;    // CSR: child codes staged from a0 on
  float C;         // histogram reference of the row's request
};

// Consumer-side wait for ring item `item` in `stage`. Several consumer warps
// share the ring, so a warp can reach a stage while the previous item there
// (another warp's) is still in flight; an mbarrier parity wait would then
// match the older phase. Waiting first for the producer to publish this
// item's number makes the stage's pending phase the item's own, after which
// the parity wait is exact. Both waits are bounded.
__device__ __forceinline__ bool wait_item(const Meta* meta, uint64_t* full, int stage,
                                          uint32_t item, uint32_t S, volatile int* abort_flag,
                                          uint32_t* status) {
  const volatile uint32_t* seqp = &meta[stage].seq;
  if (*seqp != item) {
    const uint64_t t0 = global_timer_ns();
    while (*seqp != item) {
      __nanosleep(64);
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitTimeoutNs) {
        *abort_flag = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
  return bounded_wait(&full[stage], (item / S) & 1u, abort_flag, status, kStatusTimeout);
}

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
  int coop;     // 1: every consumer warp works on every row (few rows per CTA)
  int markers;  // segment-end / exit markers per event: W (claimed) or 1 (coop)
};

struct StepWriter {
  float* scores;
  int32_t* parent;
  int32_t* code;
  int32_t* node;
  int n;
  uint32_t V;
  __device__ __forceinline__ void operator()(int r, int i, uint64_t key, int32_t val,
                                             bool valid) const {
    const size_t o = static_cast<size_t>(r) * n + i;
    if (valid) {
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

// Lowest logit a child needs to reach the key threshold `thr`, loosened by a
// relative margin far above fp32 rounding: z < zthr implies key < thr, so
// skipping such codes never drops a candidate the exact key test would keep.
__device__ __forceinline__ float zthreshold(uint64_t thr, float s, float lse) {
  if (thr == 0ull) return __int_as_float(0xFF800000);
  const float T = key_score(thr);
  const float margin = 1e-4f * (1.f + fabsf(T) + fabsf(s) + fabsf(lse));
  return ((T - s) + lse) - margin;
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

// x[k] for a warp-uniform runtime k, through constant indices only (a
// register array indexed at run time would be moved to local memory).
__device__ __forceinline__ uint4 pick_vec(const uint4 (&x)[kRegVecs], int k) {
  switch (k) {
    case 0: return x[0];
    case 1: return x[1];
    case 2: return x[2];
    case 3: return x[3];
    case 4: return x[4];
    case 5: return x[5];
    case 6: return x[6];
    case 7: return x[7];
    case 8: return x[8];
    case 9: return x[9];
    case 10: return x[10];
    case 11: return x[11];
    case 12: return x[12];
    case 13: return x[13];
    case 14: return x[14];
    default: return x[15];
  }
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
template <int BF16>
__device__ __forceinline__ void row_stats_reg(const uint4 (&x)[kRegVecs], int nvec, int lane,
                                              float& m_out, float& lse_out) {
  float m;
  if (BF16) {
    uint32_t r = 0xFF80FF80u;
    Unrolled<kRegVecs>::run([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      if (32 * k < nvec) r = bmax2(r, bmax2(bmax2(x[k].x, x[k].y), bmax2(x[k].z, x[k].w)));
    });
    m = fmaxf(bf_lo(r), bf_hi(r));
  } else {
    m = __int_as_float(0xFF800000);
    Unrolled<kRegVecs>::run([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      if (32 * k < nvec) m = fmaxf(m, vec_max<0>(x[k]));
    });
  }
  // Lane-local max for the exponentials; lanes combined once at the end.
  const float mL = m * kLog2e;
  const uint64_t l2e = pk(kLog2e, kLog2e);
  const uint64_t nml = pk(-mL, -mL);
  uint64_t a0 = 0, a1 = 0;
  Unrolled<kRegVecs>::run([&](auto kc) {
    constexpr int k = decltype(kc)::value;
    if (32 * k < nvec) {
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

// --------------------------------------------------------------- producer
// Histogram reference of request r: its first parent's score (an upper bound
// of every child score when parents arrive ranked best-first, as beam_step
// writes them); any finite value keeps the histogram bounds valid.
__device__ __forceinline__ float request_ref(const StepArgs& a, int r) {
  const float c = a.parent_scores[static_cast<int64_t>(r) * a.B_in];
  return (c > __int_as_float(0xFF800000) && c < __int_as_float(0x7F800000)) ? c : 0.f;
}

__device__ void producer(const StepArgs& a, uint8_t* stages, Meta* meta, uint64_t* full,
                         uint64_t* empty, SelCtl* ctl, int64_t row_lo, int64_t row_hi, int lane) {
  const StepConfig& cfg = a.cfg;
  const int S = cfg.S;
  const uint64_t pol = policy_evict_first();
  const uint32_t max_codes = static_cast<uint32_t>(cfg.extra_bytes / 2);
  uint32_t item = 0;
  bool ok = true;

  auto acquire = [&](uint32_t it) -> int {
    const int stage = static_cast<int>(it % S);
    if (it >= static_cast<uint32_t>(S)) {
      const uint32_t parity = ((it / S) - 1) & 1u;
      if (!bounded_wait(&empty[stage], parity, &ctl->abort_flag, a.status, kStatusTimeout))
        return -1;
    }
    return stage;
  };

  int64_t seg_lo = row_lo;
  while (ok && seg_lo < row_hi) {
    const int r = static_cast<int>(seg_lo / a.B_in);
    const int64_t seg_hi = min(row_hi, static_cast<int64_t>(r + 1) * a.B_in);
    const float C = request_ref(a, r);
    for (int64_t base = seg_lo; ok && base < seg_hi; base += 32) {
      const int64_t row = base + lane;
      const bool in = row < seg_hi;
      float s = __int_as_float(0xFF800000);
      int32_t p = -1;
      if (in) {
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
      unsigned lm = __ballot_sync(0xFFFFFFFFu, live);
      while (lm) {
        const int j = __ffs(lm) - 1;
        lm &= lm - 1;
        const float sj = __shfl_sync(0xFFFFFFFFu, s, j);
        const int32_t pj = __shfl_sync(0xFFFFFFFFu, p, j);
        const uint32_t o0j = __shfl_sync(0xFFFFFFFFu, o0, j);
        const uint32_t o1j = __shfl_sync(0xFFFFFFFFu, o1, j);
        const int stage = acquire(item);
        if (stage < 0) {
          ok = false;
          break;
        }
        if (lane == 0) {
          Meta& m = meta[stage];
          m.kind = kItemRow;
          m.req = r;
          m.row = base + j;
          m.score = sj;
          m.node = pj;
          m.o0 = o0j;
          m.o1 = o1j;
          m.C = C;
          uint8_t* dst = stages + static_cast<size_t>(stage) * cfg.stage_bytes;
          uint32_t extra = 0;
          uint32_t a0 = o0j & ~7u, nst = 0;
          if (a.layout == SIDBEAM_LAYOUT_DENSE) {
            extra = static_cast<uint32_t>(cfg.extra_bytes);
          } else if (a.layout == SIDBEAM_LAYOUT_CSR && o1j > o0j) {
            nst = min(o1j - a0, max_codes);
            extra = (nst * 2 + 15) & ~15u;
          }
          m.a0 = a0;
          m.nst = nst;
          m.seq = item;
          mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(cfg.logits_copy_bytes) + extra);
          bulk_copy_g2s(dst, a.logits + (base + j) * a.row_bytes,
                        static_cast<uint32_t>(cfg.logits_copy_bytes), &full[stage], pol);
          if (a.layout == SIDBEAM_LAYOUT_DENSE)
            bulk_copy_g2s(dst + cfg.logits_copy_bytes,
                          a.mask + static_cast<size_t>(pj) * a.mask_stride, extra, &full[stage],
                          pol);
          else if (extra)
            bulk_copy_g2s(dst + cfg.logits_copy_bytes, a.codes + a0, extra, &full[stage], pol);
        }
        __syncwarp();
        ++item;
      }
    }
    // One segment-end marker per consumer warp (claimed in order, so each warp
    // gets exactly one); in cooperative mode every warp reads every item.
    for (int w = 0; ok && w < a.markers; ++w) {
      const int stage = acquire(item);
      if (stage < 0) {
        ok = false;
        break;
      }
      if (lane == 0) {
        meta[stage].kind = kItemSegmentEnd;
        meta[stage].req = r;
        meta[stage].C = C;
        meta[stage].seq = item;
        mbar_arrive(&full[stage]);
      }
      __syncwarp();
      ++item;
    }
    seg_lo = seg_hi;
  }
  for (int w = 0; ok && w < a.markers; ++w) {
    const int stage = acquire(item);
    if (stage < 0) {
      ok = false;
      break;
    }
    if (lane == 0) {
      meta[stage].kind = kItemExit;
      meta[stage].seq = item;
      mbar_arrive(&full[stage]);
    }
    __syncwarp();
    ++item;
  }
  if (!ok) {
    // Abort: let the copies already issued land before the CTA exits.
    const uint32_t first = item > static_cast<uint32_t>(S) ? item - S : 0u;
    for (uint32_t it = first; it < item; ++it) drain_wait(&full[it % S], (it / S) & 1u);
  }
}

// --------------------------------------------------------------- consumers
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

// Code of CSR child id k: from the stage when it was staged, else from HBM/L2.
__device__ __forceinline__ int csr_code(const StepArgs& a, const uint8_t* zrow, const Meta& m,
                                        uint32_t k) {
  const uint32_t i = k - m.a0;
  if (i < m.nst) return reinterpret_cast<const uint16_t*>(zrow + a.cfg.logits_copy_bytes)[i];
  return a.codes[k];
}

// Threshold state at the start of a row.
__device__ __forceinline__ void row_thresholds(WarpBuf& wb, SelCtl* ctl, unsigned long long req) {
  const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
  if (c > wb.thr) wb.thr = c;
  if (req > wb.thr) wb.thr = req;
}

// Row worked on in place in its stage (rows over 8 KB, or CSR rows with more
// children than one 32-lane batch per warp). The caller returns the stage.
template <int BF16>
__device__ __forceinline__ void process_row_smem(const StepArgs& a, const uint8_t* zrow, const Meta& m,
                                 WarpBuf& wb, SelCtl* ctl, uint32_t* wprefix, int lane, int part,
                                 int nparts) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  const int r = m.req;
  const uint32_t b = static_cast<uint32_t>(m.row - static_cast<int64_t>(r) * a.B_in);
  const uint32_t idx0 = b * static_cast<uint32_t>(a.V);
  const float s = m.score;
  const float C = m.C;
  const ThrSinks sinks{&ctl->cta_thr, a.request_thr + r};
  const unsigned long long req_thr =
      *reinterpret_cast<volatile unsigned long long*>(a.request_thr + r);

  float rmax, lse;
  row_stats<BF16>(zrow, a.V, lane, rmax, lse);
  row_thresholds(wb, ctl, req_thr);
  float zthr = zthreshold(wb.thr, s, lse);
  if (rmax < zthr) return;  // even the row's largest logit cannot reach the threshold

  if (a.layout == SIDBEAM_LAYOUT_CSR) {
    const uint32_t k_step = static_cast<uint32_t>(32 * nparts);
    const uint32_t k_begin = m.o0 + static_cast<uint32_t>(part * 32);
    for (int pass = 0; pass < 2; ++pass) {
      for (uint32_t k0 = k_begin; k0 < m.o1; k0 += k_step) {
        const uint32_t k = k0 + lane;
        const bool in = k < m.o1;
        const int c = in ? csr_code(a, zrow, m, k) : 0;
        const float z = in ? elem<BF16>(zrow, c) : 0.f;
        const bool ok = in && z >= zthr;
        if (!__any_sync(0xFFFFFFFFu, ok)) continue;
        const float score = s + (z - lse);
        if (pass == 0) {
          warp_bin(ctl->hist, ok, score_bin(score, C), wb.binned);
        } else {
          warp_offer(wb, ok, make_key(score, idx0 + static_cast<uint32_t>(c)),
                     static_cast<int32_t>(k), a.n, lane, sinks);
          zthr = zthreshold(wb.thr, s, lse);
        }
      }
      if (pass == 0) {
        __syncwarp();
        refresh_thr(wb, ctl, a.n, C, lane, sinks);
        zthr = zthreshold(wb.thr, s, lse);
      }
    }
    return;
  }

  // Dense bitmask or no trie: walk 16-byte vectors; a vector is opened only if
  // its largest logit reaches the threshold.
  const bool dense = a.layout == SIDBEAM_LAYOUT_DENSE;
  const uint32_t* mrow = reinterpret_cast<const uint32_t*>(zrow + a.cfg.logits_copy_bytes);
  const int nvec_all = (a.V + kPerVec - 1) / kPerVec;
  const uint4* q = reinterpret_cast<const uint4*>(zrow);
  bool have_prefix = false;
  for (int pass = 0; pass < 2; ++pass) {
    for (int v0 = part * 32; v0 < nvec_all; v0 += 32 * nparts) {
      const int v = v0 + lane;
      unsigned bits = 0;
      if (v < nvec_all) {
        const uint4 x = q[v];
        if (vec_max<BF16>(x) >= zthr) {
          const int cb = v * kPerVec;
          unsigned valid = (1u << kPerVec) - 1u;
          if (dense) valid = (mrow[cb >> 5] >> (cb & 31)) & ((1u << kPerVec) - 1u);
          for (int j = 0; j < kPerVec; ++j)
            if (((valid >> j) & 1u) && cb + j < a.V && elem<BF16>(zrow, cb + j) >= zthr)
              bits |= 1u << j;
        }
      }
      if (!__any_sync(0xFFFFFFFFu, bits != 0u)) continue;
      if (pass == 1 && dense && !have_prefix) {
        dense_prefix(mrow, a.mask_words, wprefix, lane);
        have_prefix = true;
      }
      while (__any_sync(0xFFFFFFFFu, bits != 0u)) {
        const bool has = bits != 0u;
        const int j = has ? __ffs(bits) - 1 : 0;
        bits &= bits - 1u;
        const int c = v * kPerVec + j;
        const float score = has ? s + (elem<BF16>(zrow, c) - lse) : 0.f;
        if (pass == 0) {
          warp_bin(ctl->hist, has, score_bin(score, C), wb.binned);
        } else {
          const int32_t node = (has && dense) ? dense_child(mrow, wprefix, m.o0, c) : -1;
          warp_offer(wb, has, make_key(score, idx0 + static_cast<uint32_t>(c)), node, a.n, lane,
                     sinks);
        }
      }
      if (pass == 1) zthr = zthreshold(wb.thr, s, lse);
    }
    if (pass == 0) {
      __syncwarp();
      refresh_thr(wb, ctl, a.n, C, lane, sinks);
      zthr = zthreshold(wb.thr, s, lse);
    }
  }
}

// Row of up to 8 KB: copied into registers (plus the trie data the candidate
// walk needs: the dense mask row into warp-private shared memory, or this
// lane's CSR child), then the stage is returned before any arithmetic.
template <int BF16>
__device__ __forceinline__ void process_row_reg(const StepArgs& a, const uint8_t* zrow, uint64_t* empty_bar,
                                const Meta& m, WarpBuf& wb, SelCtl* ctl, uint32_t* wmask,
                                uint32_t* wprefix, int lane, int part, int nparts) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  const int V = a.V;
  const int nvec = (V + kPerVec - 1) / kPerVec;
  const int r = m.req;
  const uint32_t b = static_cast<uint32_t>(m.row - static_cast<int64_t>(r) * a.B_in);
  const uint32_t idx0 = b * static_cast<uint32_t>(V);
  const float s = m.score;
  const float C = m.C;
  const ThrSinks sinks{&ctl->cta_thr, a.request_thr + r};
  const unsigned long long req_thr =
      *reinterpret_cast<volatile unsigned long long*>(a.request_thr + r);
  const bool dense = a.layout == SIDBEAM_LAYOUT_DENSE;
  const bool csr = a.layout == SIDBEAM_LAYOUT_CSR;

  const uint4* q = reinterpret_cast<const uint4*>(zrow);
  const uint4 ninf = BF16 ? make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u)
                          : make_uint4(0xFF800000u, 0xFF800000u, 0xFF800000u, 0xFF800000u);
  uint4 x[kRegVecs];
  const int tail = V % kPerVec;
  const int vt = tail ? nvec - 1 : -1;
  Unrolled<kRegVecs>::run([&](auto kc) {
    constexpr int k = decltype(kc)::value;
    const int v = lane + 32 * k;
    x[k] = v < nvec ? q[v] : ninf;
    if (v == vt) vec_cut<BF16>(x[k], tail);
  });
  if (dense) {
    const uint32_t* mrow = reinterpret_cast<const uint32_t*>(zrow + a.cfg.logits_copy_bytes);
    for (int i = lane; i < a.mask_stride; i += 32) wmask[i] = mrow[i];
  }
  const uint32_t ck = m.o0 + static_cast<uint32_t>(part * 32 + lane);
  const bool cin = csr && ck < m.o1;
  int ccode = 0;
  float cz = 0.f;
  if (cin) {
    ccode = csr_code(a, zrow, m, ck);
    cz = elem<BF16>(zrow, ccode);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(empty_bar);  // the producer may refill the stage now

  float rmax, lse;
  row_stats_reg<BF16>(x, nvec, lane, rmax, lse);
  row_thresholds(wb, ctl, req_thr);
  float zthr = zthreshold(wb.thr, s, lse);
  if (rmax < zthr) return;

  if (csr) {
    for (int pass = 0; pass < 2; ++pass) {
      const bool ok = cin && cz >= zthr;
      if (__any_sync(0xFFFFFFFFu, ok)) {
        const float score = s + (cz - lse);
        if (pass == 0) {
          warp_bin(ctl->hist, ok, score_bin(score, C), wb.binned);
          __syncwarp();
          refresh_thr(wb, ctl, a.n, C, lane, sinks);
          zthr = zthreshold(wb.thr, s, lse);
        } else {
          warp_offer(wb, ok, make_key(score, idx0 + static_cast<uint32_t>(ccode)),
                     static_cast<int32_t>(ck), a.n, lane, sinks);
        }
      } else {
        break;
      }
    }
    return;
  }

  bool have_prefix = false;
  for (int pass = 0; pass < 2; ++pass) {
    // Which of this lane's vectors can hold a child above the threshold.
    uint32_t flags = 0;
    Unrolled<kRegVecs>::run([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      if (32 * k < nvec && (k % nparts) == part && lane + 32 * k < nvec &&
          vec_max<BF16>(x[k]) >= zthr)
        flags |= 1u << k;
    });
    uint32_t todo = __reduce_or_sync(0xFFFFFFFFu, flags);
    while (todo) {
      const int k = __ffs(todo) - 1;
      todo &= todo - 1;
      const uint4 xk = pick_vec(x, k);
      const int v = lane + 32 * k;
      unsigned bits = 0;
      if ((flags >> k) & 1u) {
        const int cb = v * kPerVec;
        unsigned valid = (1u << kPerVec) - 1u;
        if (dense) valid = (wmask[cb >> 5] >> (cb & 31)) & ((1u << kPerVec) - 1u);
#pragma unroll
        for (int j = 0; j < kPerVec; ++j)
          if (((valid >> j) & 1u) && cb + j < V && vec_elem<BF16>(xk, j) >= zthr)
            bits |= 1u << j;
      }
      if (!__any_sync(0xFFFFFFFFu, bits != 0u)) continue;
      if (pass == 1 && dense && !have_prefix) {
        dense_prefix(wmask, a.mask_words, wprefix, lane);
        have_prefix = true;
      }
      while (__any_sync(0xFFFFFFFFu, bits != 0u)) {
        const bool has = bits != 0u;
        const int j = has ? __ffs(bits) - 1 : 0;
        bits &= bits - 1u;
        const int c = v * kPerVec + j;
        const float score = has ? s + (vec_elem<BF16>(xk, j) - lse) : 0.f;
        if (pass == 0) {
          warp_bin(ctl->hist, has, score_bin(score, C), wb.binned);
        } else {
          const int32_t node = (has && dense) ? dense_child(wmask, wprefix, m.o0, c) : -1;
          warp_offer(wb, has, make_key(score, idx0 + static_cast<uint32_t>(c)), node, a.n, lane,
                     sinks);
        }
      }
      if (pass == 1) zthr = zthreshold(wb.thr, s, lse);
    }
    if (pass == 0) {
      __syncwarp();
      refresh_thr(wb, ctl, a.n, C, lane, sinks);
      zthr = zthreshold(wb.thr, s, lse);
    }
  }
}

template <int BF16, int REG>
__global__ void __launch_bounds__(REG ? kMaxStepThreadsReg : kMaxStepThreads, 1)
    beam_step_kernel(const __grid_constant__ StepArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const StepConfig& cfg = a.cfg;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + cfg.off_bars);
  uint64_t* empty = full + cfg.S;
  SelCtl* ctl = reinterpret_cast<SelCtl*>(smem + cfg.off_ctl);
  Meta* meta = reinterpret_cast<Meta*>(smem + cfg.off_meta);
  uint32_t* cta_hist = reinterpret_cast<uint32_t*>(smem + cfg.off_chist);
  uint32_t* whist = reinterpret_cast<uint32_t*>(smem + cfg.off_whist);
  uint32_t* wprefix = reinterpret_cast<uint32_t*>(smem + cfg.off_wprefix);
  uint32_t* wmask = reinterpret_cast<uint32_t*>(smem + cfg.off_wmask);
  uint8_t* stages = smem + cfg.off_stage;
  uint64_t* wkeys = reinterpret_cast<uint64_t*>(smem + cfg.off_wkeys);
  int32_t* wvals = reinterpret_cast<int32_t*>(smem + cfg.off_wvals);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < cfg.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], a.coop ? cfg.W : 1);
      meta[s].seq = 0xFFFFFFFFu;
    }
    ctl->cta_thr = 0ull;
    ctl->abort_flag = 0;
    ctl->counter = 0;
    ctl->next_item = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) ctl->hist[i] = 0u;
  __syncthreads();

  int64_t row_lo, row_hi;
  a.part.range(static_cast<int>(blockIdx.x), row_lo, row_hi);

  if (warp == 0) {
    producer(a, stages, meta, full, empty, ctl, row_lo, row_hi, lane);
    return;
  }

  Team team{static_cast<int>(threadIdx.x) - 32, cfg.W * 32, warp - 1, lane, cfg.W};
  WarpBuf wb{wkeys + static_cast<size_t>(team.warp) * cfg.Cw,
             wvals + static_cast<size_t>(team.warp) * cfg.Cw, whist + team.warp * 256, cfg.Cw,
             0, 0ull, 0};
  uint32_t* my_prefix = wprefix + team.warp * cfg.prefix_words;
  uint32_t* my_mask = wmask + team.warp * cfg.prefix_words;
  const StepWriter writer{a.out_scores, a.out_parent, a.out_code, a.out_node, a.n,
                          static_cast<uint32_t>(a.V)};
  const int part = a.coop ? team.warp : 0;
  const int nparts = a.coop ? cfg.W : 1;

  // Items are claimed in order from a shared counter (round-robin would let
  // one slow row hold back the items queued behind it); in cooperative mode
  // every warp takes every item.
  uint32_t item = 0;
  while (true) {
    if (!a.coop) {
      int claimed = 0;
      if (lane == 0) claimed = atomicAdd(&ctl->next_item, 1);
      item = static_cast<uint32_t>(__shfl_sync(0xFFFFFFFFu, claimed, 0));
    }
    const int stage = static_cast<int>(item % cfg.S);
    const bool got = wait_item(meta, full, stage, item, static_cast<uint32_t>(cfg.S),
                               &ctl->abort_flag, a.status);
    Meta m;
    int kind = kItemSegmentEnd;
    if (got) {
      m = meta[stage];
      kind = m.kind;
    } else {
      m.req = -1;
    }
    __syncwarp();
    if (kind == kItemRow) {
      const uint8_t* zrow = stages + static_cast<size_t>(stage) * cfg.stage_bytes;
      const bool reg_ok = REG && (a.layout != SIDBEAM_LAYOUT_CSR ||
                                  m.o1 - m.o0 <= static_cast<uint32_t>(32 * nparts));
      if (reg_ok) {
        process_row_reg<BF16>(a, zrow, &empty[stage], m, wb, ctl, my_mask, my_prefix, lane, part,
                              nparts);
      } else {
        process_row_smem<BF16>(a, zrow, m, wb, ctl, my_prefix, lane, part, nparts);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
      }
    } else {
      if (got && lane == 0) mbar_arrive(&empty[stage]);
      if (kind == kItemExit) {
        team_sync_or(team, false);  // pairs with any warp that stops on an abort
        break;
      }
      const int r = m.req;
      FlushArgs f;
      f.n = a.n;
      f.r = r < 0 ? 0 : r;
      f.k = static_cast<int>(blockIdx.x) - a.part.first_cta(f.r);
      f.G = a.part.contributors(f.r);
      f.maxG = a.part.maxG;
      f.part_keys = a.part_keys;
      f.part_vals = a.part_vals;
      f.part_count = a.part_count;
      f.tickets = a.tickets;
      f.request_thr = a.request_thr;
      f.ghist = a.ghist;
      f.C = m.C;
      f.wkeys = wkeys;
      f.cw = cfg.Cw;
      f.sort_keys = wkeys;
      f.sort_vals = wvals;
      f.sort_cap = cfg.W * cfg.Cw;
      f.radix_hist = cta_hist;
      if (segment_flush(team, wb, ctl, f, writer)) break;
    }
    if (a.coop) ++item;
  }
}

}  // namespace

// ------------------------------------------------------------------ host side

static int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Shared-memory plan: stage = logits row (16-byte rounded) + trie extra
// (dense mask row / staged CSR codes); per consumer warp: top-n buffer,
// radix histogram, dense prefix counts (and, on the register path, a mask copy).
bool choose_step_config(int V, int esize, int extra_bytes, int prefix_words, int n, bool reg,
                        StepConfig* cfg) {
  StepConfig c{};
  c.logits_copy_bytes = round_up(V * esize, 16);
  c.extra_bytes = extra_bytes;
  c.stage_bytes = round_up(c.logits_copy_bytes + extra_bytes, 128);
  c.prefix_words = prefix_words;
  c.reg = reg ? 1 : 0;
  int npow2 = 1;
  while (npow2 < n) npow2 <<= 1;
  const int ctl_bytes = round_up(static_cast<int>(sizeof(dev::SelCtl)), 128);
  const int meta_bytes = kMaxStages * static_cast<int>(sizeof(Meta));
  static const int kWarpsSmem[] = {12, 10, 8, 6, 4, 3, 2, 1};
  static const int kWarpsReg[] = {8, 6, 4, 3, 2, 1};
  const int* warps = reg ? kWarpsReg : kWarpsSmem;
  const int nw = reg ? 6 : 8;
  for (int wi = 0; wi < nw; ++wi) {
    const int W = warps[wi];
    const int cw = std::max(round_up(n, 32) + 128, round_up((npow2 + W - 1) / W, 32));
    int o = 0;
    c.off_bars = o;
    o += 2 * kMaxStages * 8;
    c.off_ctl = o;
    o += ctl_bytes;
    c.off_meta = o;
    o += meta_bytes;
    c.off_chist = o;
    o += 1024;
    c.off_whist = o;
    o += W * 1024;
    c.off_wprefix = o;
    o += W * c.prefix_words * 4;
    c.off_wmask = o;
    o += reg ? W * c.prefix_words * 4 : 0;
    o = round_up(o, 128);
    const int warp_bytes = W * cw * 12 + 256;
    const int avail = kSmemBudget - o - warp_bytes;
    if (avail < c.stage_bytes) continue;
    const int S = std::min(kMaxStages, avail / c.stage_bytes);
    if (S < 6 && W > 2) continue;
    c.W = W;
    c.S = S;
    c.Cw = cw;
    c.off_stage = o;
    o += S * c.stage_bytes;
    c.off_wkeys = round_up(o, 128);
    o = c.off_wkeys + W * cw * 8;
    c.off_wvals = round_up(o, 16);
    o = c.off_wvals + W * cw * 4;
    c.smem_bytes = round_up(o, 128);
    if (c.smem_bytes > kSmemBudget) continue;
    *cfg = c;
    return true;
  }
  return false;
}

// Raise the kernel's dynamic shared-memory limit to the full budget once per
// device (kept out of the per-call path, and out of any stream capture that
// follows a first eager call).
static cudaError_t opt_in_smem(const void* fn, int which) {
  static std::mutex mu;
  static bool done[4][64] = {};
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
                     cudaStream_t stream) {
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
  a.tickets = reinterpret_cast<uint32_t*>(w + ws.tickets);
  a.request_thr = reinterpret_cast<unsigned long long*>(w + ws.request_thr);
  a.part_count = reinterpret_cast<uint32_t*>(w + ws.part_count);
  a.part_keys = reinterpret_cast<unsigned long long*>(w + ws.part_keys);
  a.part_vals = reinterpret_cast<int32_t*>(w + ws.part_vals);
  a.ghist = reinterpret_cast<uint32_t*>(w + ws.ghist);

  const bool dense = a.layout == SIDBEAM_LAYOUT_DENSE;
  const int extra = dense ? a.mask_stride * 4 : (a.layout == SIDBEAM_LAYOUT_CSR ? 512 : 0);
  const int prefix_words = dense ? a.mask_stride : 0;
  const bool reg = static_cast<int64_t>(V) * esize <= 16 * 32 * kRegVecs;
  if (!choose_step_config(V, esize, extra, prefix_words, n_out, reg, &a.cfg) &&
      !(reg && choose_step_config(V, esize, extra, prefix_words, n_out, false, &a.cfg)))
    return set_error(SIDBEAM_ERR_INVALID_ARG,
                     "beam_step: V=%d with n_out=%d does not fit in shared memory", V, n_out);
  a.coop = a.part.rows_per_cta < a.cfg.W ? 1 : 0;
  a.markers = a.coop ? 1 : a.cfg.W;

  const void* fns[4] = {reinterpret_cast<const void*>(&beam_step_kernel<0, 0>),
                        reinterpret_cast<const void*>(&beam_step_kernel<1, 0>),
                        reinterpret_cast<const void*>(&beam_step_kernel<0, 1>),
                        reinterpret_cast<const void*>(&beam_step_kernel<1, 1>)};
  const int which = (a.cfg.reg ? 2 : 0) + (a.bf16 ? 1 : 0);
  cudaError_t e = opt_in_smem(fns[which], which);
  if (e != cudaSuccess) return cuda_error(e, "beam_step: cudaFuncSetAttribute");
  const dim3 grid(static_cast<unsigned>(a.part.grid));
  const dim3 block(static_cast<unsigned>(32 * (a.cfg.W + 1)));
  switch (which) {
    case 0: beam_step_kernel<0, 0><<<grid, block, a.cfg.smem_bytes, stream>>>(a); break;
    case 1: beam_step_kernel<1, 0><<<grid, block, a.cfg.smem_bytes, stream>>>(a); break;
    case 2: beam_step_kernel<0, 1><<<grid, block, a.cfg.smem_bytes, stream>>>(a); break;
    default: beam_step_kernel<1, 1><<<grid, block, a.cfg.smem_bytes, stream>>>(a); break;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "beam_step: launch");
  return SIDBEAM_OK;
}

}  // namespace sidbeam
