// Exact per-request top-n selection on 64-bit keys, shared by beam_step and
// catalog_score_topk.
//
// Keys are unique (score in the high half, 2^32-1-idx in the low half), so
// "the n largest keys" is a set with no ties, and "key >= K" for a threshold K
// found by an MSB-first radix walk selects exactly n of them.
//
// Work is cut by thresholds that are always valid lower bounds on the
// request's n-th best key (there are at least n real candidates at or above
// them), so filtering by them never drops a member of the top n:
//  * a score histogram per request: 1024 bins of 1/16 nat below a reference
//    score C (an upper bound of the request's scores; everything above C falls
//    in bin 0, everything far below in the last bin). Each CTA keeps one in
//    shared memory for its current request; candidates are counted before
//    they are offered, and the first bin whose cumulative count reaches n
//    gives a threshold one bin further down (so fp32 rounding of the bin index
//    can never make it too high). At the end of a segment the CTA adds its
//    counts to the request's global histogram;
//  * the key at which a warp buffer was compacted (below);
//  * the largest of these, shared CTA-wide (shared memory) and request-wide
//    (a global atomicMax).
// Three levels of exact selection:
//  1. warp: surviving candidates go to a shared-memory buffer of Cw >= n + 32
//     entries; when it is full the warp keeps its n best (radix walk) and
//     raises its threshold to the n-th key;
//  2. CTA (end of a request segment): entries above the request-wide bound are
//     cut to the CTA's n best and written to the CTA's slot of the request's
//     partial lists in global memory;
//  3. request: the CTA that takes the last ticket (threadfence + atomic
//     counter; nothing ever spins) reads the complete histogram and ranks the
//     partial entries (below), writes them out and zeroes the ticket, bound
//     and histogram for the next call. A CTA that holds a whole request ranks
//     its warp buffers directly, with no partial lists and no ticket.
// Ranking by histogram: every candidate that reaches the top n was counted
// exactly once, in the bin of its own fp32 score, so P[b] (the count in the
// bins above b) is exactly the number of top-n members that outrank every
// member of bin b. An entry's rank is P[b] plus the number of entries of its
// own bin with a larger key; grouping the entries by bin (counting-sort
// scatter) makes that a handful of compares per entry. Entries ranked >= n
// are dropped. When a bin is too crowded (ties, a reference far off) or the
// staging area too small, the entries are selected (radix walk) and sorted
// (bitonic) instead.
#pragma once

#include "device_utils.cuh"

namespace sidbeam {
namespace dev {

constexpr int kBarConsumers = 1;  // named barrier id used by the consumer warps
constexpr int kMaxSegCounts = 640;
constexpr int kHistBins = 1024;
constexpr float kHistScale = 16.f;  // bins per nat

// The consumer warps of a CTA (the threads that run selection).
struct Team {
  int tid;     // 0 .. T-1
  int T;       // consumer threads = 32 * nwarps
  int warp;    // consumer warp 0 .. nwarps-1
  int lane;
  int nwarps;
};

__device__ __forceinline__ void team_sync(const Team& t) { named_sync(kBarConsumers, t.T); }

// Barrier that also ORs a predicate over all consumer threads; every warp
// gets the same answer, so all of them leave together when one saw an abort.
__device__ __forceinline__ bool team_sync_or(const Team& t, bool pred) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(res)
      : "r"(pred ? 1u : 0u), "r"(kBarConsumers), "r"(t.T)
      : "memory");
  return res != 0;
}

// ------------------------------------------------------------ radix select
// Given a 256-bin histogram of the current digit (only bins < 2^width are
// non-zero), finds digit d such that the keys in higher bins number `above`
// < need <= above + hist[d]. Warp-collective (one warp).
__device__ __forceinline__ void find_digit_warp(const uint32_t* hist, uint32_t need, int lane,
                                                int& d, uint32_t& above, uint32_t& cnt) {
  uint32_t h[8];
  uint32_t s = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    h[j] = hist[lane * 8 + j];
    s += h[j];
  }
  uint32_t x = s;  // inclusive suffix sum over lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, x, o);
    if (lane + o < 32) x += y;
  }
  const uint32_t excl = x - s;
  const unsigned b = __ballot_sync(0xFFFFFFFFu, excl < need && need <= x);
  if (b == 0) {  // cannot happen when the histogram holds >= need keys
    d = 0;
    above = 0;
    cnt = need;
    return;
  }
  const int src = __ffs(b) - 1;
  int dd = 0;
  uint32_t ab = 0, ct = 0;
  bool found = false;
  uint32_t cum = excl;
#pragma unroll
  for (int j = 7; j >= 0; --j) {
    if (!found && cum + h[j] >= need) {
      found = true;
      dd = lane * 8 + j;
      ab = cum;
      ct = h[j];
    }
    cum += h[j];
  }
  d = __shfl_sync(0xFFFFFFFFu, dd, src);
  above = __shfl_sync(0xFFFFFFFFu, ab, src);
  cnt = __shfl_sync(0xFFFFFFFFu, ct, src);
}

// Histogram increment (shared-memory atomic). Lanes with `active` false add
// nothing; lanes may call it divergently.
__device__ __forceinline__ void hist_add(uint32_t* hist, bool active, uint32_t bin, int) {
  if (active) atomicAdd(&hist[bin], 1u);
}

// Score-histogram increment by a whole warp; counts the additions for the
// refresh policy. Warp-collective.
__device__ __forceinline__ void warp_bin(uint32_t* hist, bool active, uint32_t bin, int& binned,
                                         unsigned* total) {
  if (active) atomicAdd(&hist[bin], 1u);
  const int c = __popc(__ballot_sync(0xFFFFFFFFu, active));
  binned += c;
  if (c && (threadIdx.x & 31) == 0) atomicAdd(total, static_cast<unsigned>(c));
}

// Threshold K with exactly `need` keys >= K among keys[0..count) (count > need >= 1).
// Warp-collective; hist = 256 words of this warp's shared memory.
__device__ inline uint64_t warp_select(const uint64_t* keys, int count, uint32_t need,
                                       uint32_t* hist, int lane) {
  uint64_t a = ~0ull, o = 0;
  for (int i = lane; i < count; i += 32) {
    const uint64_t k = keys[i];
    a &= k;
    o |= k;
  }
  a = warp_and64(a);
  o = warp_or64(o);
  const uint64_t diff = a ^ o;
  if (diff == 0) return a;
  int hi = 64 - __clzll(static_cast<long long>(diff));  // bits >= hi are common to all keys
  uint64_t prefix = hi >= 64 ? 0ull : ((a >> hi) << hi);
  while (true) {
    const int lo = hi > 8 ? hi - 8 : 0;
    const uint32_t dmask = (1u << (hi - lo)) - 1u;
    for (int i = lane; i < 256; i += 32) hist[i] = 0;
    __syncwarp();
    for (int base = 0; base < count; base += 32) {
      const int i = base + lane;
      const uint64_t k = i < count ? keys[i] : 0ull;
      const bool match = i < count && (hi >= 64 || ((k >> hi) == (prefix >> hi)));
      hist_add(hist, match, static_cast<uint32_t>(k >> lo) & dmask, lane);
    }
    __syncwarp();
    int d;
    uint32_t above, cnt;
    find_digit_warp(hist, need, lane, d, above, cnt);
    __syncwarp();
    prefix |= static_cast<uint64_t>(d) << lo;
    need -= above;
    if (cnt == need || lo == 0) return prefix;
    hi = lo;
  }
}

// ------------------------------------------------------------ score histogram
__device__ __forceinline__ uint32_t score_bin(float score, float C) {
  const float x = (C - score) * kHistScale;
  if (!(x >= 0.f)) return 0u;  // above the reference (or NaN reference)
  if (x >= static_cast<float>(kHistBins - 1)) return kHistBins - 1;
  return static_cast<uint32_t>(x);
}

// Smallest key of any candidate whose score is >= s (its score half only).
__device__ __forceinline__ uint64_t key_floor(float s) {
  return static_cast<uint64_t>(ord_f32(s)) << 32;
}

// From a histogram with at least n counted candidates in bins 0..k, those
// candidates all score above C - (k+2)/16 (one bin of slack for fp32 rounding
// of the bin index), so key_floor of that value is a valid lower bound.
// Returns 0 when fewer than n are counted or the bound falls in the last bins.
// Warp-collective over a 1024-bin, 16-byte aligned histogram.
__device__ __forceinline__ uint64_t hist_bound(const uint32_t* hist, uint32_t n, float C,
                                               int lane) {
  // Lane l owns bins 32l .. 32l+31; its eight 16-byte reads are rotated by l
  // so that the 8 lanes of each access phase hit 8 different bank groups.
  const uint4* h4 = reinterpret_cast<const uint4*>(hist) + lane * 8;
  uint32_t s = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 v = h4[(j + lane) & 7];
    s += v.x + v.y + v.z + v.w;
  }
  uint32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned b = __ballot_sync(0xFFFFFFFFu, incl >= n);
  if (b == 0) return 0ull;
  const int src = __ffs(b) - 1;
  int k = 0;
  if (lane == src) {  // one lane walks its own 32 bins in order
    uint32_t cum = incl - s;
    int j = 0;
    for (; j < 7; ++j) {
      const uint4 v = h4[j];
      const uint32_t c = v.x + v.y + v.z + v.w;
      if (cum + c >= n) break;
      cum += c;
    }
    const uint32_t* hb = hist + lane * 32 + j * 4;
    int e = 0;
    while (e < 3 && cum + hb[e] < n) cum += hb[e++];
    k = lane * 32 + j * 4 + e;
  }
  k = __shfl_sync(0xFFFFFFFFu, k, src);
  if (k >= kHistBins - 2) return 0ull;
  return key_floor(C - static_cast<float>(k + 2) / kHistScale);
}

// hist_bound over a histogram held in registers: lane l holds bins 32l .. 32l+31
// as h[0..7] (four bins each, in order).
__device__ __forceinline__ uint64_t hist_bound_regs(const uint4 (&h)[8], uint32_t n, float C,
                                                    int lane) {
  uint32_t s = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) s += h[j].x + h[j].y + h[j].z + h[j].w;
  uint32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned b = __ballot_sync(0xFFFFFFFFu, incl >= n);
  if (b == 0) return 0ull;
  const int src = __ffs(b) - 1;
  int k = 0;
  if (lane == src) {
    uint32_t cum = incl - s;
    int found = -1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t v[4] = {h[j].x, h[j].y, h[j].z, h[j].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        cum += v[e];
        if (found < 0 && cum >= n) found = 4 * j + e;
      }
    }
    k = lane * 32 + found;
  }
  k = __shfl_sync(0xFFFFFFFFu, k, src);
  if (k >= kHistBins - 2) return 0ull;
  return key_floor(C - static_cast<float>(k + 2) / kHistScale);
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

// ------------------------------------------------------------ shared control
struct SelCtl {
  unsigned long long cta_thr;  // CTA-wide lower bound on the segment's n-th best key
  unsigned long long bcast_key;
  unsigned long long red[64];  // AND/OR partials, 2 per warp (<= 32 warps)
  int bcast_d;
  unsigned bcast_above;
  unsigned bcast_cnt;
  int counter;
  int is_last;
  int abort_flag;
  int staged;
  int rank_bad;                // rank merge: the entries did not match the histogram
  unsigned hist_total;         // candidates counted in `hist` and not yet pushed
  int push_lock;               // beam_step: one warp at a time moves `hist` to the request's
  int next_row;                // beam_step: next entry of the CTA's row table to hand out
  unsigned ref_ord[2];         // beam_step: max parent score (ordered) of a segment, by parity
  int wcount[32];
  int segoff[kMaxSegCounts + 1];
  __align__(16) uint32_t hist[kHistBins];  // score histogram of the current segment
};

// Key source for the CTA-level select: nseg buffers of stride cw.
struct WarpBufSrc {
  const uint64_t* keys;  // [nseg][cw]
  int cw;
  const int* counts;     // shared
  int nseg;
  __device__ __forceinline__ int count(int s) const { return counts[s]; }
  __device__ __forceinline__ uint64_t key(int s, int i) const { return keys[s * cw + i]; }
};

// Key source for the CTA-level select: one request's partial lists in global
// memory (list k holds segoff[k+1] - segoff[k] entries at stride n).
struct PartialSrc {
  const unsigned long long* keys;
  int n;
  const int* segoff;  // shared
  int nseg;
  __device__ __forceinline__ int count(int s) const { return segoff[s + 1] - segoff[s]; }
  __device__ __forceinline__ uint64_t key(int s, int i) const {
    return __ldcg(keys + static_cast<size_t>(s) * n + i);
  }
};

// CTA-level threshold: K with exactly `need` keys >= K over all segments of src
// (total > need >= 1). All consumer threads call it; uses team_sync.
// `hist` is a 256-word scratch histogram.
template <class Src>
__device__ uint64_t cta_select(const Team& t, const Src& src, uint32_t need, uint32_t* hist,
                               SelCtl* ctl) {
  uint64_t a = ~0ull, o = 0;
  for (int s = 0; s < src.nseg; ++s) {
    const int c = src.count(s);
    for (int i = t.tid; i < c; i += t.T) {
      const uint64_t k = src.key(s, i);
      a &= k;
      o |= k;
    }
  }
  a = warp_and64(a);
  o = warp_or64(o);
  if (t.lane == 0) {
    ctl->red[2 * t.warp] = a;
    ctl->red[2 * t.warp + 1] = o;
  }
  team_sync(t);
  a = ~0ull;
  o = 0;
  for (int w = 0; w < t.nwarps; ++w) {
    a &= ctl->red[2 * w];
    o |= ctl->red[2 * w + 1];
  }
  const uint64_t diff = a ^ o;
  if (diff == 0) return a;  // uniform across threads
  int hi = 64 - __clzll(static_cast<long long>(diff));
  uint64_t prefix = hi >= 64 ? 0ull : ((a >> hi) << hi);
  while (true) {
    const int lo = hi > 8 ? hi - 8 : 0;
    const uint32_t dmask = (1u << (hi - lo)) - 1u;
    for (int i = t.tid; i < 256; i += t.T) hist[i] = 0;
    team_sync(t);
    for (int s = 0; s < src.nseg; ++s) {
      const int c = src.count(s);
      for (int base = 0; base < c; base += t.T) {
        const int i = base + t.tid;
        const uint64_t k = i < c ? src.key(s, i) : 0ull;
        const bool match = i < c && (hi >= 64 || ((k >> hi) == (prefix >> hi)));
        hist_add(hist, match, static_cast<uint32_t>(k >> lo) & dmask, t.lane);
      }
    }
    team_sync(t);
    if (t.warp == 0) {
      int d;
      uint32_t above, cnt;
      find_digit_warp(hist, need, t.lane, d, above, cnt);
      if (t.lane == 0) {
        ctl->bcast_d = d;
        ctl->bcast_above = above;
        ctl->bcast_cnt = cnt;
      }
    }
    team_sync(t);
    const int d = ctl->bcast_d;
    const uint32_t above = ctl->bcast_above;
    const uint32_t cnt = ctl->bcast_cnt;
    prefix |= static_cast<uint64_t>(d) << lo;
    need -= above;
    if (cnt == need || lo == 0) return prefix;
    hi = lo;
  }
}

// Bitonic sort of N (a power of two) (key, value) pairs in shared memory into
// descending key order. Compare-exchanges whose partners lie within one
// aligned block of 32 run inside a warp on registers (shuffles); only strides
// of 32 and more go through shared memory with a barrier per stride.
__device__ __forceinline__ void bitonic_warp_block(const Team& t, uint64_t* keys, int32_t* vals,
                                                   int N, int size_lo, int size_hi,
                                                   int first_stride) {
  for (int blk = t.warp; blk * 32 < N; blk += t.nwarps) {
    const int i = blk * 32 + t.lane;
    const bool in = i < N;
    uint64_t k = in ? keys[i] : 0ull;
    int32_t v = in ? vals[i] : -1;
    for (int size = size_lo; size <= size_hi; size <<= 1) {
      const int s0 = size == size_lo ? first_stride : (size >> 1);
      for (int stride = s0; stride > 0; stride >>= 1) {
        const uint64_t pk = __shfl_xor_sync(0xFFFFFFFFu, k, stride);
        const int32_t pv = __shfl_xor_sync(0xFFFFFFFFu, v, stride);
        const bool lower = (t.lane & stride) == 0;
        const bool desc = (i & size) == 0;
        const bool take = (lower == desc) ? (pk > k) : (pk < k);
        if (take) {
          k = pk;
          v = pv;
        }
      }
    }
    if (in) {
      keys[i] = k;
      vals[i] = v;
    }
  }
}

__device__ inline void cta_bitonic_desc(const Team& t, uint64_t* keys, int32_t* vals, int N) {
  if (N < 2) return;
  // Sizes 2 .. min(N, 32): entirely inside warps.
  bitonic_warp_block(t, keys, vals, N, 2, N < 32 ? N : 32, 1);
  team_sync(t);
  for (int size = 64; size <= N; size <<= 1) {
    for (int stride = size >> 1; stride >= 32; stride >>= 1) {
      for (int i = t.tid; i < (N >> 1); i += t.T) {
        const int lo = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));
        const int hi = lo + stride;
        const uint64_t ka = keys[lo], kb = keys[hi];
        const bool desc = (lo & size) == 0;
        if (desc ? (ka < kb) : (ka > kb)) {
          keys[lo] = kb;
          keys[hi] = ka;
          const int32_t va = vals[lo];
          vals[lo] = vals[hi];
          vals[hi] = va;
        }
      }
      team_sync(t);
    }
    bitonic_warp_block(t, keys, vals, N, size, size, 16);
    team_sync(t);
  }
}

// ------------------------------------------------------------ rank merge
// Entries with values: nseg lists (list s holds count(s) entries).
struct WarpListSrc {  // warp buffers in shared memory, stride cw
  static constexpr bool kFlat = false;
  const uint64_t* keys;
  const int32_t* vals;
  int cw;
  const int* counts;
  int nseg;
  __device__ __forceinline__ int count(int s) const { return counts[s]; }
  __device__ __forceinline__ uint64_t key(int s, int i) const { return keys[s * cw + i]; }
  __device__ __forceinline__ int32_t val(int s, int i) const { return vals[s * cw + i]; }
};
struct PartialListSrc {  // one request's partial lists in global memory, stride n
  static constexpr bool kFlat = true;
  const unsigned long long* keys;
  const int32_t* vals;
  int n;
  const int* segoff;  // shared: list s holds segoff[s+1] - segoff[s] entries
  int nseg;
  __device__ __forceinline__ int total() const { return segoff[nseg]; }
  // Position in global memory of flat entry i (list found by binary search).
  __device__ __forceinline__ size_t at(int i) const {
    int lo = 0, hi = nseg;  // segoff[lo] <= i < segoff[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (segoff[mid] <= i) lo = mid; else hi = mid;
    }
    return static_cast<size_t>(lo) * n + (i - segoff[lo]);
  }
  __device__ __forceinline__ int count(int s) const { return segoff[s + 1] - segoff[s]; }
  __device__ __forceinline__ uint64_t key(int s, int i) const {
    return __ldcg(keys + static_cast<size_t>(s) * n + i);
  }
  __device__ __forceinline__ int32_t val(int s, int i) const {
    return __ldcg(vals + static_cast<size_t>(s) * n + i);
  }
};

// Compare budget of the in-bin ranking (sum over bins of count^2).
constexpr uint32_t kRankWorkLimit = 1u << 18;

// Ranks the entries of `src` by the complete score histogram `hist` (see the
// header) and hands ranks 0..n-1 to `out`. Returns false, having written
// nothing, when the entries must be selected and sorted instead (a crowded
// bin, too little staging room, or entries that do not match the histogram).
// P and cur: 1024 words of shared scratch each; stk/stv: `cap` staging slots.
// All team threads call it; the result is the same for all of them.
template <class Src, class Writer>
__device__ bool rank_merge(const Team& t, SelCtl* ctl, const uint32_t* hist, const Src& src,
                           uint32_t n, int r, float C, uint64_t* stk, int32_t* stv, int cap,
                           uint32_t* P, uint32_t* cur, const Writer& out) {
  // 1. Exclusive prefix counts P (each thread a contiguous chunk of bins),
  //    the bin bK of the n-th best, and the in-bin compare work.
  const int per = (kHistBins + t.T - 1) / t.T;
  const int b0 = t.tid * per;
  const int b1 = b0 + per < kHistBins ? b0 + per : kHistBins;
  uint32_t mine = 0;
  for (int b = b0; b < b1; ++b) mine += hist[b];
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (t.lane >= o) incl += y;
  }
  if (t.lane == 31) ctl->red[t.warp] = incl;
  if (t.tid == 0) {
    ctl->bcast_d = kHistBins;
    ctl->bcast_cnt = 0u;
    ctl->rank_bad = 0;
  }
  team_sync(t);
  uint32_t base = incl - mine;
  for (int w = 0; w < t.warp; ++w) base += static_cast<uint32_t>(ctl->red[w]);
  for (int b = b0; b < b1; ++b) {
    const uint32_t c = hist[b];
    P[b] = base;
    cur[b] = 0u;
    if (base + c >= n) {
      atomicMin(&ctl->bcast_d, b);
      break;  // the bins after this one are below bK: never needed
    }
    base += c;
  }
  team_sync(t);
  int bK = ctl->bcast_d;
  if (bK >= kHistBins) bK = kHistBins - 1;  // fewer than n candidates: all of them rank
  {
    uint32_t work = 0;
    for (int b = b0; b < b1 && b <= bK; ++b) {
      const uint32_t c = hist[b] < 4096u ? hist[b] : 4096u;
      work += c * c;
    }
    work = warp_sum_u(work);
    if (t.lane == 0 && work) atomicAdd(&ctl->bcast_cnt, work);
  }
  team_sync(t);
  const uint32_t total = P[bK] + hist[bK];
  if (total > static_cast<uint32_t>(cap) || ctl->bcast_cnt > kRankWorkLimit) return false;
  for (int i = t.tid; i < static_cast<int>(total); i += t.T) stk[i] = 0ull;
  team_sync(t);
  // 2. Scatter the entries of bins 0..bK into their bins' slot ranges.
  auto place = [&](uint64_t key, int32_t val) {
    if (key == 0ull) return;
    const uint32_t b = score_bin(key_score(key), C);
    if (b > static_cast<uint32_t>(bK)) return;
    const uint32_t slot = P[b] + atomicAdd(&cur[b], 1u);
    if (slot < P[b] + hist[b]) {
      stk[slot] = key;
      stv[slot] = val;
    } else {
      ctl->rank_bad = 1;
    }
  };
  if constexpr (Src::kFlat) {
    // Global lists: eight independent loads per thread before any use.
    constexpr int kU = 8;
    const int M = src.total();
    for (int base_i = 0; base_i < M; base_i += kU * t.T) {
      uint64_t key[kU];
      int32_t val[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = base_i + u * t.T + t.tid;
        key[u] = 0ull;
        val[u] = -1;
        if (i < M) {
          const size_t at = src.at(i);
          key[u] = __ldcg(src.keys + at);
          val[u] = __ldcg(src.vals + at);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) place(key[u], val[u]);
    }
  } else {
    for (int s = 0; s < src.nseg; ++s) {
      const int c = src.count(s);
      for (int i = t.tid; i < c; i += t.T) place(src.key(s, i), src.val(s, i));
    }
  }
  team_sync(t);
  // Every bin above bK must be complete (all its candidates rank < n).
  for (int b = t.tid; b < bK; b += t.T)
    if (cur[b] != hist[b]) ctl->rank_bad = 1;
  team_sync(t);
  if (ctl->rank_bad) return false;
  // 3. Rank = entries in the bins above + larger keys of the same bin.
  const int filled = static_cast<int>(P[bK] + cur[bK]);
  for (int i = t.tid; i < filled; i += t.T) {
    const uint64_t key = stk[i];
    const uint32_t b = score_bin(key_score(key), C);
    const uint32_t lo = P[b], hi = lo + cur[b];
    uint32_t rank = lo;
    for (uint32_t j = lo; j < hi; ++j) rank += stk[j] > key ? 1u : 0u;
    if (rank < n) out(r, static_cast<int>(rank), key, stv[i], true);
  }
  for (int i = (filled < static_cast<int>(n) ? filled : static_cast<int>(n)) + t.tid;
       i < static_cast<int>(n); i += t.T)
    out(r, i, 0ull, -1, false);
  return true;
}

// ------------------------------------------------------------ warp buffers
struct WarpBuf {
  uint64_t* keys;   // [cw] shared
  int32_t* vals;    // [cw] shared
  uint32_t* hist;   // [256] shared, radix-select scratch
  int cw;
  int count;        // warp-uniform
  uint64_t thr;     // warp-uniform: candidates need key >= thr
  int binned;       // warp-uniform: candidates counted in the CTA histogram since the last refresh
};

// Candidates counted by this warp in the CTA histogram before it rescans it.
constexpr int kRefreshAfter = 32;

// Where a warp publishes its thresholds.
struct ThrSinks {
  unsigned long long* cta_thr;     // shared
  unsigned long long* request_thr; // global, may be null
};

__device__ __forceinline__ void publish_thr(uint64_t K, int lane, const ThrSinks& sinks) {
  if (lane == 0) {
    atomicMax(sinks.cta_thr, static_cast<unsigned long long>(K));
    if (sinks.request_thr) atomicMax(sinks.request_thr, static_cast<unsigned long long>(K));
  }
}

// Keep the n best of the buffer (count > n), raise and publish the threshold.
__device__ __forceinline__ void warp_compact(WarpBuf& wb, uint32_t n, int lane,
                                             const ThrSinks& sinks) {
  __syncwarp();
  const uint64_t K = warp_select(wb.keys, wb.count, n, wb.hist, lane);
  __syncwarp();
  int out = 0;
  for (int base = 0; base < wb.count; base += 32) {
    const int i = base + lane;
    const bool keep = i < wb.count && wb.keys[i] >= K;
    const uint64_t k = keep ? wb.keys[i] : 0ull;
    const int32_t v = keep ? wb.vals[i] : 0;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
    __syncwarp();
    if (keep) {
      const int pos = out + __popc(bal & lanemask_lt());
      wb.keys[pos] = k;
      wb.vals[pos] = v;
    }
    out += __popc(bal);
    __syncwarp();
  }
  wb.count = out;
  if (K > wb.thr) wb.thr = K;
  publish_thr(K, lane, sinks);
  __syncwarp();
}

// warp_compact behind a call (for code that offers from many unrolled sites:
// the rare compaction then exists once instead of once per site).
struct CompactOut {
  uint64_t thr;
  int count;
};
static __device__ __noinline__ CompactOut warp_compact_call(uint64_t* keys, int32_t* vals, uint32_t* hist,
                                                     int cw, int count, uint64_t thr, uint32_t n,
                                                     int lane, unsigned long long* cta_thr,
                                                     unsigned long long* request_thr) {
  WarpBuf wb{keys, vals, hist, cw, count, thr, 0};
  warp_compact(wb, n, lane, ThrSinks{cta_thr, request_thr});
  return CompactOut{wb.thr, wb.count};
}

// warp_offer with the compaction behind a call.
__device__ __forceinline__ void warp_offer_nc(WarpBuf& wb, bool valid, uint64_t key, int32_t val,
                                              uint32_t n, int lane, const ThrSinks& sinks) {
  bool pass = valid && key >= wb.thr;
  unsigned bal = __ballot_sync(0xFFFFFFFFu, pass);
  if (bal == 0) return;
  int cnt = __popc(bal);
  if (wb.count + cnt > wb.cw) {
    const CompactOut c = warp_compact_call(wb.keys, wb.vals, wb.hist, wb.cw, wb.count, wb.thr, n,
                                           lane, sinks.cta_thr, sinks.request_thr);
    wb.count = c.count;
    wb.thr = c.thr;
    pass = pass && key >= wb.thr;
    bal = __ballot_sync(0xFFFFFFFFu, pass);
    cnt = __popc(bal);
  }
  if (pass) {
    const int pos = wb.count + __popc(bal & lanemask_lt());
    wb.keys[pos] = key;
    wb.vals[pos] = val;
  }
  wb.count += cnt;
}

// Offer one candidate per lane (only lanes with valid = true). Warp-collective:
// every lane of the warp must call it with the same wb state.
__device__ __forceinline__ void warp_offer(WarpBuf& wb, bool valid, uint64_t key, int32_t val,
                                           uint32_t n, int lane, const ThrSinks& sinks) {
  bool pass = valid && key >= wb.thr;
  unsigned bal = __ballot_sync(0xFFFFFFFFu, pass);
  if (bal == 0) return;
  int cnt = __popc(bal);
  if (wb.count + cnt > wb.cw) {  // then count > cw - 32 >= n: compaction is possible
    warp_compact(wb, n, lane, sinks);
    pass = pass && key >= wb.thr;
    bal = __ballot_sync(0xFFFFFFFFu, pass);
    cnt = __popc(bal);
  }
  if (pass) {
    const int pos = wb.count + __popc(bal & lanemask_lt());
    wb.keys[pos] = key;
    wb.vals[pos] = val;
  }
  wb.count += cnt;
}

// Raise the warp threshold from the CTA histogram and the CTA-wide bound
// (the request-wide bound is read once per row by the caller, not here, to
// keep an L2 round trip off this path). Warp-collective.
__device__ __forceinline__ void refresh_thr(WarpBuf& wb, SelCtl* ctl, uint32_t n, float C,
                                            int lane, const ThrSinks& sinks) {
  if ((wb.binned < kRefreshAfter && wb.thr != 0ull) ||
      *reinterpret_cast<volatile unsigned*>(&ctl->hist_total) < n) {
    const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
    if (c > wb.thr) wb.thr = c;
    return;
  }
  wb.binned = 0;
  const uint64_t hb = hist_bound(ctl->hist, n, C, lane);
  const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
  uint64_t t = wb.thr;
  if (c > t) t = c;
  if (hb > t) {
    t = hb;
    publish_thr(hb, lane, sinks);
  }
  wb.thr = t;
}

// ------------------------------------------------------------ segment end
// Everything a CTA needs to hand its segment of request r over.
struct FlushArgs {
  int n;                  // beams (or K) to select per request
  int r;                  // request of the segment
  int k;                  // this CTA's contributor index for request r
  int G;                  // contributors of request r
  int maxG;               // partial-list slots per request
  int pcap;               // capacity (and stride) of one partial list
  unsigned long long* part_keys;  // [R][maxG][pcap]
  int32_t* part_vals;             // [R][maxG][pcap]
  uint32_t* part_count;           // [R][maxG]
  uint32_t* tickets;              // [R]
  unsigned long long* request_thr;  // [R]
  uint32_t* ghist;                // [R][kHistBins]
  float C;                        // histogram reference score of request r
  const uint64_t* wkeys;  // all warp buffers, [nwarps][cw]
  int cw;
  uint64_t* sort_keys;    // shared scratch for the final sort (aliases the warp buffers)
  int32_t* sort_vals;
  int sort_cap;           // entries available at sort_keys / sort_vals
  uint32_t* radix_hist;   // 256-word scratch for cta_select
  int32_t* wvals;         // all warp buffers' values, [nwarps][cw]
  uint32_t* rank_P;       // 1024-word scratch for the rank merge (null: no rank merge)
  uint32_t* rank_cur;     // 1024-word scratch for the rank merge
  uint64_t* direct_keys;  // staging for ranking a whole request held by this CTA
  int32_t* direct_vals;   //   (null when no free area is available)
  int direct_cap;
};

// Warp-aggregated append position: this lane's slot among the `keep` lanes.
__device__ __forceinline__ int append_pos(int* counter, bool keep, int lane) {
  const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
  int base = 0;
  if (lane == 0 && bal) base = atomicAdd(counter, __popc(bal));
  base = __shfl_sync(0xFFFFFFFFu, base, 0);
  return base + __popc(bal & lanemask_lt());
}

// The last contributor of request r: bound from the complete histogram, copy
// the partial entries above it into shared memory, select the n best, sort
// them and hand each rank to `out(r, rank, key, val, valid)`.
template <class Writer>
__device__ void request_merge(const Team& t, SelCtl* ctl, const FlushArgs& f, const Writer& out) {
  const int G = f.G < kMaxSegCounts ? f.G : kMaxSegCounts;
  const size_t list0 = static_cast<size_t>(f.r) * f.maxG;
  // The CTA histogram area now receives the request's complete histogram.
  uint32_t* gh = f.ghist + static_cast<size_t>(f.r) * kHistBins;
  for (int i = t.tid; i < kHistBins; i += t.T) ctl->hist[i] = __ldcg(gh + i);
  for (int k = t.tid; k < G; k += t.T) {
    const int c = static_cast<int>(__ldcg(f.part_count + list0 + k));
    ctl->segoff[k + 1] = c < f.pcap ? c : f.pcap;
  }
  team_sync(t);
  if (t.warp == 0) {  // exclusive prefix sum of the list sizes
    int carry = 0;
    for (int k0 = 0; k0 < G; k0 += 32) {
      const int k = k0 + t.lane;
      const int c = k < G ? ctl->segoff[k + 1] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (t.lane >= o) incl += y;
      }
      if (k < G) ctl->segoff[k + 1] = carry + incl;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (t.lane == 0) {
      ctl->segoff[0] = 0;
      ctl->counter = 0;
    }
  }
  team_sync(t);
  {
    const unsigned long long* lists0 = f.part_keys + list0 * f.pcap;
    const int32_t* lvals0 = f.part_vals + list0 * f.pcap;
    if (f.rank_P &&
        rank_merge(t, ctl, ctl->hist, PartialListSrc{lists0, lvals0, f.pcap, ctl->segoff, G},
                   static_cast<uint32_t>(f.n), f.r, f.C, f.sort_keys, f.sort_vals, f.sort_cap,
                   f.rank_P, f.rank_cur, out)) {
      for (int i = t.tid; i < kHistBins; i += t.T) gh[i] = 0u;
      if (t.tid == 0) {
        f.tickets[f.r] = 0u;
        f.request_thr[f.r] = 0ull;
      }
      return;
    }
  }
  team_sync(t);
  if (t.warp == 0) {
    const uint64_t hb = hist_bound(ctl->hist, static_cast<uint32_t>(f.n), f.C, t.lane);
    if (t.lane == 0) {
      const unsigned long long g =
          *reinterpret_cast<volatile unsigned long long*>(f.request_thr + f.r);
      ctl->bcast_key = hb > g ? hb : g;
    }
  }
  team_sync(t);
  const uint64_t K0 = ctl->bcast_key;
  const int total = ctl->segoff[G];
  const unsigned long long* lists = f.part_keys + list0 * f.pcap;
  const int32_t* lvals = f.part_vals + list0 * f.pcap;
  // Filtered copy of all partial entries >= K0 into [0, cap): flat index,
  // segment found by binary search, four independent loads per thread.
  uint64_t* stk = f.sort_keys;
  int32_t* stv = f.sort_vals;
  const int cap = f.sort_cap;
  for (int base = 0; base < total; base += 4 * t.T) {
    uint64_t key[4];
    int32_t val[4];
    bool in[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * t.T + t.tid;
      in[u] = i < total;
      key[u] = 0ull;
      val[u] = -1;
      if (in[u]) {
        int lo = 0, hi = G;  // segoff[lo] <= i < segoff[hi]
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (ctl->segoff[mid] <= i) lo = mid; else hi = mid;
        }
        const size_t at = static_cast<size_t>(lo) * f.pcap + (i - ctl->segoff[lo]);
        key[u] = __ldcg(lists + at);
        val[u] = __ldcg(lvals + at);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bool keep = in[u] && key[u] >= K0 && key[u] != 0ull;
      const int pos = append_pos(&ctl->counter, keep, t.lane);
      if (keep && pos < cap) {
        stk[pos] = key[u];
        stv[pos] = val[u];
      }
    }
  }
  team_sync(t);
  int M = ctl->counter;
  if (M > cap) {
    // The bound left more entries than shared memory holds (a poor histogram
    // reference): select straight from the lists in L2 instead.
    M = total;
    const int sel_all = M < f.n ? M : f.n;
    int N_all = 1;
    while (N_all < sel_all) N_all <<= 1;
    uint64_t Kg = 0;
    if (M > f.n)
      Kg = cta_select(t, PartialSrc{lists, f.pcap, ctl->segoff, G}, f.n, f.radix_hist, ctl);
    if (t.tid == 0) ctl->counter = 0;
    for (int i = t.tid; i < N_all; i += t.T) {
      stk[i] = 0ull;
      stv[i] = -1;
    }
    team_sync(t);
    for (int base = 0; base < total; base += t.T) {
      const int i = base + t.tid;
      uint64_t key = 0ull;
      int32_t val = -1;
      if (i < total) {
        int lo = 0, hi = G;
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (ctl->segoff[mid] <= i) lo = mid; else hi = mid;
        }
        const size_t at = static_cast<size_t>(lo) * f.pcap + (i - ctl->segoff[lo]);
        key = __ldcg(lists + at);
        val = __ldcg(lvals + at);
      }
      const bool keep = i < total && key >= Kg && key != 0ull;
      const int pos = append_pos(&ctl->counter, keep, t.lane);
      if (keep && pos < N_all) {
        stk[pos] = key;
        stv[pos] = val;
      }
    }
    team_sync(t);
    cta_bitonic_desc(t, stk, stv, N_all);
    for (int i = t.tid; i < f.n; i += t.T) {
      const bool valid = i < sel_all;
      out(f.r, i, valid ? stk[i] : 0ull, valid ? stv[i] : -1, valid);
    }
    for (int i = t.tid; i < kHistBins; i += t.T) gh[i] = 0u;
    if (t.tid == 0) {
      f.tickets[f.r] = 0u;
      f.request_thr[f.r] = 0ull;
    }
    return;
  }
  const int sel = M < f.n ? M : f.n;
  int N = 1;
  while (N < sel) N <<= 1;
  uint64_t K = 0;
  if (M > f.n) {
    if (t.tid == 0) ctl->staged = M;
    team_sync(t);
    K = cta_select(t, WarpBufSrc{stk, 0, &ctl->staged, 1}, f.n, f.radix_hist, ctl);
  }
  // Sort buffer: behind the staged entries if they fit, else the staged entries
  // themselves (keys below K zeroed: they sort last).
  uint64_t* sk = stk;
  int32_t* sv = stv;
  const int m32 = (M + 31) & ~31;
  if (M > f.n && m32 + N <= cap) {
    sk = stk + m32;
    sv = stv + m32;
    if (t.tid == 0) ctl->counter = 0;
    for (int i = t.tid; i < N; i += t.T) {
      sk[i] = 0ull;
      sv[i] = -1;
    }
    team_sync(t);
    for (int base = 0; base < M; base += t.T) {
      const int i = base + t.tid;
      const bool keep = i < M && stk[i] >= K;
      const int pos = append_pos(&ctl->counter, keep, t.lane);
      if (keep && pos < N) {
        sk[pos] = stk[i];
        sv[pos] = stv[i];
      }
    }
  } else {
    const int span = N > M ? N : M;
    for (int i = t.tid; i < span; i += t.T) {
      if (i >= M || stk[i] < K) {
        stk[i] = 0ull;
        stv[i] = -1;
      }
    }
  }
  team_sync(t);
  if (sk == stk && M > N) {
    // Entries above K are scattered over [0, M): pack them into [0, N) first.
    // (Only reached when the staging area had no room for a second buffer.)
    if (t.tid == 0) {
      int w = 0;
      for (int i = 0; i < M; ++i)
        if (stk[i] != 0ull) {
          stk[w] = stk[i];
          stv[w] = stv[i];
          ++w;
        }
      for (int i = w; i < M; ++i) {
        stk[i] = 0ull;
        stv[i] = -1;
      }
    }
    team_sync(t);
  }
  cta_bitonic_desc(t, sk, sv, N);
  const uint64_t* ok_keys = sk;
  const int32_t* ok_vals = sv;
  for (int i = t.tid; i < f.n; i += t.T) {
    const bool valid = i < sel;
    out(f.r, i, valid ? ok_keys[i] : 0ull, valid ? ok_vals[i] : -1, valid);
  }
  // Leave the request's histogram, ticket and bound zeroed for the next call.
  for (int i = t.tid; i < kHistBins; i += t.T) gh[i] = 0u;
  if (t.tid == 0) {
    f.tickets[f.r] = 0u;
    f.request_thr[f.r] = 0ull;
  }
}

// End of a request segment for this CTA (all consumer warps call it).
// Returns true when the CTA must stop (an abort was seen by any warp).
template <class Writer>
__device__ bool segment_flush(const Team& t, WarpBuf& wb, SelCtl* ctl, const FlushArgs& f,
                              const Writer& out) {
  if (t.lane == 0) ctl->wcount[t.warp] = wb.count;
  if (team_sync_or(t, ctl->abort_flag != 0)) return true;
  if (f.G == 1 && f.direct_keys && f.rank_P &&
      rank_merge(t, ctl, ctl->hist, WarpListSrc{f.wkeys, f.wvals, f.cw, ctl->wcount, t.nwarps},
                 static_cast<uint32_t>(f.n), f.r, f.C, f.direct_keys, f.direct_vals,
                 f.direct_cap, f.rank_P, f.rank_cur, out)) {
    team_sync(t);
    for (int i = t.tid; i < kHistBins; i += t.T) ctl->hist[i] = 0u;
    wb.count = 0;
    wb.thr = 0;
    if (t.tid == 0) {
      ctl->cta_thr = 0ull;
      ctl->hist_total = 0u;
      f.request_thr[f.r] = 0ull;
    }
    team_sync(t);
    return false;
  }
  // 1. Add this segment's histogram to the request's (read back only by the
  //    merging CTA); bound the flush by this CTA's histogram and the shared bounds.
  uint32_t* gh = f.ghist + static_cast<size_t>(f.r) * kHistBins;
  for (int i = t.tid; i < kHistBins; i += t.T) {
    const uint32_t c = ctl->hist[i];
    if (c) atomicAdd(gh + i, c);
  }
  if (t.warp == 0) {
    const uint64_t hb = hist_bound(ctl->hist, static_cast<uint32_t>(f.n), f.C, t.lane);
    if (t.lane == 0) {
      const unsigned long long g =
          *reinterpret_cast<volatile unsigned long long*>(f.request_thr + f.r);
      const unsigned long long c = ctl->cta_thr;
      unsigned long long K = hb;
      if (g > K) K = g;
      if (c > K) K = c;
      ctl->bcast_key = K;
      ctl->counter = 0;
    }
  }
  team_sync(t);
  uint64_t K = ctl->bcast_key;
  // 2. Entries above the bound; cut to the CTA's n best if there are more.
  {
    int ge = 0;
    for (int base = 0; base < wb.count; base += 32) {
      const int i = base + t.lane;
      ge += __popc(__ballot_sync(0xFFFFFFFFu, i < wb.count && wb.keys[i] >= K));
    }
    if (t.lane == 0 && ge) atomicAdd(&ctl->counter, ge);
  }
  team_sync(t);
  if (ctl->counter > f.pcap) {  // more survivors than the list holds: keep the n best
    const uint64_t Kc = cta_select(t, WarpBufSrc{f.wkeys, f.cw, ctl->wcount, t.nwarps}, f.n,
                                   f.radix_hist, ctl);
    if (Kc > K) K = Kc;
    if (t.tid == 0) atomicMax(f.request_thr + f.r, static_cast<unsigned long long>(K));
  }
  team_sync(t);
  if (t.tid == 0) ctl->counter = 0;
  team_sync(t);
  const size_t slot = (static_cast<size_t>(f.r) * f.maxG + f.k) * f.pcap;
  for (int base = 0; base < wb.count; base += 32) {
    const int i = base + t.lane;
    const bool keep = i < wb.count && wb.keys[i] >= K;
    const int pos = append_pos(&ctl->counter, keep, t.lane);
    if (keep && pos < f.pcap) {
      f.part_keys[slot + pos] = wb.keys[i];
      f.part_vals[slot + pos] = wb.vals[i];
    }
  }
  __threadfence();  // every thread's histogram adds and list writes, before the ticket
  team_sync(t);
  // 3. Ticket; the last contributor merges the request.
  if (t.tid == 0) {
    const int c = ctl->counter < f.pcap ? ctl->counter : f.pcap;
    f.part_count[static_cast<size_t>(f.r) * f.maxG + f.k] = static_cast<uint32_t>(c);
    __threadfence();
    const unsigned tk = atomicAdd(f.tickets + f.r, 1u);
    ctl->is_last = (tk == static_cast<unsigned>(f.G - 1)) ? 1 : 0;
  }
  team_sync(t);
  if (ctl->is_last) {
    __threadfence();
    request_merge(t, ctl, f, out);
    team_sync(t);
  }
  // 4. Reset for the next segment.
  for (int i = t.tid; i < kHistBins; i += t.T) ctl->hist[i] = 0u;
  wb.count = 0;
  wb.thr = 0;
  if (t.tid == 0) {
    ctl->cta_thr = 0ull;
    ctl->hist_total = 0u;
  }
  team_sync(t);
  return false;
}

}  // namespace dev
}  // namespace sidbeam
