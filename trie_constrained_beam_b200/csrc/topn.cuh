// Exact per-request top-n selection on 64-bit keys, shared by beam_step and
// catalog_score_topk.
//
// Keys are unique (score in the high half, 2^32-1-idx in the low half), so
// "the n largest keys" is a set with no ties, and "key >= K" for a threshold K
// found by an MSB-first radix walk selects exactly n of them.
//
// Three levels, all exact:
//  1. warp: candidates above the warp's threshold are appended to a
//     shared-memory buffer of Cw >= n + 32 entries; when it is full, the warp
//     finds the n-th largest key K by a radix walk, keeps the n keys >= K and
//     raises its threshold to K. Any such K is a lower bound on the request's
//     n-th best key, so it is also published CTA-wide (shared memory) and
//     request-wide (a global atomicMax) for other warps and CTAs to filter with.
//  2. CTA (at the end of a request segment): the union of the warp buffers is
//     cut to its n best, filtered by the request-wide bound, and written to the
//     CTA's slot of a per-request partial list in global memory.
//  3. request: the CTA that takes the last ticket of the request (a
//     threadfence + atomic counter; nothing ever spins) selects the n best of
//     all partial lists, sorts them (bitonic, descending) and writes them out.
//     It then zeroes the ticket and the request bound for the next call.
#pragma once

#include "device_utils.cuh"

namespace sidbeam {
namespace dev {

constexpr int kBarConsumers = 1;  // named barrier id used by the consumer warps
constexpr int kMaxSegCounts = 1024;

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

// Threshold K with exactly `need` keys >= K among keys[0..count) (count > need >= 1).
// Warp-collective; hist = 256 words of this warp's shared memory.
__device__ inline uint64_t warp_select(const uint64_t* keys, int count, uint32_t need, uint32_t* hist,
                                int lane) {
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
    for (int i = lane; i < count; i += 32) {
      const uint64_t k = keys[i];
      const bool match = hi >= 64 || ((k >> hi) == (prefix >> hi));
      if (match) atomicAdd(&hist[static_cast<uint32_t>(k >> lo) & dmask], 1u);
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

// Shared-memory control block of the selection (one per CTA).
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
  int wcount[32];
  int segcnt[kMaxSegCounts];
};

// Key sources for the CTA-level select.
struct WarpBufSrc {
  const uint64_t* keys;  // [nwarps][cw]
  int cw;
  const int* counts;     // shared
  int nseg;
  __device__ __forceinline__ int count(int s) const { return counts[s]; }
  __device__ __forceinline__ uint64_t key(int s, int i) const { return keys[s * cw + i]; }
};
struct PartialSrc {
  const unsigned long long* keys;  // partial lists of one request: [maxG][n]
  int n;
  const int* counts;               // shared copy of the list sizes
  int nseg;
  __device__ __forceinline__ int count(int s) const { return counts[s]; }
  __device__ __forceinline__ uint64_t key(int s, int i) const {
    return __ldcg(keys + static_cast<size_t>(s) * n + i);
  }
};

// CTA-level threshold: K with exactly `need` keys >= K over all segments of src
// (total > need >= 1). All consumer threads call it; uses team_sync.
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
      for (int i = t.tid; i < c; i += t.T) {
        const uint64_t k = src.key(s, i);
        const bool match = hi >= 64 || ((k >> hi) == (prefix >> hi));
        if (match) atomicAdd(&hist[static_cast<uint32_t>(k >> lo) & dmask], 1u);
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
// descending key order.
__device__ inline void cta_bitonic_desc(const Team& t, uint64_t* keys, int32_t* vals, int N) {
  for (int size = 2; size <= N; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
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
  }
}

// Per-warp candidate buffer.
struct WarpBuf {
  uint64_t* keys;   // [cw] shared
  int32_t* vals;    // [cw] shared
  uint32_t* hist;   // [256] shared
  int cw;
  int count;        // warp-uniform
  uint64_t thr;     // warp-uniform: candidates need key >= thr
};

// Where a warp publishes its thresholds.
struct ThrSinks {
  unsigned long long* cta_thr;     // shared
  unsigned long long* request_thr; // global, may be null
};

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
  if (lane == 0) {
    atomicMax(sinks.cta_thr, static_cast<unsigned long long>(K));
    if (sinks.request_thr) atomicMax(sinks.request_thr, static_cast<unsigned long long>(K));
  }
  __syncwarp();
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

// Everything a CTA needs to hand its segment of request r over.
struct FlushArgs {
  int n;                  // beams (or K) to select per request
  int r;                  // request of the segment
  int k;                  // this CTA's contributor index for request r
  int G;                  // contributors of request r
  int maxG;               // partial-list slots per request
  unsigned long long* part_keys;  // [R][maxG][n]
  int32_t* part_vals;             // [R][maxG][n]
  uint32_t* part_count;           // [R][maxG]
  uint32_t* tickets;              // [R]
  unsigned long long* request_thr;  // [R]
  const uint64_t* wkeys;  // all warp buffers, [nwarps][cw]
  int cw;
  uint64_t* sort_keys;    // shared scratch for the final sort (aliases the warp buffers)
  int32_t* sort_vals;
};

// The last contributor of request r: select the n best of all partial lists,
// sort them and hand each rank to `out(r, rank, key, val, valid)`.
template <class Writer>
__device__ void request_merge(const Team& t, SelCtl* ctl, uint32_t* hist, const FlushArgs& f,
                              const Writer& out) {
  const int G = f.G < kMaxSegCounts ? f.G : kMaxSegCounts;
  const size_t list0 = static_cast<size_t>(f.r) * f.maxG;
  for (int k = t.tid; k < G; k += t.T) {
    const int c = static_cast<int>(__ldcg(f.part_count + list0 + k));
    ctl->segcnt[k] = c < f.n ? c : f.n;
  }
  team_sync(t);
  int M = 0;
  for (int k = 0; k < G; ++k) M += ctl->segcnt[k];
  const unsigned long long* lists = f.part_keys + list0 * f.n;
  const int32_t* lvals = f.part_vals + list0 * f.n;
  uint64_t K = 0;
  if (M > f.n) K = cta_select(t, PartialSrc{lists, f.n, ctl->segcnt, G}, f.n, hist, ctl);
  const int sel = M < f.n ? M : f.n;
  int N = 1;
  while (N < sel) N <<= 1;
  for (int i = t.tid; i < N; i += t.T) {
    f.sort_keys[i] = 0ull;
    f.sort_vals[i] = -1;
  }
  if (t.tid == 0) ctl->counter = 0;
  team_sync(t);
  for (int k = 0; k < G; ++k) {
    const int c = ctl->segcnt[k];
    for (int i = t.tid; i < c; i += t.T) {
      const uint64_t key = __ldcg(lists + static_cast<size_t>(k) * f.n + i);
      if (key >= K) {
        const int pos = atomicAdd(&ctl->counter, 1);
        if (pos < N) {
          f.sort_keys[pos] = key;
          f.sort_vals[pos] = __ldcg(lvals + static_cast<size_t>(k) * f.n + i);
        }
      }
    }
  }
  team_sync(t);
  cta_bitonic_desc(t, f.sort_keys, f.sort_vals, N);
  for (int i = t.tid; i < f.n; i += t.T) {
    const bool valid = i < sel;
    out(f.r, i, valid ? f.sort_keys[i] : 0ull, valid ? f.sort_vals[i] : -1, valid);
  }
}

// End of a request segment for this CTA (all consumer warps call it).
// Returns true when the CTA must stop (an abort was seen by any warp).
template <class Writer>
__device__ bool segment_flush(const Team& t, WarpBuf& wb, SelCtl* ctl, uint32_t* hist,
                              const FlushArgs& f, const Writer& out) {
  if (t.lane == 0) ctl->wcount[t.warp] = wb.count;
  if (team_sync_or(t, ctl->abort_flag != 0)) return true;
  int total = 0;
  for (int w = 0; w < t.nwarps; ++w) total += ctl->wcount[w];
  uint64_t K = 0;
  if (total > f.n)
    K = cta_select(t, WarpBufSrc{f.wkeys, f.cw, ctl->wcount, t.nwarps}, f.n, hist, ctl);
  if (t.tid == 0) {
    unsigned long long old;
    if (total > f.n)
      old = atomicMax(f.request_thr + f.r, static_cast<unsigned long long>(K));
    else
      old = *reinterpret_cast<volatile unsigned long long*>(f.request_thr + f.r);
    ctl->bcast_key = old > K ? old : K;
    ctl->counter = 0;
  }
  team_sync(t);
  K = ctl->bcast_key;
  const size_t slot = (static_cast<size_t>(f.r) * f.maxG + f.k) * f.n;
  for (int base = 0; base < wb.count; base += 32) {
    const int i = base + t.lane;
    const bool keep = i < wb.count && wb.keys[i] >= K;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
    int pos0 = 0;
    if (t.lane == 0 && bal) pos0 = atomicAdd(&ctl->counter, __popc(bal));
    pos0 = __shfl_sync(0xFFFFFFFFu, pos0, 0);
    if (keep) {
      const int pos = pos0 + __popc(bal & lanemask_lt());
      if (pos < f.n) {
        f.part_keys[slot + pos] = wb.keys[i];
        f.part_vals[slot + pos] = wb.vals[i];
      }
    }
  }
  team_sync(t);
  if (t.tid == 0) {
    const int c = ctl->counter < f.n ? ctl->counter : f.n;
    f.part_count[static_cast<size_t>(f.r) * f.maxG + f.k] = static_cast<uint32_t>(c);
    __threadfence();
    const unsigned tk = atomicAdd(f.tickets + f.r, 1u);
    ctl->is_last = (tk == static_cast<unsigned>(f.G - 1)) ? 1 : 0;
  }
  team_sync(t);
  if (ctl->is_last) {
    __threadfence();
    request_merge(t, ctl, hist, f, out);
    if (t.tid == 0) {
      f.tickets[f.r] = 0u;
      f.request_thr[f.r] = 0ull;
    }
  }
  wb.count = 0;
  wb.thr = 0;
  if (t.tid == 0) ctl->cta_thr = 0ull;
  team_sync(t);
  return false;
}

}  // namespace dev
}  // namespace sidbeam
