// beam_stream: the constrained expansion step (temperature 0) as a streaming
// kernel: every warp streams its own rows from HBM and scores them from
// registers.
//
// flashrec 0.1.0 (PyPI page), Features > Decoding ("SID constraint"): a fused
// kernel restricts every continuation to the catalog trie (dense or CSR);
// Features > Serving ("API"): deterministic top-k at temperature 0.
//
// Design (sm_100a):
//  * One CTA per SM over the row partition of launch.h (a request's rows are
//    spread over a group of CTAs, each taking every G-th parent slot, so that
//    every CTA gets its share of the request's best parents).
//  * The warps of a CTA form teams of K warps; team m takes the CTA's rows m,
//    m + T, m + 2T, ... (T teams). A row is cut into K chunks of at most 8 KB,
//    one per warp of the team, held in registers (16 vectors of 16 bytes per
//    lane); the team combines its partial (max, sum) once per row. K = 1 for
//    rows of up to 8 KB; K grows when the CTA has fewer rows than warps.
//  * Streaming: each warp copies its next D rows' chunks (and their trie data:
//    the chunk's child-bitmask bytes, or the node's child codes) into its own
//    shared-memory stages with 16-byte cp.async copies while it computes the
//    current row; a stage is refilled as soon as its row is in registers.
//    Nothing waits on another warp's copies.
//  * Per row: max with packed bf16 max, then sum 2^(z log2e - m log2e) with
//    packed fp32 FMA/add and ex2.approx, each lane against its own max; lanes
//    and team warps are combined once: lse = m + log(sum).
//  * Candidates: a child c is kept with key = (ordered fp32 score s + (z_c -
//    lse)) << 32 | (2^32-1 - (b V + c)) when it reaches a threshold that is
//    always a valid lower bound on the request's n-th best key (topn.cuh).
//    Rows test their lane maxima against the threshold first; rows with hits
//    find them in registers; rows with very many hits count them into the
//    CTA's score histogram first, raise the threshold, then offer.
//  * At the end of a request segment the warps hand their candidates over
//    (topn.cuh: rank merge inside the CTA, or partial lists merged by the
//    request's last CTA).
// The logits are read exactly once from HBM.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"
#include "launch.h"
#include "stream_plan.h"
#include "topn.cuh"

namespace sidbeam {
namespace {

using namespace dev;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kRegVecs = 16;
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr int kOnePassHits = 64;   // rows with more hits are counted first, then offered
constexpr unsigned kPushAfter = 64;
constexpr int kTeamBarBase = 2;    // named barriers 2.. are the teams' (1: all warps)
constexpr int32_t kRowNoTrie = -2; // meta.mrow of a row in the unconstrained mode
constexpr int32_t kRowList = -1;   // meta.mrow of a row whose children come as codes

struct SArgs {
  const uint8_t* logits;
  int64_t row_bytes;  // ld * sizeof(dtype)
  int V;
  const float* parent_scores;
  const int32_t* parent_nodes;
  int R, B_in, n;
  int layout;  // 0 = no trie, SIDBEAM_LAYOUT_DENSE, SIDBEAM_LAYOUT_CSR
  const uint32_t* off;
  const uint32_t* mask;       // dense: [P][stride]; CSR: rows of the nodes with many children
  const int32_t* mask_idx;    // CSR: [P] row of `mask` or -1; null when none
  int mask_stride;            // words per bitmask row (a multiple of 4)
  const uint16_t* codes;      // CSR child codes
  int64_t n_parent;
  float* out_scores;
  int32_t* out_parent;
  int32_t* out_code;
  int32_t* out_node;
  const int32_t* out_width;
  uint32_t* status;
  uint32_t* tickets;
  unsigned long long* request_thr;
  uint32_t* part_count;
  unsigned long long* part_keys;
  int32_t* part_vals;
  uint32_t* ghist;
  Partition part;
  StreamPlan plan;
};

// --------------------------------------------------------------- writer
// Ranks at or past a request's width (out_width) are written as padding: the
// top-w of a request are the first w ranks of its top-n.
struct StepOut {
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
      scores[o] = __int_as_float(0xFF800000);
      parent[o] = -1;
      code[o] = -1;
      node[o] = -1;
    }
  }
};

// --------------------------------------------------------------- row math
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint64_t pk(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float pk_lo(uint64_t p) { return __uint_as_float(static_cast<uint32_t>(p)); }
__device__ __forceinline__ float pk_hi(uint64_t p) {
  return __uint_as_float(static_cast<uint32_t>(p >> 32));
}
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

template <int BF16>
__device__ __forceinline__ float vec_max(const uint4& q) {
  if (BF16) {
    const uint32_t w = bmax2(bmax2(q.x, q.y), bmax2(q.z, q.w));
    return fmaxf(bf_lo(w), bf_hi(w));
  }
  return fmaxf(fmaxf(__uint_as_float(q.x), __uint_as_float(q.y)),
               fmaxf(__uint_as_float(q.z), __uint_as_float(q.w)));
}

// Packed pair of partial sums of 2^(z log2e - m log2e) over the 16 bytes q.
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
template <int BF16>
__device__ __forceinline__ void vec_cut(uint4& x, int keep) {
  uint32_t* w = reinterpret_cast<uint32_t*>(&x);
  if (BF16) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (2 * k >= keep) w[k] = 0xFF80FF80u;
      else if (2 * k + 1 >= keep) w[k] = (w[k] & 0x0000FFFFu) | 0xFF800000u;
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k >= keep) w[k] = 0xFF800000u;
  }
}

// Lane maximum and the lane's sum of 2^((z - lm) log2e) over its vectors
// x[i] (chunk vector lane + 32 i, i < 16; vectors past the chunk are -inf).
// FULL: all 16 vectors of every lane are real (straight-line code).
template <int BF16, bool FULL>
__device__ __forceinline__ void lane_stats(const uint4 (&x)[kRegVecs], int nvec, float& lm,
                                           float& ls) {
  float m;
  if (BF16) {
    uint32_t r = 0xFF80FF80u;
#pragma unroll
    for (int i = 0; i < kRegVecs; ++i)
      if (FULL || 32 * i < nvec) r = bmax2(r, bmax2(bmax2(x[i].x, x[i].y), bmax2(x[i].z, x[i].w)));
    m = fmaxf(bf_lo(r), bf_hi(r));
  } else {
    m = __int_as_float(0xFF800000);
#pragma unroll
    for (int i = 0; i < kRegVecs; ++i)
      if (FULL || 32 * i < nvec) m = fmaxf(m, vec_max<0>(x[i]));
  }
  const float mL = (m > __int_as_float(0xFF800000)) ? m * kLog2e : 0.f;
  const uint64_t l2e = pk(kLog2e, kLog2e);
  const uint64_t nml = pk(-mL, -mL);
  uint64_t a0 = 0, a1 = 0;
#pragma unroll
  for (int i = 0; i < kRegVecs; ++i) {
    if (FULL || 32 * i < nvec) {
      if (i & 1) a1 = fadd2(a1, vec_sumexp2<BF16>(x[i], l2e, nml));
      else a0 = fadd2(a0, vec_sumexp2<BF16>(x[i], l2e, nml));
    }
  }
  const uint64_t a = fadd2(a0, a1);
  lm = m;
  ls = pk_lo(a) + pk_hi(a);
}

// Lane (max, sum) pairs combined over the warp: sum relative to the warp max.
__device__ __forceinline__ void warp_stats(float lm, float ls, float& wm, float& ws) {
  const float mw = warp_max(lm);
  float s = (lm > __int_as_float(0xFF800000)) ? ls * ex2_approx((lm - mw) * kLog2e) : 0.f;
  ws = warp_sum(s);
  wm = mw;
}

// Node id of a dense-row child code c (bit `bit` of the per-warp mask copy):
// first child id + set bits before it.
__device__ __forceinline__ int32_t mask_child(const uint32_t* wm32, const uint32_t* wpre,
                                              uint32_t base, int bit) {
  const uint32_t w = wm32[bit >> 5];
  return static_cast<int32_t>(base + wpre[bit >> 5] + __popc(w & ((1u << (bit & 31)) - 1u)));
}

// Set-bit counts before every word of the per-warp mask copy (warp-collective).
__device__ __forceinline__ void mask_prefix(const uint32_t* wm32, int words, uint32_t* wpre,
                                            int lane) {
  uint32_t carry = 0;
  for (int k0 = 0; k0 < words; k0 += 32) {
    const int k = k0 + lane;
    const uint32_t p = k < words ? static_cast<uint32_t>(__popc(wm32[k])) : 0u;
    uint32_t incl = p;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    if (k < words) wpre[k] = carry + incl - p;
    carry += __shfl_sync(kFull, incl, 31);
  }
  __syncwarp();
}

// --------------------------------------------------------------- selection glue
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

// Moves this CTA's histogram counts into request r's global histogram and
// raises the shared bounds from the global one (one warp at a time; the
// others skip). Counts move by atomic exchange, so each candidate stays
// counted exactly once; the segment end pushes what is left.
__device__ __noinline__ uint64_t push_histogram(uint32_t* ghist, SelCtl* ctl, int r, uint32_t n,
                                                float C, uint64_t thr, ThrSinks sinks, int lane) {
  int got = 0;
  if (lane == 0) got = atomicCAS(&ctl->push_lock, 0, 1) == 0 ? 1 : 0;
  if (!__shfl_sync(kFull, got, 0)) return thr;
  uint32_t* gh = ghist + static_cast<size_t>(r) * kHistBins;
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
  const uint64_t hb = hist_bound_regs(h, n, C, lane);
  if (hb > thr) {
    thr = hb;
    publish_thr(hb, lane, sinks);
  }
  __syncwarp();
  if (lane == 0) atomicExch(&ctl->push_lock, 0);
  return thr;
}

__device__ __forceinline__ float finite_or_ninf(float x) {
  return (x > __int_as_float(0xFF800000) && x < __int_as_float(0x7F800000))
             ? x
             : __int_as_float(0xFF800000);
}

// Histogram reference of request r: its largest finite parent score (every
// child score is at most its parent's), the same in every CTA. Two slots
// alternate so that one can be cleared while the other is read. All
// consumer threads call it.
// This thread's part of the maximum (loads only; combined by segment_ref_finish).
__device__ __forceinline__ float segment_ref_part(const SArgs& a, const Team& t, int r) {
  float m = __int_as_float(0xFF800000);
  const float* ps = a.parent_scores + static_cast<int64_t>(r) * a.B_in;
  for (int i = t.tid; i < a.B_in; i += t.T) m = fmaxf(m, finite_or_ninf(ps[i]));
  return m;
}
__device__ __forceinline__ float segment_ref_finish(const Team& t, SelCtl* ctl, int slot, float m) {
  m = warp_max(m);
  if (t.lane == 0 && m > __int_as_float(0xFF800000)) atomicMax(&ctl->ref_ord[slot], ord_f32(m));
  team_sync(t);
  const unsigned o = *reinterpret_cast<volatile unsigned*>(&ctl->ref_ord[slot]);
  if (t.tid == 0) ctl->ref_ord[slot ^ 1] = 0u;
  return o ? unord_f32(o) : 0.f;
}
__device__ __forceinline__ float segment_ref(const SArgs& a, const Team& t, SelCtl* ctl, int r,
                                             int slot) {
  return segment_ref_finish(t, ctl, slot, segment_ref_part(a, t, r));
}

// End of the segment of request r (all consumer warps, in the same order).
__device__ __noinline__ bool segment_end(const SArgs& a, Team team, WarpBuf wb, SelCtl* ctl,
                                         uint64_t* wkeys, int32_t* wvals, uint32_t* whist,
                                         uint32_t* chist, uint8_t* stages, int r, int r_last,
                                         float C) {
  const StreamPlan& p = a.plan;
  FlushArgs f;
  f.n = a.n;
  f.r = r;
  f.k = static_cast<int>(blockIdx.x) - a.part.first_cta(r);
  f.G = a.part.contributors(r);
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
  f.cw = p.Cw;
  f.sort_keys = wkeys;
  f.sort_vals = wvals;
  f.sort_cap = p.W * p.Cw;
  f.radix_hist = chist;
  f.wvals = wvals;
  f.rank_P = whist;
  f.rank_cur = whist + kHistBins;
  // The stages are idle only at the CTA's last segment (every row consumed).
  const bool last = r == r_last;
  const int direct_cap = (p.W * p.D * p.stage_bytes / 12) & ~1;
  f.direct_keys = last ? reinterpret_cast<uint64_t*>(stages) : nullptr;
  f.direct_vals =
      last ? reinterpret_cast<int32_t*>(stages + static_cast<size_t>(direct_cap) * 8) : nullptr;
  f.direct_cap = last ? direct_cap : 0;
  f.read_request_bound = 0;  // the warps fold the request's bound in row by row
  const StepOut out{a.out_scores, a.out_parent, a.out_code, a.out_node,
                    a.n, static_cast<uint32_t>(a.V), a.out_width};
  return segment_flush(team, wb, ctl, f, out);
}

// --------------------------------------------------------------- streaming
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Waits until at most `pending` of this thread's most recent copy groups are
// still in flight (pending: 0 .. 3).
__device__ __forceinline__ void cp_async_wait(int pending) {
  switch (pending) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
  }
}

// Programmatic dependent launch: wait for the grid this launch depends on
// (its writes are then visible), and let the next one start launching.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The rows of a CTA: row(i) = first + stride * i, i < count.
struct RowSeq {
  int64_t first;
  int64_t stride;
  int count;
  __device__ __forceinline__ int64_t row(int i) const { return first + stride * i; }
};

// Parent data of a row (16 bytes): score (-inf = dead), child id range
// o0..o1, and the row kind: a child-bitmask row index (>= 0), kRowList
// (children as codes) or kRowNoTrie.
__device__ __forceinline__ uint4 row_meta(const SArgs& a, int64_t row) {
  float s = a.parent_scores[row];
  const int32_t p = a.layout ? a.parent_nodes[row] : 0;
  bool live = s != __int_as_float(0xFF800000);
  uint32_t o0 = 0, o1 = 0;
  int32_t mrow = kRowNoTrie;
  if (a.layout) {
    if (p < 0) {
      live = false;
    } else if (static_cast<int64_t>(p) >= a.n_parent) {
      if (live) atomicOr(a.status, kStatusBadNode);
      live = false;
    }
    if (live) {
      o0 = a.off[p];
      o1 = a.off[p + 1];
      mrow = a.layout == SIDBEAM_LAYOUT_DENSE ? p : (a.mask_idx ? a.mask_idx[p] : kRowList);
    }
  }
  if (!live) s = __int_as_float(0xFF800000);
  return make_uint4(__float_as_uint(s), o0, o1, static_cast<uint32_t>(mrow));
}

// A global load issued where it stands (asm volatile keeps it in place), so
// that its latency overlaps the work up to the first use of the value.
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 shfl_u4(const uint4& v, int src) {
  return make_uint4(__shfl_sync(kFull, v.x, src), __shfl_sync(kFull, v.y, src),
                    __shfl_sync(kFull, v.z, src), __shfl_sync(kFull, v.w, src));
}

// What one warp copies of a row: its logits chunk and the trie data the
// chunk needs.
struct ChunkCopy {
  int c0;       // first code of the chunk
  int cbytes;   // logits bytes of the chunk (whole 16-byte vectors; 0: empty chunk)
  int mb0;      // first byte of the chunk's bitmask bytes in a bitmask row
  int mbytes;   // bitmask bytes copied
  int ebase;    // stage offset of the trie data (the plan's chunk_bytes)
};

// Issues this warp's 16-byte copies of row `row` (parent data m) into `stage`:
// the logits chunk (logits), the trie data (extra), or both. Dead rows copy
// nothing. The caller commits the group.
template <int ESIZE>
__device__ __forceinline__ void issue_chunk(const SArgs& a, const ChunkCopy& cc, uint8_t* stage,
                                            int64_t row, const uint4& m, bool logits, bool extra,
                                            int lane) {
  if (m.x == 0xFF800000u) return;
  if (logits) {
    const uint8_t* src = a.logits + row * a.row_bytes + static_cast<int64_t>(cc.c0) * ESIZE;
    for (int o = lane * 16; o < cc.cbytes; o += 512) cp_async16(stage + o, src + o);
  }
  if (extra) {
    const int32_t mrow = static_cast<int32_t>(m.w);
    if (mrow >= 0) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>(a.mask + static_cast<size_t>(mrow) * a.mask_stride) + cc.mb0;
      for (int o = lane * 16; o < cc.mbytes; o += 512) cp_async16(stage + cc.ebase + o, src + o);
    } else if (mrow == kRowList && m.z > m.y) {
      const uint32_t a0 = m.y & ~7u;
      uint32_t nc = m.z - a0;
      if (nc > static_cast<uint32_t>(kListStageCodes + 8)) nc = kListStageCodes + 8;
      const int nb = static_cast<int>((nc * 2u + 15u) & ~15u);
      const uint8_t* src = reinterpret_cast<const uint8_t*>(a.codes + a0);
      for (int o = lane * 16; o < nb; o += 512) cp_async16(stage + cc.ebase + o, src + o);
    }
  }
}

// --------------------------------------------------------------- kernel
template <int BF16>
__global__ void __launch_bounds__(kStreamMaxWarps * 32, 1)
    beam_stream_kernel(const __grid_constant__ SArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kPerVec = BF16 ? 8 : 4;
  constexpr int kEsize = BF16 ? 2 : 4;
  const StreamPlan& p = a.plan;
  SelCtl* ctl = reinterpret_cast<SelCtl*>(smem + p.off_ctl);
  uint32_t* chist = reinterpret_cast<uint32_t*>(smem + p.off_chist);
  uint32_t* whist = reinterpret_cast<uint32_t*>(smem + p.off_whist);
  uint8_t* stages = smem + p.off_stage;
  uint64_t* wkeys = reinterpret_cast<uint64_t*>(smem + p.off_wkeys);
  int32_t* wvals = reinterpret_cast<int32_t*>(smem + p.off_wvals);

  const int W = p.W, K = p.K, D = p.D;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int T = W / K;          // teams
  const int tm = warp / K;      // this warp's team
  const int j = warp - tm * K;  // this warp's chunk of every row
  const int team_bar = kTeamBarBase + tm;
  const Team team{static_cast<int>(threadIdx.x), W * 32, warp, lane, W};
  float* tslot = reinterpret_cast<float*>(smem + p.off_team + static_cast<size_t>(tm) * 2 * kTeamSlotBytes);
  uint32_t* wm32 = reinterpret_cast<uint32_t*>(smem + p.off_wmask + warp * p.mcopy_bytes);
  uint32_t* wpre = reinterpret_cast<uint32_t*>(smem + p.off_wprefix + warp * p.mcopy_bytes);
  uint8_t* my_stages = stages + static_cast<size_t>(warp) * D * p.stage_bytes;
  uint4* smeta = reinterpret_cast<uint4*>(smem + p.off_meta) + warp * kMaxStreamDepth;

  // This warp's chunk of every row: codes c0 .. c1-1 in nvec 16-byte vectors.
  const int c0 = j * p.CW;
  const int c1 = c0 + p.CW < a.V ? c0 + p.CW : a.V;
  const int nvec = c0 < a.V ? (c1 - c0 + kPerVec - 1) / kPerVec : 0;
  const int tail = (c1 - c0) % kPerVec;  // elements in the last vector (0: a full vector)
  const bool full_chunk = nvec == 32 * kRegVecs && tail == 0;
  ChunkCopy cc;
  cc.c0 = c0;
  cc.cbytes = nvec * 16;
  cc.mb0 = (c0 >> 3) & ~15;
  cc.mbytes = p.mcopy_bytes < a.mask_stride * 4 - cc.mb0 ? p.mcopy_bytes : a.mask_stride * 4 - cc.mb0;
  cc.ebase = p.chunk_bytes;

  // The team's rows. With at least as many rows as teams, team m takes the
  // CTA's rows m, m + T, ...; with fewer, each row goes to P teams, which all
  // compute its statistics (in the same order) and split its candidates.
  RowSeq cq;
  a.part.rows(static_cast<int>(blockIdx.x), 0, 1, cq.first, cq.stride, cq.count);
  const int groups = cq.count < T ? (cq.count > 0 ? cq.count : 1) : T;
  const int P = T / groups;
  const int grp = tm / P;
  const int part = tm - grp * P;
  RowSeq q;
  q.first = cq.first + cq.stride * grp;
  q.stride = cq.stride * groups;
  q.count = grp < groups && grp < cq.count ? (cq.count - grp + groups - 1) / groups : 0;

  if (threadIdx.x == 0) {
    ctl->cta_thr = 0ull;
    ctl->abort_flag = 0;
    ctl->counter = 0;
    ctl->ref_ord[0] = 0u;
    ctl->ref_ord[1] = 0u;
    ctl->hist_total = 0u;
    ctl->push_lock = 0;
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) ctl->hist[i] = 0u;
  __syncthreads();
  griddep_launch();
  griddep_wait();  // no global memory is touched before this point

  // 1. The logits of the first D rows go out before any parent data is read.
  for (int k = 0; k < D; ++k) {
    if (k < q.count)
      issue_chunk<kEsize>(a, cc, my_stages + k * p.stage_bytes, q.row(k), make_uint4(0u, 0u, 0u, 0u),
                          true, false, lane);
    cp_async_commit();
  }
  // 2. Parent data, 32 rows at a time (lane k: row base + k), then the trie
  //    data of the first rows; the first segment's histogram reference (the
  //    request's largest parent score) is loaded alongside.
  int64_t lo, hi;
  a.part.range(static_cast<int>(blockIdx.x), lo, hi);
  const int r_first = static_cast<int>(lo / a.B_in);
  const int r_last = static_cast<int>((hi - 1) / a.B_in);
  const float mref = segment_ref_part(a, team, r_first);
  int mbase = 0;
  uint4 mb = make_uint4(0xFF800000u, 0u, 0u, 0u);
  if (lane < q.count) mb = row_meta(a, q.row(lane));
  for (int k = 0; k < D; ++k) {
    const uint4 mk = shfl_u4(mb, k);
    if (lane == 0) smeta[k] = mk;  // parent data of the row in stage k
    if (k < q.count)
      issue_chunk<kEsize>(a, cc, my_stages + k * p.stage_bytes, q.row(k), mk, false, true, lane);
    cp_async_commit();
  }

  WarpBuf wb{wkeys + static_cast<size_t>(warp) * p.Cw, wvals + static_cast<size_t>(warp) * p.Cw,
             whist + warp * 256, p.Cw, 0, 0ull, 0};
  int ref_slot = 0;
  float C = segment_ref_finish(team, ctl, ref_slot, mref);
  int cur_r = r_first;
  int64_t seg_end = static_cast<int64_t>(cur_r + 1) * a.B_in;
  const uint4 ninf = BF16 ? make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u)
                          : make_uint4(0xFF800000u, 0xFF800000u, 0xFF800000u, 0xFF800000u);

  auto flush = [&]() -> bool {
    const bool stop =
        segment_end(a, team, wb, ctl, wkeys, wvals, whist, chist, stages, cur_r, r_last, C);
    wb.count = 0;
    wb.thr = 0ull;
    if (stop) return true;
    if (cur_r < r_last) C = segment_ref(a, team, ctl, cur_r + 1, ref_slot ^= 1);
    ++cur_r;
    seg_end += a.B_in;
    return false;
  };

  bool stopped = false;
  for (int t = 0; t < q.count; ++t) {
    const int64_t row = q.row(t);
    while (row >= seg_end && !stopped) stopped = flush();
    if (stopped) break;
    const int r = cur_r;
    const int slot = t % D;
    const uint8_t* stage = my_stages + slot * p.stage_bytes;
    const uint4 m = smeta[slot];
    const float s = __uint_as_float(m.x);
    const uint32_t o0 = m.y, o1 = m.z;
    const int32_t mrow = static_cast<int32_t>(m.w);
    const bool dead = s == __int_as_float(0xFF800000);
    const bool multi = a.part.contributors(r) > 1;
    // The request's shared bound, loaded now (an L2 round trip) and first
    // used after the row's statistics.
    unsigned long long req = 0ull;
    if (multi && !dead) req = ld_relaxed_u64(a.request_thr + r);

    // Row chunk into registers, with the trie data it needs: the bitmask
    // bytes into the warp's copy, or each lane's child (code, logit) of a
    // list row. Then the stage takes the row D places ahead.
    cp_async_wait(D - 1);
    __syncwarp();
    uint4 x[kRegVecs];
    const uint4* src = reinterpret_cast<const uint4*>(stage);
    if (!dead && full_chunk) {
#pragma unroll
      for (int i = 0; i < kRegVecs; ++i) x[i] = src[lane + 32 * i];
    } else {
#pragma unroll
      for (int i = 0; i < kRegVecs; ++i) {
        const int v = lane + 32 * i;
        x[i] = (!dead && v < nvec) ? src[v] : ninf;
        if (tail && v == nvec - 1) vec_cut<BF16>(x[i], tail);
      }
    }
    const uint32_t nch = o1 - o0;
    int lcode = -1;
    float lz = 0.f;
    bool hold = false;  // a list row with more children than lanes keeps its stage
    if (!dead && mrow >= 0) {
      const uint4* ms = reinterpret_cast<const uint4*>(stage + cc.ebase);
      for (int i = lane; i < (cc.mbytes >> 4); i += 32) reinterpret_cast<uint4*>(wm32)[i] = ms[i];
    } else if (!dead && mrow == kRowList) {
      const uint32_t a0 = o0 & ~7u;
      const uint16_t* scodes = reinterpret_cast<const uint16_t*>(stage + cc.ebase);
      if (static_cast<uint32_t>(lane) < nch) {
        const uint32_t k = o0 + lane;
        const int code = (k - a0 < static_cast<uint32_t>(kListStageCodes + 8)) ? scodes[k - a0] : a.codes[k];
        if (code >= c0 && code < c1) {
          lcode = code;
          lz = BF16 ? __uint_as_float(static_cast<uint32_t>(
                          reinterpret_cast<const uint16_t*>(stage)[code - c0]) << 16)
                    : reinterpret_cast<const float*>(stage)[code - c0];
        }
      }
      hold = nch > 32u;
    }
    __syncwarp();
    auto refill = [&]() {
      const int qn = t + D;
      if (qn < q.count) {
        if (qn >= mbase + 32) {  // next 32 rows' parent data
          mbase += 32;
          mb = make_uint4(0xFF800000u, 0u, 0u, 0u);
          if (mbase + lane < q.count) mb = row_meta(a, q.row(mbase + lane));
        }
        const uint4 mn = shfl_u4(mb, qn - mbase);
        if (lane == 0) smeta[slot] = mn;
        issue_chunk<kEsize>(a, cc, my_stages + slot * p.stage_bytes, q.row(qn), mn, true, true, lane);
      }
      cp_async_commit();
    };
    if (!hold) refill();

    // Statistics of the chunk; the team combines its warps' (max, sum).
    float lm = __int_as_float(0xFF800000), ls = 0.f;
    if (!dead) {
      if (full_chunk) lane_stats<BF16, true>(x, nvec, lm, ls);
      else lane_stats<BF16, false>(x, nvec, lm, ls);
    }
    float wmx, wsum;
    warp_stats(lm, ls, wmx, wsum);
    float lse;
    if (K == 1) {
      lse = wmx + logf(wsum);
    } else {
      float* ts = tslot + (t & 1) * (kTeamSlotBytes / 4);
      if (lane == 0) {
        ts[j] = wmx;
        ts[kMaxTeamWarps + j] = wsum;
      }
      named_sync(team_bar, K * 32);
      float M = __int_as_float(0xFF800000);
      for (int u = 0; u < K; ++u) M = fmaxf(M, ts[u]);
      float sum = 0.f;
      for (int u = 0; u < K; ++u) {
        const float mu = ts[u];
        if (mu > __int_as_float(0xFF800000)) sum += ts[kMaxTeamWarps + u] * ex2_approx((mu - M) * kLog2e);
      }
      lse = M + logf(sum);
    }

    if (!dead) {
      // Candidates of this warp's chunk.
      const uint32_t b = static_cast<uint32_t>(row - static_cast<int64_t>(r) * a.B_in);
      const uint32_t idx0 = b * static_cast<uint32_t>(a.V);
      const ThrSinks sinks{&ctl->cta_thr, multi ? a.request_thr + r : nullptr};
      {
        const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
        if (c > wb.thr) wb.thr = c;
        if (req > wb.thr) wb.thr = req;
        if (req > c && lane == 0) atomicMax(&ctl->cta_thr, req);  // the CTA's bound holds it too
      }
      float zthr = zthreshold(wb.thr, s, lse);
      bool binned_any = false;
      if (mrow == kRowList) {
        const bool okc = lcode >= 0 && lz >= zthr && lane % P == part;
        if (__any_sync(kFull, okc)) {
          const float score = s + (lz - lse);
          warp_bin(ctl->hist, okc, score_bin(score, C), wb.binned, &ctl->hist_total);
          warp_offer_nc(wb, okc, make_key(score, idx0 + static_cast<uint32_t>(lcode)),
                        static_cast<int32_t>(o0 + lane), static_cast<uint32_t>(a.n), lane, sinks);
          binned_any = true;
        }
        if (hold) {
          // More children than lanes: the rest straight from the held stage.
          const uint32_t a0 = o0 & ~7u;
          const uint16_t* scodes = reinterpret_cast<const uint16_t*>(stage + cc.ebase);
          for (uint32_t k0 = o0 + 32; k0 < o1; k0 += 32) {
            const uint32_t k = k0 + lane;
            int code = -1;
            float z = 0.f;
            if (k < o1) {
              code = (k - a0 < static_cast<uint32_t>(kListStageCodes + 8)) ? scodes[k - a0] : a.codes[k];
              if (code >= c0 && code < c1)
                z = BF16 ? __uint_as_float(static_cast<uint32_t>(
                               reinterpret_cast<const uint16_t*>(stage)[code - c0]) << 16)
                         : reinterpret_cast<const float*>(stage)[code - c0];
              else
                code = -1;
            }
            zthr = zthreshold(wb.thr, s, lse);
            const bool okk = code >= 0 && z >= zthr && (k - o0) % P == static_cast<uint32_t>(part);
            if (!__any_sync(kFull, okk)) continue;
            const float score = s + (z - lse);
            warp_bin(ctl->hist, okk, score_bin(score, C), wb.binned, &ctl->hist_total);
            warp_offer_nc(wb, okk, make_key(score, idx0 + static_cast<uint32_t>(code)),
                          static_cast<int32_t>(k), static_cast<uint32_t>(a.n), lane, sinks);
            binned_any = true;
          }
        }
      } else if (__any_sync(kFull, lm >= zthr)) {
        // Bitmask rows and rows without a trie: hit bits per vector (byte i
        // of the packed words: the valid codes of vector lane + 32 i with
        // z >= zthr).
        const bool masked = mrow >= 0;
        uint32_t hp[kRegVecs / 4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < kRegVecs; ++i) {
          const int v = lane + 32 * i;
          if ((full_chunk || v < nvec) && i % P == part && vec_max<BF16>(x[i]) >= zthr) {
            const int cv = c0 + kPerVec * v;
            unsigned vb = (1u << kPerVec) - 1u;
            if (masked) {
              const int bit = cv - 8 * cc.mb0;
              vb = (reinterpret_cast<const uint8_t*>(wm32)[bit >> 3] >> (bit & 7)) & vb;
            }
            if (a.V - cv < kPerVec) vb &= (1u << (a.V - cv)) - 1u;
            unsigned bits = 0u;
#pragma unroll
            for (int e = 0; e < kPerVec; ++e)
              if (((vb >> e) & 1u) && vec_elem<BF16>(x[i], e) >= zthr) bits |= 1u << e;
            hp[i >> 2] |= bits << ((i & 3) * 8);
          }
        }
        const int nh = static_cast<int>(
            __reduce_add_sync(kFull, __popc(hp[0]) + __popc(hp[1]) + __popc(hp[2]) + __popc(hp[3])));
        if (nh > 0) {
          bool have_prefix = false;
          uint32_t nbase = o0;
          // One walk over the hit bits; mode 0: count and offer, 1: count
          // only, 2: offer only. Offers go in only while the warp buffer has
          // room for a full round (no call inside the walk, so the row stays
          // in registers); when it fills, the walk stops, the buffer is
          // compacted and the walk resumes with the bits that are left.
          auto walk = [&](int mode) {
            if (masked && mode != 1 && !have_prefix) {
              mask_prefix(wm32, cc.mbytes >> 2, wpre, lane);
              if (cc.mb0 > 0) {  // set bits of the row before the chunk's copy
                const uint32_t* mr = a.mask + static_cast<size_t>(mrow) * a.mask_stride;
                uint32_t cnt = 0;
                for (int w = lane; w < (cc.mb0 >> 2); w += 32) cnt += __popc(__ldg(mr + w));
                nbase = o0 + warp_sum_u(cnt);
              }
              have_prefix = true;
            }
            for (;;) {
              bool full = false;
#pragma unroll
              for (int i = 0; i < kRegVecs; ++i) {
                if (!full_chunk && 32 * i >= nvec) continue;
                unsigned bits = (hp[i >> 2] >> ((i & 3) * 8)) & 0xFFu;
                while (!full && __any_sync(kFull, bits != 0u)) {
                  if (mode != 1 && wb.count + 32 > wb.cw) {
                    full = true;
                    break;
                  }
                  const int e = bits ? __ffs(bits) - 1 : 0;
                  const bool had = bits != 0u;
                  bits &= bits - 1u;
                  const float z = vec_elem<BF16>(x[i], e);
                  const int code = c0 + kPerVec * (lane + 32 * i) + e;
                  const float score = s + (z - lse);
                  if (mode != 2)
                    warp_bin(ctl->hist, had, score_bin(score, C), wb.binned, &ctl->hist_total);
                  if (mode != 1) {
                    const uint64_t key = make_key(score, idx0 + static_cast<uint32_t>(code));
                    const bool pass = had && z >= zthr && key >= wb.thr;
                    const unsigned bal = __ballot_sync(kFull, pass);
                    if (pass) {
                      const int pos = wb.count + __popc(bal & lanemask_lt());
                      wb.keys[pos] = key;
                      wb.vals[pos] = masked ? mask_child(wm32, wpre, nbase, code - 8 * cc.mb0) : -1;
                    }
                    wb.count += __popc(bal);
                  }
                }
                hp[i >> 2] = (hp[i >> 2] & ~(0xFFu << ((i & 3) * 8))) | (bits << ((i & 3) * 8));
              }
              if (!full) break;
              __syncwarp();
              warp_compact(wb, static_cast<uint32_t>(a.n), lane, sinks);  // inline: no call
              zthr = zthreshold(wb.thr, s, lse);
            }
          };
          // Few hits: count and offer in one walk. Many: count them all lane
          // by lane (no votes: every lane bins its own hits), raise the
          // threshold from this CTA's histogram, keep only the hits that
          // still reach it, and offer those.
          if (nh <= kOnePassHits) {
            walk(0);
          } else {
#pragma unroll
            for (int i = 0; i < kRegVecs; ++i) {
              if (!full_chunk && 32 * i >= nvec) continue;
              const unsigned bits = (hp[i >> 2] >> ((i & 3) * 8)) & 0xFFu;
              if (bits) {
#pragma unroll 1
                for (int e = 0; e < kPerVec; ++e)
                  if ((bits >> e) & 1u)
                    atomicAdd(&ctl->hist[score_bin(s + (vec_elem<BF16>(x[i], e) - lse), C)], 1u);
              }
            }
            wb.binned += nh;
            if (lane == 0) atomicAdd(&ctl->hist_total, static_cast<unsigned>(nh));
            __syncwarp();
            wb.binned = kRefreshAfter;  // rescan this CTA's histogram now (inline: no call)
            refresh_thr(wb, ctl, static_cast<uint32_t>(a.n), C, lane, sinks);
            const float z1 = zthreshold(wb.thr, s, lse);
            if (z1 > zthr) zthr = z1;
#pragma unroll
            for (int i = 0; i < kRegVecs; ++i) {
              if (!full_chunk && 32 * i >= nvec) continue;
              const unsigned bits = (hp[i >> 2] >> ((i & 3) * 8)) & 0xFFu;
              unsigned keep = 0u;
              if (bits) {
#pragma unroll 1
                for (int e = 0; e < kPerVec; ++e)
                  if (((bits >> e) & 1u) && vec_elem<BF16>(x[i], e) >= zthr) keep |= 1u << e;
              }
              hp[i >> 2] = (hp[i >> 2] & ~(0xFFu << ((i & 3) * 8))) | (keep << ((i & 3) * 8));
            }
            walk(2);
          }
          binned_any = true;
        }
      }
      if (binned_any) {
        __syncwarp();
        refresh_row(wb, ctl, static_cast<uint32_t>(a.n), C, lane, sinks);
        if (multi && *reinterpret_cast<volatile unsigned*>(&ctl->hist_total) >= kPushAfter)
          wb.thr = push_histogram(a.ghist, ctl, r, static_cast<uint32_t>(a.n), C, wb.thr, sinks,
                                  lane);
      }
    }
    if (hold) {
      __syncwarp();
      refill();
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  // Remaining segment ends (every warp, in the same order).
  if (!stopped)
    while (cur_r <= r_last)
      if (flush()) break;
}

}  // namespace

// ------------------------------------------------------------------ host side

static cudaError_t stream_opt_in(const void* fn, int which) {
  static std::mutex mu;
  static bool done[2][64] = {};
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

// The deterministic step on the streaming kernel. Returns SIDBEAM_ERR_INVALID_ARG
// (with nothing launched) when no plan fits the shape.
int launch_beam_stream(const sidbeam_trie* trie, int step, const void* logits, int dtype,
                       int64_t ld, const float* parent_scores, const int32_t* parent_nodes, int R,
                       int B_in, int n_out, int V, float* out_scores, int32_t* out_parent,
                       int32_t* out_code, int32_t* out_node, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream, const int32_t* out_width) {
  SArgs a{};
  a.logits = static_cast<const uint8_t*>(logits);
  const bool bf16 = dtype == SIDBEAM_BF16;
  const int esize = bf16 ? 2 : 4;
  a.row_bytes = ld * esize;
  a.V = V;
  a.parent_scores = parent_scores;
  a.parent_nodes = parent_nodes;
  a.R = R;
  a.B_in = B_in;
  a.n = n_out;
  bool has_mask = false, has_list = false;
  int stride = ((V + 31) / 32 + 3) / 4 * 4;
  if (trie) {
    const StepTrie& st = trie->steps[step];
    a.layout = st.layout;
    a.off = st.off;
    a.mask = st.mask;
    a.mask_idx = st.mask_idx;
    a.codes = st.codes;
    a.n_parent = st.n_parent;
    stride = st.mask_stride;
    has_mask = st.layout == SIDBEAM_LAYOUT_DENSE || st.mask_idx != nullptr;
    has_list = st.layout == SIDBEAM_LAYOUT_CSR;
  }
  a.mask_stride = stride;
  a.out_scores = out_scores;
  a.out_parent = out_parent;
  a.out_code = out_code;
  a.out_node = out_node;
  a.out_width = out_width;
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
  const int ctl_bytes = (static_cast<int>(sizeof(dev::SelCtl)) + 127) / 128 * 128;
  if (!choose_stream_plan(V, esize, has_mask, stride, has_list, n_out, ctl_bytes, kSmemBudget,
                          &a.plan))
    return set_error(SIDBEAM_ERR_INVALID_ARG,
                     "beam_step: V=%d with n_out=%d does not fit in shared memory", V, n_out);
  const void* fn = bf16 ? reinterpret_cast<const void*>(&beam_stream_kernel<1>)
                        : reinterpret_cast<const void*>(&beam_stream_kernel<0>);
  cudaError_t e = stream_opt_in(fn, bf16 ? 1 : 0);
  if (e != cudaSuccess) return cuda_error(e, "beam_step: cudaFuncSetAttribute");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(a.part.grid));
  cfg.blockDim = dim3(static_cast<unsigned>(32 * a.plan.W));
  cfg.dynamicSmemBytes = static_cast<size_t>(a.plan.smem_bytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = bf16 ? cudaLaunchKernelEx(&cfg, beam_stream_kernel<1>, a)
           : cudaLaunchKernelEx(&cfg, beam_stream_kernel<0>, a);
  if (e != cudaSuccess) return cuda_error(e, "beam_step: launch");
  return SIDBEAM_OK;
}

}  // namespace sidbeam
