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
//    live rows only, issues an untiled bulk copy (cp.async.bulk, TMA engine)
//    of the logits row -- plus the node's bitmask row at dense levels -- into
//    a ring of S shared-memory stages, completing on an mbarrier.
//  * Warps 1..W are consumers. Each takes ring items round-robin, computes the
//    row max and sum of exp over the FULL codebook (fp32, warp shuffles),
//    lse = m + log(sum), then walks the node's valid children and offers
//    key(score = s + (z_c - lse), idx = b*V + c) to its top-n buffer.
//  * At the end of each segment the consumer warps run the CTA merge and, in
//    the last contributing CTA of the request, the request merge (topn.cuh).
// The logits are read exactly once from HBM; nothing else is re-read.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "device_utils.cuh"
#include "internal.h"
#include "launch.h"
#include "topn.cuh"

namespace sidbeam {
namespace {

using namespace dev;

constexpr float kLog2e = 1.4426950408889634f;

enum ItemKind : int32_t { kItemRow = 0, kItemSegmentEnd = 1, kItemExit = 2 };

struct __align__(16) Meta {
  int32_t kind;
  int32_t req;
  int64_t row;
  float score;
  int32_t node;
  uint32_t o0;
  uint32_t o1;
  uint32_t seq;   // ring item number; written before the full-barrier arrive
  uint32_t pad[3];
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
  Partition part;
  StepConfig cfg;
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

// Max of the 16 bytes `q` as 8 bf16 or 4 fp32 values.
template <int BF16>
__device__ __forceinline__ float vec_max(const uint4& q) {
  if (BF16) {
    const float a = fmaxf(fmaxf(__uint_as_float(q.x << 16), __uint_as_float(q.x & 0xFFFF0000u)),
                          fmaxf(__uint_as_float(q.y << 16), __uint_as_float(q.y & 0xFFFF0000u)));
    const float b = fmaxf(fmaxf(__uint_as_float(q.z << 16), __uint_as_float(q.z & 0xFFFF0000u)),
                          fmaxf(__uint_as_float(q.w << 16), __uint_as_float(q.w & 0xFFFF0000u)));
    return fmaxf(a, b);
  }
  return fmaxf(fmaxf(__uint_as_float(q.x), __uint_as_float(q.y)),
               fmaxf(__uint_as_float(q.z), __uint_as_float(q.w)));
}

// Sum of exp(z - m) over the 16 bytes `q`, as 2^(z*log2e - m*log2e), tree-added.
template <int BF16>
__device__ __forceinline__ float vec_sumexp(const uint4& q, float mL) {
  if (BF16) {
    const float e0 = ex2_approx(fmaf(__uint_as_float(q.x << 16), kLog2e, -mL));
    const float e1 = ex2_approx(fmaf(__uint_as_float(q.x & 0xFFFF0000u), kLog2e, -mL));
    const float e2 = ex2_approx(fmaf(__uint_as_float(q.y << 16), kLog2e, -mL));
    const float e3 = ex2_approx(fmaf(__uint_as_float(q.y & 0xFFFF0000u), kLog2e, -mL));
    const float e4 = ex2_approx(fmaf(__uint_as_float(q.z << 16), kLog2e, -mL));
    const float e5 = ex2_approx(fmaf(__uint_as_float(q.z & 0xFFFF0000u), kLog2e, -mL));
    const float e6 = ex2_approx(fmaf(__uint_as_float(q.w << 16), kLog2e, -mL));
    const float e7 = ex2_approx(fmaf(__uint_as_float(q.w & 0xFFFF0000u), kLog2e, -mL));
    return ((e0 + e1) + (e2 + e3)) + ((e4 + e5) + (e6 + e7));
  }
  const float e0 = ex2_approx(fmaf(__uint_as_float(q.x), kLog2e, -mL));
  const float e1 = ex2_approx(fmaf(__uint_as_float(q.y), kLog2e, -mL));
  const float e2 = ex2_approx(fmaf(__uint_as_float(q.z), kLog2e, -mL));
  const float e3 = ex2_approx(fmaf(__uint_as_float(q.w), kLog2e, -mL));
  return (e0 + e1) + (e2 + e3);
}

// Full-codebook log-normaliser of one row in shared memory (warp-collective).
// Returns lse = m + log(sum_c exp(z_c - m)) in fp32.
template <int BF16>
__device__ __forceinline__ float row_lse(const uint8_t* row, int V, int lane) {
  constexpr int kPerVec = BF16 ? 8 : 4;
  const int nvec = V / kPerVec;  // full 16-byte vectors
  const int tail0 = nvec * kPerVec;
  const uint4* q = reinterpret_cast<const uint4*>(row);
  float m = __int_as_float(0xFF800000);
  for (int v = lane; v < nvec; v += 32) m = fmaxf(m, vec_max<BF16>(q[v]));
  if (lane < V - tail0) m = fmaxf(m, elem<BF16>(row, tail0 + lane));
  m = warp_max(m);
  const float mL = m * kLog2e;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  int v = lane;
  for (; v + 96 < nvec; v += 128) {
    a0 += vec_sumexp<BF16>(q[v], mL);
    a1 += vec_sumexp<BF16>(q[v + 32], mL);
    a2 += vec_sumexp<BF16>(q[v + 64], mL);
    a3 += vec_sumexp<BF16>(q[v + 96], mL);
  }
  for (; v < nvec; v += 32) a0 += vec_sumexp<BF16>(q[v], mL);
  if (lane < V - tail0) a1 += ex2_approx(fmaf(elem<BF16>(row, tail0 + lane), kLog2e, -mL));
  const float s = warp_sum((a0 + a1) + (a2 + a3));
  return m + logf(s);
}

// --------------------------------------------------------------- producer
__device__ void producer(const StepArgs& a, uint8_t* stages, Meta* meta, uint64_t* full,
                         uint64_t* empty, SelCtl* ctl, int64_t row_lo, int64_t row_hi, int lane) {
  const StepConfig& cfg = a.cfg;
  const int S = cfg.S;
  const uint64_t pol = policy_evict_first();
  const uint32_t tx_bytes =
      static_cast<uint32_t>(cfg.logits_copy_bytes + (a.layout == SIDBEAM_LAYOUT_DENSE ? cfg.mask_copy_bytes : 0));
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
          m.seq = item;
          uint8_t* dst = stages + static_cast<size_t>(stage) * cfg.stage_bytes;
          mbar_arrive_expect_tx(&full[stage], tx_bytes);
          bulk_copy_g2s(dst, a.logits + (base + j) * a.row_bytes,
                        static_cast<uint32_t>(cfg.logits_copy_bytes), &full[stage], pol);
          if (a.layout == SIDBEAM_LAYOUT_DENSE)
            bulk_copy_g2s(dst + cfg.logits_copy_bytes,
                          a.mask + static_cast<size_t>(pj) * a.mask_stride,
                          static_cast<uint32_t>(cfg.mask_copy_bytes), &full[stage], pol);
        }
        __syncwarp();
        ++item;
      }
    }
    // One segment-end marker per consumer warp (round-robin => each gets one).
    for (int w = 0; ok && w < cfg.W; ++w) {
      const int stage = acquire(item);
      if (stage < 0) {
        ok = false;
        break;
      }
      if (lane == 0) {
        meta[stage].kind = kItemSegmentEnd;
        meta[stage].req = r;
        meta[stage].seq = item;
        mbar_arrive(&full[stage]);
      }
      __syncwarp();
      ++item;
    }
    seg_lo = seg_hi;
  }
  for (int w = 0; ok && w < cfg.W; ++w) {
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
template <int BF16>
__device__ void process_row(const StepArgs& a, const uint8_t* zrow, const Meta& m, WarpBuf& wb,
                            SelCtl* ctl, int lane) {
  const int r = m.req;
  const uint32_t b = static_cast<uint32_t>(m.row - static_cast<int64_t>(r) * a.B_in);
  const uint32_t idx0 = b * static_cast<uint32_t>(a.V);
  const float s = m.score;
  const ThrSinks sinks{&ctl->cta_thr, a.request_thr + r};
  const unsigned long long req_thr =
      *reinterpret_cast<volatile unsigned long long*>(a.request_thr + r);

  // CSR: start the first batch of child-code loads before the reductions.
  uint32_t k_first = m.o0 + lane;
  int c_first = 0;
  if (a.layout == SIDBEAM_LAYOUT_CSR && k_first < m.o1) c_first = a.codes[k_first];

  const float lse = row_lse<BF16>(zrow, a.V, lane);

  const unsigned long long cthr = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
  if (cthr > wb.thr) wb.thr = cthr;
  if (req_thr > wb.thr) wb.thr = req_thr;

  if (a.layout == SIDBEAM_LAYOUT_CSR) {
    for (uint32_t k0 = m.o0; k0 < m.o1; k0 += 32) {
      const uint32_t k = k0 + lane;
      const bool valid = k < m.o1;
      int c = c_first;
      if (k0 != m.o0) c = valid ? a.codes[k] : 0;
      const float z = valid ? elem<BF16>(zrow, c) : 0.f;
      const float score = s + (z - lse);
      warp_offer(wb, valid, make_key(score, idx0 + static_cast<uint32_t>(c)),
                 static_cast<int32_t>(k), a.n, lane, sinks);
    }
  } else if (a.layout == SIDBEAM_LAYOUT_DENSE) {
    const uint32_t* mrow = reinterpret_cast<const uint32_t*>(zrow + a.cfg.logits_copy_bytes);
    uint32_t child = m.o0;
    for (int j = 0; j < a.mask_words; ++j) {
      const uint32_t w = mrow[j];
      if (w == 0) continue;
      const bool valid = (w >> lane) & 1u;
      const int c = j * 32 + lane;
      const float z = valid ? elem<BF16>(zrow, c) : 0.f;
      const float score = s + (z - lse);
      warp_offer(wb, valid, make_key(score, idx0 + static_cast<uint32_t>(c)),
                 static_cast<int32_t>(child + __popc(w & lanemask_lt())), a.n, lane, sinks);
      child += __popc(w);
    }
  } else {
    for (int c0 = 0; c0 < a.V; c0 += 32) {
      const int c = c0 + lane;
      const bool valid = c < a.V;
      const float z = valid ? elem<BF16>(zrow, c) : 0.f;
      const float score = s + (z - lse);
      warp_offer(wb, valid, make_key(score, idx0 + static_cast<uint32_t>(c)), -1, a.n, lane,
                 sinks);
    }
  }
}

template <int BF16>
__global__ void __launch_bounds__(kMaxStepThreads, 1)
    beam_step_kernel(const __grid_constant__ StepArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const StepConfig& cfg = a.cfg;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + cfg.off_bars);
  uint64_t* empty = full + cfg.S;
  SelCtl* ctl = reinterpret_cast<SelCtl*>(smem + cfg.off_ctl);
  Meta* meta = reinterpret_cast<Meta*>(smem + cfg.off_meta);
  uint32_t* cta_hist = reinterpret_cast<uint32_t*>(smem + cfg.off_chist);
  uint32_t* whist = reinterpret_cast<uint32_t*>(smem + cfg.off_whist);
  uint8_t* stages = smem + cfg.off_stage;
  uint64_t* wkeys = reinterpret_cast<uint64_t*>(smem + cfg.off_wkeys);
  int32_t* wvals = reinterpret_cast<int32_t*>(smem + cfg.off_wvals);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < cfg.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      meta[s].seq = 0xFFFFFFFFu;
    }
    ctl->cta_thr = 0ull;
    ctl->abort_flag = 0;
    ctl->counter = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t total = a.part.total_rows;
  const int64_t row_lo = static_cast<int64_t>(blockIdx.x) * a.part.rows_per_cta;
  const int64_t row_hi = min(total, row_lo + a.part.rows_per_cta);

  if (warp == 0) {
    producer(a, stages, meta, full, empty, ctl, row_lo, row_hi, lane);
    return;
  }

  Team team{static_cast<int>(threadIdx.x) - 32, cfg.W * 32, warp - 1, lane, cfg.W};
  WarpBuf wb{wkeys + static_cast<size_t>(team.warp) * cfg.Cw,
             wvals + static_cast<size_t>(team.warp) * cfg.Cw, whist + team.warp * 256, cfg.Cw,
             0, 0ull};
  const StepWriter writer{a.out_scores, a.out_parent, a.out_code, a.out_node, a.n,
                          static_cast<uint32_t>(a.V)};

  uint32_t item = static_cast<uint32_t>(team.warp);
  while (true) {
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
      process_row<BF16>(a, stages + static_cast<size_t>(stage) * cfg.stage_bytes, m, wb, ctl,
                        lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
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
      f.wkeys = wkeys;
      f.cw = cfg.Cw;
      f.sort_keys = wkeys;
      f.sort_vals = wvals;
      if (segment_flush(team, wb, ctl, cta_hist, f, writer)) break;
    }
    item += static_cast<uint32_t>(cfg.W);
  }
}

}  // namespace

// ------------------------------------------------------------------ host side

static int round_up(int x, int m) { return (x + m - 1) / m * m; }

bool choose_step_config(int V, int esize, int mask_stride_words, int n, StepConfig* cfg) {
  StepConfig c{};
  c.logits_copy_bytes = round_up(V * esize, 16);
  c.mask_copy_bytes = mask_stride_words * 4;
  c.stage_bytes = round_up(c.logits_copy_bytes + c.mask_copy_bytes, 128);
  int npow2 = 1;
  while (npow2 < n) npow2 <<= 1;
  const int fixed_head = 2 * kMaxStages * 8;                             // barriers
  const int ctl_bytes = round_up(static_cast<int>(sizeof(dev::SelCtl)), 128);
  const int meta_bytes = kMaxStages * static_cast<int>(sizeof(Meta));
  static const int kWarps[] = {8, 6, 4, 3, 2, 1};
  for (int W : kWarps) {
    const int cw = std::max(round_up(n, 32) + 512, round_up((npow2 + W - 1) / W, 32));
    int o = 0;
    c.off_bars = o;
    o += fixed_head;
    c.off_ctl = o;
    o += ctl_bytes;
    c.off_meta = o;
    o += meta_bytes;
    c.off_chist = o;
    o += 1024;
    c.off_whist = o;
    o += W * 1024;
    o = round_up(o, 128);
    const int warp_bytes = W * cw * 12 + 256;
    const int avail = kSmemBudget - o - warp_bytes;
    if (avail < c.stage_bytes) continue;
    int S = std::min(kMaxStages, avail / c.stage_bytes);
    if (S < 4 && W > 2) continue;
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

  a.part = make_partition(R, B_in, device_sm_count());
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

  if (!choose_step_config(V, esize, a.layout == SIDBEAM_LAYOUT_DENSE ? a.mask_stride : 0, n_out,
                          &a.cfg))
    return set_error(SIDBEAM_ERR_INVALID_ARG,
                     "beam_step: V=%d with n_out=%d does not fit in shared memory", V, n_out);

  const void* fn = a.bf16 ? reinterpret_cast<const void*>(&beam_step_kernel<1>)
                          : reinterpret_cast<const void*>(&beam_step_kernel<0>);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       a.cfg.smem_bytes);
  if (e != cudaSuccess) return cuda_error(e, "beam_step: cudaFuncSetAttribute");
  const dim3 grid(static_cast<unsigned>(a.part.grid));
  const dim3 block(static_cast<unsigned>(32 * (a.cfg.W + 1)));
  if (a.bf16)
    beam_step_kernel<1><<<grid, block, a.cfg.smem_bytes, stream>>>(a);
  else
    beam_step_kernel<0><<<grid, block, a.cfg.smem_bytes, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "beam_step: launch");
  return SIDBEAM_OK;
}

}  // namespace sidbeam
