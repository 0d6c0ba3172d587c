// The fused lm_head step: tcgen05 GEMM (lmhead.cu) -> per-row log-normaliser
// from the GEMM's per-tile partials -> the row's valid children scored from
// the child logits the GEMM kept -> per-request top-n (topn.cuh).
//
// flashrec 0.1.0 (PyPI page), Features > Decoding ("SID constraint"): the
// lm_head over the SID token range feeds the constrained step; the step's
// semantics are beam_step's (full-codebook log-softmax, trie mask, parent
// score added, deterministic top-n).
//
// Three launches on the caller's stream:
//  1. child bitmap per row (dense level: the node's mask row; CSR level: its
//     child codes set; dead rows all zero), so the GEMM epilogue and the
//     selection see one layout;
//  2. the GEMM in fused mode: per (row, 256-code tile) (max, sum exp) and the
//     fp32 logits of the valid children only (the full logits never reach HBM);
//  3. selection: per row lse = m + log(sum_j s_j * exp(m_j - m)); every valid
//     child c gives key(s_b + (z_c - lse), b*V + c) with node id = first child
//     id + rank of c among the node's set bits; warps offer to their top-n
//     buffers above shared lower bounds, segments end in the partial-list /
//     rank merge of topn.cuh.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "device_utils.cuh"
#include "internal.h"
#include "launch.h"
#include "lmhead.h"
#include "topn.cuh"

namespace sidbeam {
namespace {

using namespace dev;

constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr int kSelWarps = 8;
constexpr int kBatch = 16;  // child logits loaded per lane per round
constexpr uint32_t kHeavyChildren = 1024;  // parents with more children are walked by the CTA
constexpr int kHeavyList = 64;             // deferred parents per segment (more: walked at once)
constexpr float kL2e = 1.4426950408889634f;

struct FusedLayout {
  WorkspaceLayout sel;
  size_t partial, bitmap, zlog, total;
};

FusedLayout fused_layout(int R, int maxG, int n, int64_t M, int V) {
  FusedLayout f{};
  f.sel = workspace_layout(R, maxG, n);
  const int64_t ntiles = (V + kLmheadTileN - 1) / kLmheadTileN;
  const int64_t words = (V + 31) / 32;
  size_t o = f.sel.total;
  f.partial = align256(o);
  o = f.partial + static_cast<size_t>(M * ntiles) * 8;
  f.bitmap = align256(o);
  o = f.bitmap + static_cast<size_t>(M * words) * 4;
  f.zlog = align256(o);
  o = f.zlog + static_cast<size_t>(M) * V * 4;
  f.total = align256(o);
  return f;
}

// ------------------------------------------------------------ 1. child bitmaps
struct BitmapArgs {
  const float* parent_scores;
  const int32_t* parent_nodes;
  int64_t M;
  int layout;
  const uint32_t* off;
  const uint32_t* mask;
  int mask_stride;
  const uint16_t* codes;
  int64_t n_parent;
  int words;
  uint32_t* bitmap;  // [M][words]
  uint32_t* status;
};

// One warp per row. A row is dead when its parent score is -inf or its node
// is negative (bitmap all zero); a node past the level's end is reported. A
// CSR row is assembled in the warp's shared-memory copy (its sorted codes put
// up to 32 lanes on one word, which shared-memory atomics absorb far faster
// than global ones) and stored with plain coalesced writes.
constexpr int kBitmapWarps = 8;
__global__ void __launch_bounds__(kBitmapWarps * 32) child_bitmap_kernel(const BitmapArgs a) {
  extern __shared__ uint32_t sbits[];  // [kBitmapWarps][words]
  const int lane = threadIdx.x & 31;
  uint32_t* mine = sbits + static_cast<size_t>(threadIdx.x >> 5) * a.words;
  const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t row = w0; row < a.M; row += nw) {
    uint32_t* out = a.bitmap + row * a.words;
    const float s = a.parent_scores[row];
    const int32_t p = a.parent_nodes[row];
    bool live = s != __int_as_float(0xFF800000) && p >= 0;
    if (live && static_cast<int64_t>(p) >= a.n_parent) {
      if (lane == 0) atomicOr(a.status, kStatusBadNode);
      live = false;
    }
    if (live && a.layout == SIDBEAM_LAYOUT_DENSE) {
      const uint32_t* src = a.mask + static_cast<int64_t>(p) * a.mask_stride;
      for (int i = lane; i < a.words; i += 32) out[i] = src[i];
      continue;
    }
    if (!live) {
      for (int i = lane; i < a.words; i += 32) out[i] = 0u;
      continue;
    }
    for (int i = lane; i < a.words; i += 32) mine[i] = 0u;
    __syncwarp();
    // Codes 16 bytes at a time from id o0 rounded down to 8 (the code array is
    // padded by 8), four loads per lane in flight.
    const uint32_t o0 = a.off[p], o1 = a.off[p + 1];
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
        const uint32_t w4[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t id = a0 + v * 8u + e;
          if (v < nv && id >= o0 && id < o1) {
            const uint32_t c = (w4[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu;
            atomicOr(&mine[c >> 5], 1u << (c & 31));
          }
        }
      }
    }
    __syncwarp();
    for (int i = lane; i < a.words; i += 32) out[i] = mine[i];
    __syncwarp();  // the copy is read out before the next row clears it
  }
}

// ------------------------------------------------------------ 3. selection
struct SelArgs {
  const float* parent_scores;
  const int32_t* parent_nodes;
  int R, B_in, n, V;
  int layout;              // 0 = no trie
  const uint32_t* off;
  const float2* partial;   // [M][ntiles]
  int ntiles;
  const uint32_t* bitmap;  // [M][words] (trie levels)
  int words;
  const float* zlog;       // [M][V]: child logits (every logit without a trie)
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
  int Cw;
  int coop;
};

struct SelWriter {
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
      scores[o] = __int_as_float(0xFF800000);
      parent[o] = -1;
      code[o] = -1;
      node[o] = -1;
    }
  }
};

// Largest finite parent score of request r (the histogram reference; same
// value in every CTA). All team threads call it.
__device__ float request_reference(const SelArgs& a, const Team& t, SelCtl* ctl, int r,
                                   int slot) {
  float m = __int_as_float(0xFF800000);
  const float* ps = a.parent_scores + static_cast<int64_t>(r) * a.B_in;
  for (int i = t.tid; i < a.B_in; i += t.T) {
    const float x = ps[i];
    if (x > __int_as_float(0xFF800000) && x < __int_as_float(0x7F800000)) m = fmaxf(m, x);
  }
  m = warp_max(m);
  if (t.lane == 0 && m > __int_as_float(0xFF800000)) atomicMax(&ctl->ref_ord[slot], ord_f32(m));
  team_sync(t);
  const unsigned o = *reinterpret_cast<volatile unsigned*>(&ctl->ref_ord[slot]);
  if (t.tid == 0) ctl->ref_ord[slot ^ 1] = 0u;
  return o ? unord_f32(o) : 0.f;
}

__global__ void __launch_bounds__(kSelWarps * 32, 1) lmhead_select_kernel(const SelArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  SelCtl* ctl = reinterpret_cast<SelCtl*>(smem);
  uint8_t* p = smem + ((sizeof(SelCtl) + 127) / 128) * 128;
  uint32_t* cta_hist = reinterpret_cast<uint32_t*>(p);  // 256 words
  p += 1024;
  uint32_t* whist = reinterpret_cast<uint32_t*>(p);     // 2 x 1024 words (>= W x 256)
  p += 8192;
  int64_t* heavy = reinterpret_cast<int64_t*>(p);        // deferred rows of the segment
  int* heavy_count = reinterpret_cast<int*>(heavy + kHeavyList);
  p += kHeavyList * 8 + 128;
  uint64_t* wkeys = reinterpret_cast<uint64_t*>(p);
  p += static_cast<size_t>(kSelWarps) * a.Cw * 8;
  int32_t* wvals = reinterpret_cast<int32_t*>(p);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Team team{static_cast<int>(threadIdx.x), kSelWarps * 32, warp, lane, kSelWarps};
  if (threadIdx.x == 0) {
    ctl->cta_thr = 0ull;
    ctl->abort_flag = 0;
    ctl->counter = 0;
    ctl->ref_ord[0] = 0u;
    ctl->ref_ord[1] = 0u;
    ctl->hist_total = 0u;
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) ctl->hist[i] = 0u;
  if (threadIdx.x == 0) *heavy_count = 0;
  __syncthreads();

  int64_t seq_first, seq_stride;
  int seq_count;
  a.part.rows(static_cast<int>(blockIdx.x), a.coop ? 0 : warp, a.coop ? 1 : kSelWarps, seq_first,
              seq_stride, seq_count);
  int64_t lo, hi;
  a.part.range(static_cast<int>(blockIdx.x), lo, hi);
  const int r_first = static_cast<int>(lo / a.B_in);
  const int r_last = static_cast<int>((hi - 1) / a.B_in);
  int ref_slot = 0;
  float C = request_reference(a, team, ctl, r_first, ref_slot);
  const int part = a.coop ? warp : 0;
  const int nparts = a.coop ? kSelWarps : 1;

  WarpBuf wb{wkeys + static_cast<size_t>(warp) * a.Cw, wvals + static_cast<size_t>(warp) * a.Cw,
             whist + warp * 256, a.Cw, 0, 0ull, 0};
  const SelWriter writer{a.out_scores, a.out_parent, a.out_code, a.out_node, a.n,
                         static_cast<uint32_t>(a.V)};
  int cur_r = r_first;
  // Scores row `row` (of request r): this warp takes part `part` of `nparts`
  // of the row's bitmap words.
  auto do_row = [&](int64_t row, int r, int part, int nparts) {
    const float s = a.parent_scores[row];
    const int32_t pn = a.layout ? a.parent_nodes[row] : 0;
    if (s == __int_as_float(0xFF800000) || pn < 0) return;  // dead row (bad nodes: bitmap 0)
    // lse from the per-tile partials (over all V codes of the level).
    float mj = __int_as_float(0xFF800000);
    for (int t = lane; t < a.ntiles; t += 32) mj = fmaxf(mj, a.partial[row * a.ntiles + t].x);
    const float m = warp_max(mj);
    float sum = 0.f;
    for (int t = lane; t < a.ntiles; t += 32) {
      const float2 ps = a.partial[row * a.ntiles + t];
      if (ps.x > __int_as_float(0xFF800000)) sum += ps.y * ex2_approx((ps.x - m) * kL2e);
    }
    sum = warp_sum(sum);
    const float lse = m + logf(sum);
    {  // no child of the row can reach the bounds already known: nothing to walk
      const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
      if (c > wb.thr) wb.thr = c;
      if (m < zthreshold(wb.thr, s, lse)) return;
    }
    const uint32_t b = static_cast<uint32_t>(row - static_cast<int64_t>(r) * a.B_in);
    const uint32_t idx0 = b * static_cast<uint32_t>(a.V);
    const uint32_t o0 = a.layout ? a.off[pn] : 0u;
    const ThrSinks sinks{&ctl->cta_thr, a.request_thr + r};
    {
      const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&ctl->cta_thr);
      const unsigned long long q =
          *reinterpret_cast<volatile unsigned long long*>(a.request_thr + r);
      if (c > wb.thr) wb.thr = c;
      if (q > wb.thr) wb.thr = q;
    }
    // This warp's words: [wb0, wb1) of the row; lane chunks of `per` words.
    const int W = a.words;
    const int wb0 = static_cast<int>(static_cast<int64_t>(W) * part / nparts);
    const int wb1 = static_cast<int>(static_cast<int64_t>(W) * (part + 1) / nparts);
    const int per = (wb1 - wb0 + 31) / 32;
    const int l0 = min(wb1, wb0 + lane * per), l1 = min(wb1, l0 + per);
    const uint32_t* brow = a.layout ? a.bitmap + row * W : nullptr;
    auto word = [&](int w) -> uint32_t {
      if (!brow) {  // no trie: every code below V
        const int c0 = w * 32;
        return a.V - c0 >= 32 ? ~0u : ((1u << (a.V - c0)) - 1u);
      }
      return brow[w];
    };
    // Rank of the lane's first word: set bits in words [0, l0).
    uint32_t before = 0;
    if (brow) {
      uint32_t pre = 0;  // words before this warp's part
      for (int w = lane; w < wb0; w += 32) pre += __popc(brow[w]);
      pre = warp_sum_u(pre);
      uint32_t mine = 0;
      for (int w = l0; w < l1; ++w) mine += __popc(brow[w]);
      uint32_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      before = pre + incl - mine;
    }
    // Walk the lane's set bits kBatch at a time (independent logit loads in
    // flight together; a node may have thousands of children). A lane whose
    // tiles' largest logits (the GEMM's per-tile maxima) cannot reach the
    // threshold loads none of its children's logits.
    float zthr = zthreshold(wb.thr, s, lse);
    int cw = l0;
    if (l0 < l1) {
      constexpr int kTileWords = kLmheadTileN / 32;
      float tmax = __int_as_float(0xFF800000);
      for (int t = l0 / kTileWords; t <= (l1 - 1) / kTileWords; ++t)
        tmax = fmaxf(tmax, a.partial[row * a.ntiles + t].x);
      if (tmax < zthr) cw = l1;
    }
    uint32_t bits = cw < l1 ? word(cw) : 0u;
    while (true) {
      int code[kBatch];
      int32_t node[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        while (bits == 0u && cw < l1) {
          before += __popc(word(cw));
          ++cw;
          bits = cw < l1 ? word(cw) : 0u;
        }
        code[u] = -1;
        node[u] = -1;
        if (bits != 0u) {
          const int bpos = __ffs(bits) - 1;
          const uint32_t full_word = word(cw);
          code[u] = cw * 32 + bpos;
          if (brow)
            node[u] = static_cast<int32_t>(o0 + before +
                                           __popc(full_word & ((1u << bpos) - 1u)));
          bits &= bits - 1u;
        }
      }
      if (!__any_sync(kFull, code[0] >= 0)) break;
      float z[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        z[u] = code[u] >= 0 ? __ldcg(a.zlog + row * a.V + code[u]) : 0.f;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const bool has = code[u] >= 0 && z[u] >= zthr;
        if (!__any_sync(kFull, has)) continue;
        const float score = s + (z[u] - lse);
        warp_bin(ctl->hist, has, score_bin(score, C), wb.binned, &ctl->hist_total);
        warp_offer_nc(wb, has, make_key(score, idx0 + static_cast<uint32_t>(code[u])), node[u],
                      static_cast<uint32_t>(a.n), lane, sinks);
        zthr = zthreshold(wb.thr, s, lse);
      }
    }
    __syncwarp();
    refresh_thr(wb, ctl, static_cast<uint32_t>(a.n), C, lane, sinks);
  };

  auto flush = [&]() -> bool {
    team_sync(team);
    const int nh = min(*reinterpret_cast<volatile int*>(heavy_count), kHeavyList);
    for (int h = 0; h < nh; ++h) do_row(heavy[h], cur_r, warp, kSelWarps);
    team_sync(team);
    if (team.tid == 0) *heavy_count = 0;
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
    f.cw = a.Cw;
    f.sort_keys = wkeys;
    f.sort_vals = wvals;
    f.sort_cap = kSelWarps * a.Cw;
    f.radix_hist = cta_hist;
    f.wvals = wvals;
    f.rank_P = whist;
    f.rank_cur = whist + kHistBins;
    f.direct_keys = nullptr;
    f.direct_vals = nullptr;
    f.direct_cap = 0;
    const bool stop = segment_flush(team, wb, ctl, f, writer);
    wb.count = 0;
    wb.thr = 0ull;
    if (stop) return true;
    if (cur_r < r_last) C = request_reference(a, team, ctl, cur_r + 1, ref_slot ^= 1);
    ++cur_r;
    return false;
  };

  bool stopped = false;
  for (int i = 0; i < seq_count && !stopped; ++i) {
    const int64_t row = seq_first + seq_stride * i;
    const int r = static_cast<int>(row / a.B_in);
    while (r > cur_r && !stopped) stopped = flush();
    if (stopped) break;
    if (!a.coop && a.layout) {
      // A parent with very many children waits for the segment end, where all
      // warps of the CTA walk it together (one warp alone would hold the CTA).
      const int32_t pn = a.parent_nodes[row];
      if (pn >= 0 && a.parent_scores[row] != __int_as_float(0xFF800000) &&
          a.off[pn + 1] - a.off[pn] > kHeavyChildren) {
        int slot = 0;
        if (lane == 0) slot = atomicAdd(heavy_count, 1);
        slot = __shfl_sync(kFull, slot, 0);
        if (slot < kHeavyList) {
          if (lane == 0) heavy[slot] = row;
          continue;
        }
      }
    }
    do_row(row, r, part, nparts);
  }
  if (!stopped)
    while (cur_r <= r_last)
      if (flush()) break;
}

}  // namespace

// Host: bitmap, GEMM and selection launches of one fused step.
int launch_fused_lmhead(const sidbeam_trie* trie, int step, const void* hidden,
                        const void* w_sid, int d, const float* parent_scores,
                        const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                        float* out_scores, int32_t* out_parent, int32_t* out_code,
                        int32_t* out_node, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  const int64_t M = static_cast<int64_t>(R) * B_in;
  const Partition part = make_partition(R, B_in, std::min(device_sm_count(), 640));
  const FusedLayout L = fused_layout(R, part.maxG, n_out, M, V);
  if (!workspace || workspace_bytes < L.total)
    return set_error(SIDBEAM_ERR_WORKSPACE, "fused_lmhead_step: workspace of %zu bytes, need %zu",
                     workspace_bytes, L.total);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const int words = (V + 31) / 32;
  const int ntiles = (V + kLmheadTileN - 1) / kLmheadTileN;
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.sel.status);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(w + L.bitmap);
  const StepTrie* st = trie ? &trie->steps[step] : nullptr;

  if (st) {
    BitmapArgs b{};
    b.parent_scores = parent_scores;
    b.parent_nodes = parent_nodes;
    b.M = M;
    b.layout = st->layout;
    b.off = st->off;
    b.mask = st->mask;
    b.mask_stride = st->mask_stride;
    b.codes = st->codes;
    b.n_parent = st->n_parent;
    b.words = words;
    b.bitmap = bitmap;
    b.status = status;
    int64_t g = (M + kBitmapWarps - 1) / kBitmapWarps;
    if (g > 148 * 8) g = 148 * 8;
    const size_t sbytes = static_cast<size_t>(kBitmapWarps) * words * 4;  // <= 32 KB (V <= 32768)
    child_bitmap_kernel<<<static_cast<unsigned>(g), kBitmapWarps * 32, sbytes, stream>>>(b);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_error(e, "fused_lmhead_step: bitmap launch");
  }

  GemmArgs g{};
  g.M = static_cast<int>(M);
  g.N = V;
  g.K = d;
  g.mode = kLmheadFused;
  g.logits = reinterpret_cast<float*>(w + L.zlog);
  g.ld_out = V;
  g.partial = reinterpret_cast<float2*>(w + L.partial);
  g.bitmap = st ? bitmap : nullptr;
  g.words = words;
  g.status = status;
  int rc = launch_lmhead_gemm(hidden, w_sid, g, stream);
  if (rc != SIDBEAM_OK) return rc;

  SelArgs s{};
  s.parent_scores = parent_scores;
  s.parent_nodes = parent_nodes;
  s.R = R;
  s.B_in = B_in;
  s.n = n_out;
  s.V = V;
  s.layout = st ? st->layout : 0;
  s.off = st ? st->off : nullptr;
  s.partial = g.partial;
  s.ntiles = ntiles;
  s.bitmap = st ? bitmap : nullptr;
  s.words = words;
  s.zlog = g.logits;
  s.out_scores = out_scores;
  s.out_parent = out_parent;
  s.out_code = out_code;
  s.out_node = out_node;
  s.status = status;
  s.tickets = reinterpret_cast<uint32_t*>(w + L.sel.tickets);
  s.request_thr = reinterpret_cast<unsigned long long*>(w + L.sel.request_thr);
  s.part_count = reinterpret_cast<uint32_t*>(w + L.sel.part_count);
  s.part_keys = reinterpret_cast<unsigned long long*>(w + L.sel.part_keys);
  s.part_vals = reinterpret_cast<int32_t*>(w + L.sel.part_vals);
  s.ghist = reinterpret_cast<uint32_t*>(w + L.sel.ghist);
  s.part = part;
  int npow2 = 1;
  while (npow2 < n_out) npow2 <<= 1;
  // Warp buffers: n plus 512 entries of slack, so that parents with thousands
  // of children above the bound compact their buffers rarely.
  s.Cw = std::max((n_out + 31) / 32 * 32 + 512, (npow2 + kSelWarps - 1) / kSelWarps / 32 * 32 + 32);
  s.coop = part.rows_per_cta < kSelWarps ? 1 : 0;
  const size_t smem = ((sizeof(SelCtl) + 127) / 128) * 128 + 1024 + 8192 + kHeavyList * 8 + 128 +
                      static_cast<size_t>(kSelWarps) * s.Cw * 12;
  if (smem > static_cast<size_t>(kSmemBudget))
    return set_error(SIDBEAM_ERR_INVALID_ARG, "fused_lmhead_step: n_out=%d too large", n_out);
  cudaError_t e = cudaFuncSetAttribute(lmhead_select_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_error(e, "fused_lmhead_step: cudaFuncSetAttribute");
  lmhead_select_kernel<<<part.grid, kSelWarps * 32, smem, stream>>>(s);
  e = cudaGetLastError();
  return e == cudaSuccess ? SIDBEAM_OK : cuda_error(e, "fused_lmhead_step: select launch");
}

size_t fused_lmhead_workspace(int R, int B_in, int n_out, int V) {
  const Partition part = make_partition(R, B_in, std::min(device_sm_count(), 640));
  return fused_layout(R, part.maxG, n_out, static_cast<int64_t>(R) * B_in, V).total;
}

}  // namespace sidbeam
