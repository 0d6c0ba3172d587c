// catalog_score_topk: one-pass scoring of every catalog SID, then top-K.
//
// SPRINT (paper summary), inference paragraph: every valid SID of the prefix
// trie is scored by the sum of its tokens' per-position log-probabilities (a
// lookup in an L-by-M table per request), and the K best are returned.
//
// With a user vector u_r per request and an embedding e_j per catalog SID the
// score also gets the SID-level similarity term of that paragraph (and of the
// closing paragraph: one pass gives the table and a user vector; scoring a SID
// is a lookup plus one matrix product): score += <u_r, e_j>, the [R x d] x
// [N x d]^T product computed pair by pair next to the lookup, in fp32 from the
// bf16 embeddings (four interleaved partial sums, added pairwise at the end).
//
// (request, leaf) pairs are laid out request-major and split evenly over the
// CTAs, exactly like beam rows in beam_step. A CTA keeps the current
// request's table in shared memory. Token sums: each lane scores 8
// consecutive leaves at a time (one 16-byte load of their codes per level, all
// levels' loads in flight before the first lookup), a warp 256; with the
// similarity term a lane scores one leaf at a time. Candidates go through the
// same warp / CTA / request top-n machinery as beam_step (topn.cuh).
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

constexpr int kScoreWarps = 8;
constexpr int kLeavesPerLane = 8;  // token sums: consecutive leaves per lane (one 16-byte code load)
constexpr int kLevelBatch = 6;     // levels whose code loads are issued before the lookups

struct ScoreConfig {
  int W, Cw, ctas_per_sm;
  int off_ctl, off_chist, off_whist, off_table, off_user, off_wkeys, off_wvals, smem_bytes;
};

struct ScoreArgs {
  const uint16_t* leaf_codes;  // [depth][stride], stride a multiple of 8, zero past N
  int64_t stride;
  int64_t N;
  int depth;
  const float* logp;  // [R][depth][Vmax]
  int Vmax;
  int K;
  float* out_scores;
  int32_t* out_leaf;
  uint32_t* status;
  uint32_t* tickets;
  unsigned long long* request_thr;
  uint32_t* part_count;
  unsigned long long* part_keys;
  int32_t* part_vals;
  uint32_t* ghist;
  Partition part;
  ScoreConfig cfg;
  const float* user;      // [R][d] f32, or null (no similarity term)
  const uint16_t* emb;    // [N][d] bf16 bits, leaf-id order
  int d;                  // multiple of 8
  const float* emb_norm;  // max_j ||e_j||, for the histogram reference
};

struct ScoreWriter {
  float* scores;
  int32_t* leaf;
  int K;
  __device__ __forceinline__ void operator()(int r, int i, uint64_t key, int32_t, bool valid) const {
    const size_t o = static_cast<size_t>(r) * K + i;
    scores[o] = valid ? key_score(key) : __int_as_float(0xFF800000);
    leaf[o] = valid ? static_cast<int32_t>(key_idx(key)) : -1;
  }
};

// max_j ||e_j||_2 of the embedding rows (one warp per row, atomicMax on the
// bits of a non-negative float, which order like the values); *out must start
// at zero.
__global__ void emb_norm_kernel(const uint16_t* emb, int64_t N, int d, float* out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  float best = 0.f;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       j < N; j += warps) {
    float s = 0.f;
    for (int k = lane; k < d; k += 32) {
      const float x = __uint_as_float(static_cast<uint32_t>(emb[j * d + k]) << 16);
      s = fmaf(x, x, s);
    }
    best = fmaxf(best, warp_sum(s));
  }
  if (lane == 0) atomicMax(reinterpret_cast<unsigned*>(out), __float_as_uint(sqrtf(best)));
}

template <int SIM>
__global__ void __launch_bounds__(kScoreWarps * 32, 2)
    catalog_score_kernel(const __grid_constant__ ScoreArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const ScoreConfig& cfg = a.cfg;
  SelCtl* ctl = reinterpret_cast<SelCtl*>(smem + cfg.off_ctl);
  uint32_t* cta_hist = reinterpret_cast<uint32_t*>(smem + cfg.off_chist);
  uint32_t* whist = reinterpret_cast<uint32_t*>(smem + cfg.off_whist);
  float* table = reinterpret_cast<float*>(smem + cfg.off_table);
  float* user = reinterpret_cast<float*>(smem + cfg.off_user);
  uint64_t* wkeys = reinterpret_cast<uint64_t*>(smem + cfg.off_wkeys);
  int32_t* wvals = reinterpret_cast<int32_t*>(smem + cfg.off_wvals);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Team team{static_cast<int>(threadIdx.x), cfg.W * 32, warp, lane, cfg.W};
  if (threadIdx.x == 0) {
    ctl->cta_thr = 0ull;
    ctl->abort_flag = 0;
    ctl->counter = 0;
    ctl->hist_total = 0u;
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) ctl->hist[i] = 0u;
  WarpBuf wb{wkeys + static_cast<size_t>(warp) * cfg.Cw, wvals + static_cast<size_t>(warp) * cfg.Cw,
             whist + warp * 256, cfg.Cw, 0, 0ull, 0};
  const ScoreWriter writer{a.out_scores, a.out_leaf, a.K};
  int64_t row_lo, row_hi;
  a.part.range(static_cast<int>(blockIdx.x), row_lo, row_hi);
  const int tsize = a.depth * a.Vmax;

  for (int64_t seg_lo = row_lo; seg_lo < row_hi;) {
    const int r = static_cast<int>(seg_lo / a.N);
    const int64_t seg_hi = min(row_hi, static_cast<int64_t>(r + 1) * a.N);
    const float* src = a.logp + static_cast<size_t>(r) * tsize;
    for (int i = threadIdx.x; i < tsize; i += blockDim.x) table[i] = src[i];
    if (SIM)
      for (int i = threadIdx.x; i < a.d; i += blockDim.x)
        user[i] = a.user[static_cast<size_t>(r) * a.d + i];
    team_sync(team);
    const ThrSinks sinks{&ctl->cta_thr, a.request_thr + r};
    // Histogram reference: the largest possible SID score of this request
    // (sum over positions of the best code); every warp computes the same value.
    float C = 0.f;
    for (int l = 0; l < a.depth; ++l) {
      float mx = __int_as_float(0xFF800000);
      for (int c = lane; c < a.Vmax; c += 32) mx = fmaxf(mx, table[l * a.Vmax + c]);
      C += warp_max(mx);
    }
    if (SIM) {  // the similarity adds at most ||u_r|| max_j ||e_j|| (Cauchy-Schwarz)
      float uu = 0.f;
      for (int k = lane; k < a.d; k += 32) uu = fmaf(user[k], user[k], uu);
      C += sqrtf(warp_sum(uu)) * *a.emb_norm;
    }
    if (!(C > __int_as_float(0xFF800000) && C < __int_as_float(0x7F800000))) C = 0.f;
    const int64_t j_lo = seg_lo - static_cast<int64_t>(r) * a.N;
    const int64_t j_hi = seg_hi - static_cast<int64_t>(r) * a.N;
    int batches = 0;
    if constexpr (!SIM) {
      // Lane: leaves jv .. jv+7 (jv a multiple of 8; those outside [j_lo, j_hi)
      // are computed from the zero padding or a neighbour's codes and dropped).
      constexpr int E = kLeavesPerLane;
      const int64_t jstart = j_lo & ~static_cast<int64_t>(E - 1);
      // Up to kLevelBatch levels: the next block's codes are loaded while this
      // block's lookups run (software pipelining, one block ahead).
      const bool pf = a.depth <= kLevelBatch;
      uint4 qn[kLevelBatch];
      if (pf) {
        const int64_t jv0 =
            jstart + static_cast<int64_t>(warp) * 32 * E + static_cast<int64_t>(E) * lane;
#pragma unroll
        for (int u = 0; u < kLevelBatch; ++u) {
          qn[u] = make_uint4(0u, 0u, 0u, 0u);
          if (jv0 < j_hi && u < a.depth)
            qn[u] = __ldg(reinterpret_cast<const uint4*>(
                a.leaf_codes + static_cast<int64_t>(u) * a.stride + jv0));
        }
      }
      for (int64_t jb = jstart + static_cast<int64_t>(warp) * 32 * E; jb < j_hi;
           jb += static_cast<int64_t>(cfg.W) * 32 * E) {
        const int64_t jv = jb + static_cast<int64_t>(E) * lane;
        const bool any_in = jv < j_hi;
        float sc[E];
        for (int l0 = 0; l0 < a.depth; l0 += kLevelBatch) {
          uint4 q[kLevelBatch];
          if (l0 == 0 && pf) {
#pragma unroll
            for (int u = 0; u < kLevelBatch; ++u) q[u] = qn[u];
          } else {
#pragma unroll
            for (int u = 0; u < kLevelBatch; ++u) {
              q[u] = make_uint4(0u, 0u, 0u, 0u);
              if (any_in && l0 + u < a.depth)
                q[u] = __ldg(reinterpret_cast<const uint4*>(
                    a.leaf_codes + static_cast<int64_t>(l0 + u) * a.stride + jv));
            }
          }
          if (l0 == 0 && pf) {  // next iteration's codes in flight during these lookups
            const int64_t jn = jv + static_cast<int64_t>(cfg.W) * 32 * E;
#pragma unroll
            for (int u = 0; u < kLevelBatch; ++u) {
              qn[u] = make_uint4(0u, 0u, 0u, 0u);
              if (jn < j_hi && u < a.depth)
                qn[u] = __ldg(reinterpret_cast<const uint4*>(
                    a.leaf_codes + static_cast<int64_t>(u) * a.stride + jn));
            }
          }
#pragma unroll
          for (int u = 0; u < kLevelBatch; ++u) {
            if (l0 + u < a.depth) {
              const float* tl = table + (l0 + u) * a.Vmax;
              const uint32_t w4[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
              for (int e = 0; e < E; ++e) {
                const float v = tl[(w4[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu];
                sc[e] = (l0 + u == 0) ? v : sc[e] + v;  // levels added in order
              }
            }
          }
        }
        bool pass[E];
        bool any = false;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int64_t j = jv + e;
          pass[e] = j >= j_lo && j < j_hi &&
                    make_key(sc[e], static_cast<uint32_t>(j)) >= wb.thr;
          any |= pass[e];
        }
        if (!__any_sync(0xFFFFFFFFu, any)) continue;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint32_t j = static_cast<uint32_t>(jv + e);
          const uint64_t key = make_key(sc[e], j);
          const bool ok = pass[e] && key >= wb.thr;  // the threshold may have risen
          if (!__any_sync(0xFFFFFFFFu, ok)) continue;
          warp_bin(ctl->hist, ok, score_bin(sc[e], C), wb.binned, &ctl->hist_total);
          if ((++batches & 7) == 0)
            refresh_thr(wb, ctl, static_cast<uint32_t>(a.K), C, lane, sinks);
          warp_offer(wb, ok, key, static_cast<int32_t>(j), static_cast<uint32_t>(a.K), lane,
                     sinks);
        }
      }
    }
    for (int64_t j0 = j_lo + static_cast<int64_t>(warp) * 32; SIM && j0 < j_hi;
         j0 += static_cast<int64_t>(cfg.W) * 32) {
      const int64_t j = j0 + lane;
      const bool valid = j < j_hi;
      float score = 0.f;
      if (valid) {
        score = table[a.leaf_codes[j]];
        for (int l = 1; l < a.depth; ++l)
          score += table[l * a.Vmax + a.leaf_codes[static_cast<int64_t>(l) * a.stride + j]];
        if (SIM) {  // <u_r, e_j>: 16-byte loads of the leaf's bf16 row, four partial sums
          const uint4* er = reinterpret_cast<const uint4*>(a.emb + j * a.d);
          float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
          const float4* u4 = reinterpret_cast<const float4*>(user);  // 16-byte aligned region
#pragma unroll 2
          for (int k8 = 0; k8 < (a.d >> 3); ++k8) {
            const uint4 q = __ldg(er + k8);
            const float4 ua = u4[2 * k8], ub = u4[2 * k8 + 1];  // broadcast loads
            d0 = fmaf(__uint_as_float(q.x << 16), ua.x, d0);
            d1 = fmaf(__uint_as_float(q.x & 0xFFFF0000u), ua.y, d1);
            d2 = fmaf(__uint_as_float(q.y << 16), ua.z, d2);
            d3 = fmaf(__uint_as_float(q.y & 0xFFFF0000u), ua.w, d3);
            d0 = fmaf(__uint_as_float(q.z << 16), ub.x, d0);
            d1 = fmaf(__uint_as_float(q.z & 0xFFFF0000u), ub.y, d1);
            d2 = fmaf(__uint_as_float(q.w << 16), ub.z, d2);
            d3 = fmaf(__uint_as_float(q.w & 0xFFFF0000u), ub.w, d3);
          }
          score += (d0 + d1) + (d2 + d3);
        }
      }
      const uint64_t key = make_key(score, static_cast<uint32_t>(j));
      const bool pass = valid && key >= wb.thr;
      if (!__any_sync(0xFFFFFFFFu, pass)) continue;
      warp_bin(ctl->hist, pass, score_bin(score, C), wb.binned, &ctl->hist_total);
      if ((++batches & 7) == 0) refresh_thr(wb, ctl, static_cast<uint32_t>(a.K), C, lane, sinks);
      warp_offer(wb, pass, key, static_cast<int32_t>(j), static_cast<uint32_t>(a.K), lane, sinks);
    }
    FlushArgs f;
    f.n = a.K;
    f.r = r;
    f.k = static_cast<int>(blockIdx.x) - a.part.first_cta(r);
    f.G = a.part.contributors(r);
    f.maxG = a.part.maxG;
    f.pcap = partial_cap(a.K);
    f.part_keys = a.part_keys;
    f.part_vals = a.part_vals;
    f.part_count = a.part_count;
    f.tickets = a.tickets;
    f.request_thr = a.request_thr;
    f.wkeys = wkeys;
    f.cw = cfg.Cw;
    f.sort_keys = wkeys;
    f.sort_vals = wvals;
    f.sort_cap = cfg.W * cfg.Cw;
    f.ghist = a.ghist;
    f.C = C;
    f.radix_hist = cta_hist;
    f.wvals = wvals;
    f.rank_P = whist;  // the warps' radix scratch is free during a flush: 2 x 1024 words
    f.rank_cur = whist + kHistBins;
    f.direct_keys = nullptr;
    f.direct_vals = nullptr;
    f.direct_cap = 0;
    if (segment_flush(team, wb, ctl, f, writer)) return;
    seg_lo = seg_hi;
  }
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

bool choose_score_config(int depth, int Vmax, int K, int d, ScoreConfig* out) {
  ScoreConfig c{};
  c.W = kScoreWarps;
  static_assert(kScoreWarps * 256 >= 2 * dev::kHistBins, "rank-merge scratch lives in whist");
  int npow2 = 1;
  while (npow2 < K) npow2 <<= 1;
  // Warp buffers: K plus 128 entries of slack between compactions (small
  // enough that two CTAs of the wide-catalog shape share an SM).
  c.Cw = std::max(round_up(K, 32) + 128, round_up((npow2 + c.W - 1) / c.W, 32));
  int o = 0;
  c.off_ctl = o;
  o += round_up(static_cast<int>(sizeof(SelCtl)), 128);
  c.off_chist = o;
  o += 1024;
  c.off_whist = o;
  o += c.W * 1024;
  c.off_table = o;
  o = round_up(o + depth * Vmax * 4, 128);
  c.off_user = o;
  o = round_up(o + d * 4, 128);
  c.off_wkeys = o;
  o += c.W * c.Cw * 8;
  c.off_wvals = o;
  o += c.W * c.Cw * 4;
  c.smem_bytes = round_up(o, 128);
  if (c.smem_bytes > kSmemBudget) return false;
  c.ctas_per_sm = std::max(1, std::min(4, kSmemBudget / c.smem_bytes));
  *out = c;
  return true;
}

}  // namespace
}  // namespace sidbeam

using namespace sidbeam;
using sidbeam::dev::kMaxSegCounts;

static int score_vmax(const sidbeam_trie* t) {
  int v = 1;
  for (int l = 0; l < t->depth; ++l) v = std::max(v, t->V[l]);
  return v;
}

extern "C" size_t catalog_score_workspace_size(const sidbeam_trie* trie, int R, int K) {
  if (!trie || R < 1 || K < 1 || K > SIDBEAM_MAX_BEAM) return 0;
  ScoreConfig cfg;
  if (!choose_score_config(trie->depth, score_vmax(trie), K, 0, &cfg)) return 0;
  const Partition p = make_partition(
      R, trie->n_leaves, std::min(device_sm_count() * cfg.ctas_per_sm, kMaxSegCounts));
  return workspace_layout(R, p.maxG, K).total;
}

// Both entry points: the token-sum scorer (user == nullptr) and the one with
// the similarity term.
static int catalog_score_impl(const sidbeam_trie* trie, const float* logp, const float* user,
                              const uint16_t* emb, int d, int R, int K, float* out_scores,
                              int32_t* out_leaf, void* workspace, size_t workspace_bytes,
                              void* stream, const char* who) {
  if (!trie || !logp || !out_scores || !out_leaf)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
  if (R < 1 || K < 1 || K > SIDBEAM_MAX_BEAM)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "%s: R=%d K=%d", who, R, K);
  if (static_cast<int64_t>(R) * trie->n_leaves > (1ll << 40))
    return set_error(SIDBEAM_ERR_INVALID_ARG, "%s: R * leaves too large", who);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return set_error(SIDBEAM_ERR_WORKSPACE, "%s: workspace must be 256-byte aligned", who);
  const bool sim = user != nullptr;
  if (sim) {
    if (!emb) return set_error(SIDBEAM_ERR_INVALID_ARG, "%s: NULL sid_emb", who);
    if (d < 8 || d > 1024 || d % 8 != 0)
      return set_error(SIDBEAM_ERR_INVALID_ARG, "%s: d=%d must be a multiple of 8 in [8, 1024]",
                       who, d);
    if ((reinterpret_cast<uintptr_t>(emb) & 15u) != 0)
      return set_error(SIDBEAM_ERR_ALIGNMENT, "%s: sid_emb must be 16-byte aligned", who);
  }
  ScoreArgs a{};
  a.Vmax = score_vmax(trie);
  ScoreConfig base;
  if (!choose_score_config(trie->depth, a.Vmax, K, 0, &base) ||
      !choose_score_config(trie->depth, a.Vmax, K, sim ? d : 0, &a.cfg))
    return set_error(SIDBEAM_ERR_INVALID_ARG,
                     "%s: the [depth x V] table does not fit in shared memory", who);
  a.leaf_codes = trie->leaf_codes;
  a.stride = trie->leaf_codes_stride;
  a.N = trie->n_leaves;
  a.depth = trie->depth;
  a.logp = logp;
  a.K = K;
  a.out_scores = out_scores;
  a.out_leaf = out_leaf;
  a.user = user;
  a.emb = emb;
  a.d = sim ? d : 0;
  // The partition (and so the workspace) is the token-sum scorer's, whatever d.
  a.part = make_partition(
      R, trie->n_leaves, std::min(device_sm_count() * base.ctas_per_sm, kMaxSegCounts));
  const WorkspaceLayout ws = workspace_layout(R, a.part.maxG, K);
  if (!workspace || workspace_bytes < ws.total)
    return set_error(SIDBEAM_ERR_WORKSPACE, "%s: workspace of %zu bytes, need %zu", who,
                     workspace_bytes, ws.total);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<uint32_t*>(w + ws.status);
  a.tickets = reinterpret_cast<uint32_t*>(w + ws.tickets);
  a.request_thr = reinterpret_cast<unsigned long long*>(w + ws.request_thr);
  a.part_count = reinterpret_cast<uint32_t*>(w + ws.part_count);
  a.part_keys = reinterpret_cast<unsigned long long*>(w + ws.part_keys);
  a.part_vals = reinterpret_cast<int32_t*>(w + ws.part_vals);
  a.ghist = reinterpret_cast<uint32_t*>(w + ws.ghist);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (sim) {  // max_j ||e_j|| into the status block's free bytes, for the histogram reference
    float* norm = reinterpret_cast<float*>(w + ws.status + kEmbNormOffset);
    a.emb_norm = norm;
    e = cudaMemsetAsync(norm, 0, sizeof(float), st);
    if (e != cudaSuccess) return cuda_error(e, "catalog_score_topk_sim: memset");
    const int64_t blocks64 = std::min<int64_t>((a.N + 7) / 8, 148 * 8);
    emb_norm_kernel<<<static_cast<unsigned>(std::max<int64_t>(blocks64, 1)), 256, 0, st>>>(
        emb, a.N, d, norm);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_error(e, "catalog_score_topk_sim: norm launch");
  }
  const void* fn = sim ? reinterpret_cast<const void*>(&catalog_score_kernel<1>)
                       : reinterpret_cast<const void*>(&catalog_score_kernel<0>);
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, a.cfg.smem_bytes);
  if (e != cudaSuccess) return cuda_error(e, "catalog_score_topk: cudaFuncSetAttribute");
  if (sim)
    catalog_score_kernel<1><<<a.part.grid, a.cfg.W * 32, a.cfg.smem_bytes, st>>>(a);
  else
    catalog_score_kernel<0><<<a.part.grid, a.cfg.W * 32, a.cfg.smem_bytes, st>>>(a);
  e = cudaGetLastError();
  return e == cudaSuccess ? SIDBEAM_OK : cuda_error(e, "catalog_score_topk: launch");
}

extern "C" int catalog_score_topk(const sidbeam_trie* trie, const float* logp, int R, int K,
                                  float* out_scores, int32_t* out_leaf, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return catalog_score_impl(trie, logp, nullptr, nullptr, 0, R, K, out_scores, out_leaf,
                            workspace, workspace_bytes, stream, "catalog_score_topk");
}

extern "C" int catalog_score_topk_sim(const sidbeam_trie* trie, const float* logp,
                                      const float* user, const uint16_t* sid_emb, int d, int R,
                                      int K, float* out_scores, int32_t* out_leaf,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!user) return set_error(SIDBEAM_ERR_INVALID_ARG, "catalog_score_topk_sim: NULL user");
  return catalog_score_impl(trie, logp, user, sid_emb, d, R, K, out_scores, out_leaf, workspace,
                            workspace_bytes, stream, "catalog_score_topk_sim");
}
