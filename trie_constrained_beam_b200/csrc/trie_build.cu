// sid_trie_build and the trie accessors.
//
// flashrec 0.1.0 (PyPI page), Features > Decoding ("SID constraint"): the
// catalog trie is stored either densely or as CSR. Here every step t (level-t
// nodes -> level-(t+1) codes) gets its own layout:
//   dense: a V-bit child bitmask per node (rows padded to 16 bytes so one bulk
//          copy moves a row) plus the first child id per node;
//   CSR  : child id range per node plus the uint16 code of every child.
// Node ids are lexicographic ranks of the distinct prefixes of each level, so
// a node's children are consecutive ids in code order and leaf ids are the
// ranks of the sorted unique SIDs.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <memory>
#include <numeric>
#include <vector>

#include "internal.h"

namespace sidbeam {
namespace {

struct DeviceAllocs {
  std::vector<void*> ptrs;
  ~DeviceAllocs() {
    for (void* p : ptrs) cudaFree(p);
  }
  template <class T>
  cudaError_t alloc(T** p, size_t bytes) {
    void* q = nullptr;
    cudaError_t e = cudaMalloc(&q, bytes < 16 ? 16 : bytes);
    if (e == cudaSuccess) {
      ptrs.push_back(q);
      *p = static_cast<T*>(q);
    }
    return e;
  }
  void release() { ptrs.clear(); }
};

__global__ void leaf_codes_aos_kernel(const uint16_t* __restrict__ soa, int64_t stride,
                                      int64_t n, int depth, int32_t* __restrict__ out) {
  const int64_t total = n * depth;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t leaf = i / depth;
    const int l = static_cast<int>(i - leaf * depth);
    out[i] = soa[l * stride + leaf];
  }
}

}  // namespace
}  // namespace sidbeam

using namespace sidbeam;

extern "C" int sid_trie_build(const int32_t* sids, int64_t n_sids, int depth,
                              const int32_t* codes_per_level, const int32_t* layout_per_level,
                              void* stream_ptr, sidbeam_trie** out) {
  if (!sids || !codes_per_level || !out)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_build: NULL argument");
  if (depth < 1 || depth > SIDBEAM_MAX_DEPTH)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_build: depth %d outside [1, %d]", depth,
                     SIDBEAM_MAX_DEPTH);
  if (n_sids < 1 || n_sids > 0x7FFFFFFFll)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_build: n_sids %lld outside [1, 2^31-1]",
                     static_cast<long long>(n_sids));
  int bits_total = 0;
  for (int l = 0; l < depth; ++l) {
    const int V = codes_per_level[l];
    if (V < 1 || V > SIDBEAM_MAX_V)
      return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_build: V[%d] = %d outside [1, %d]", l,
                       V, SIDBEAM_MAX_V);
    if (layout_per_level) {
      const int lay = layout_per_level[l];
      if (lay != SIDBEAM_LAYOUT_AUTO && lay != SIDBEAM_LAYOUT_DENSE && lay != SIDBEAM_LAYOUT_CSR)
        return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_build: bad layout %d at level %d",
                         lay, l);
    }
    int b = 1;
    while ((1 << b) < V) ++b;
    bits_total += b;
  }
  for (int64_t i = 0; i < n_sids; ++i)
    for (int l = 0; l < depth; ++l) {
      const int32_t c = sids[i * depth + l];
      if (c < 0 || c >= codes_per_level[l])
        return set_error(SIDBEAM_ERR_BAD_CATALOG,
                         "sid_trie_build: row %lld level %d code %d outside [0, %d)",
                         static_cast<long long>(i), l + 1, c, codes_per_level[l]);
    }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);

  // 1. Sort input rows by (SID, row) and keep the first row of each SID.
  std::vector<uint32_t> order(static_cast<size_t>(n_sids));
  std::iota(order.begin(), order.end(), 0u);
  if (bits_total <= 64) {
    std::vector<std::pair<uint64_t, uint32_t>> kv(static_cast<size_t>(n_sids));
    for (int64_t i = 0; i < n_sids; ++i) {
      uint64_t k = 0;
      for (int l = 0; l < depth; ++l) {
        int b = 1;
        while ((1 << b) < codes_per_level[l]) ++b;
        k = (k << b) | static_cast<uint64_t>(sids[i * depth + l]);
      }
      kv[static_cast<size_t>(i)] = {k, static_cast<uint32_t>(i)};
    }
    std::sort(kv.begin(), kv.end());
    for (int64_t i = 0; i < n_sids; ++i) order[static_cast<size_t>(i)] = kv[i].second;
  } else {
    std::sort(order.begin(), order.end(), [&](uint32_t x, uint32_t y) {
      const int32_t* a = sids + static_cast<int64_t>(x) * depth;
      const int32_t* b = sids + static_cast<int64_t>(y) * depth;
      for (int l = 0; l < depth; ++l)
        if (a[l] != b[l]) return a[l] < b[l];
      return x < y;
    });
  }
  auto same_prefix = [&](uint32_t x, uint32_t y, int len) {
    const int32_t* a = sids + static_cast<int64_t>(x) * depth;
    const int32_t* b = sids + static_cast<int64_t>(y) * depth;
    for (int l = 0; l < len; ++l)
      if (a[l] != b[l]) return false;
    return true;
  };
  std::vector<uint32_t> leaf_row;  // input row of each leaf (first occurrence)
  leaf_row.reserve(static_cast<size_t>(n_sids));
  for (int64_t i = 0; i < n_sids; ++i)
    if (i == 0 || !same_prefix(order[i], order[i - 1], depth)) leaf_row.push_back(order[i]);
  order.clear();
  order.shrink_to_fit();
  const int64_t N = static_cast<int64_t>(leaf_row.size());

  // 2. Level nodes. first_leaf[l][q] = first leaf of level-l node q.
  std::vector<std::vector<uint32_t>> first_leaf(depth + 1);
  first_leaf[0].push_back(0);
  for (int l = 1; l <= depth; ++l) {
    std::vector<uint32_t>& fl = first_leaf[l];
    for (int64_t j = 0; j < N; ++j)
      if (j == 0 || !same_prefix(leaf_row[j], leaf_row[j - 1], l))
        fl.push_back(static_cast<uint32_t>(j));
    if (fl.size() > 0x7FFFFFFFu)
      return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_build: too many nodes at level %d", l);
  }

  std::unique_ptr<sidbeam_trie> t(new sidbeam_trie());
  t->depth = depth;
  cudaGetDevice(&t->device);
  for (int l = 0; l <= depth; ++l) t->n_nodes[l] = static_cast<int64_t>(first_leaf[l].size());
  t->n_leaves = N;
  DeviceAllocs dev;
  cudaError_t e = cudaSuccess;

  // 3. One structure per step t.
  for (int tt = 0; tt < depth; ++tt) {
    StepTrie& st = t->steps[tt];
    const int V = codes_per_level[tt];
    st.V = V;
    st.n_parent = t->n_nodes[tt];
    st.n_child = t->n_nodes[tt + 1];
    t->V[tt] = V;
    // Parent of each child node: the level-tt node containing its first leaf.
    // Walk children and parents together (both sorted by first leaf).
    std::vector<uint32_t> off(static_cast<size_t>(st.n_parent) + 1, 0u);
    std::vector<uint16_t> child_code(static_cast<size_t>(st.n_child));
    {
      const std::vector<uint32_t>& P = first_leaf[tt];
      const std::vector<uint32_t>& C = first_leaf[tt + 1];
      int64_t p = 0;
      for (int64_t q = 0; q < st.n_child; ++q) {
        while (p + 1 < st.n_parent && P[p + 1] <= C[q]) ++p;
        off[p + 1] += 1;
        child_code[q] = static_cast<uint16_t>(sids[static_cast<int64_t>(leaf_row[C[q]]) * depth + tt]);
      }
      for (int64_t i = 0; i < st.n_parent; ++i) off[i + 1] += off[i];
    }
    int lay = layout_per_level ? layout_per_level[tt] : SIDBEAM_LAYOUT_AUTO;
    if (lay == SIDBEAM_LAYOUT_AUTO)
      lay = (16 * st.n_child > static_cast<int64_t>(V) * st.n_parent) ? SIDBEAM_LAYOUT_DENSE
                                                                       : SIDBEAM_LAYOUT_CSR;
    st.layout = lay;
    st.mask_words = (V + 31) / 32;
    st.mask_stride = (st.mask_words + 3) / 4 * 4;
    const size_t off_bytes = (static_cast<size_t>(st.n_parent) + 1) * 4;
    if ((e = dev.alloc(&st.off, off_bytes)) != cudaSuccess) return cuda_error(e, "sid_trie_build");
    if ((e = cudaMemcpyAsync(st.off, off.data(), off_bytes, cudaMemcpyHostToDevice, stream)) !=
        cudaSuccess)
      return cuda_error(e, "sid_trie_build");
    st.bytes = off_bytes;
    if (lay == SIDBEAM_LAYOUT_DENSE) {
      const size_t words = static_cast<size_t>(st.n_parent) * st.mask_stride;
      std::vector<uint32_t> mask(words, 0u);
      for (int64_t p = 0; p < st.n_parent; ++p)
        for (uint32_t q = off[p]; q < off[p + 1]; ++q) {
          const int c = child_code[q];
          mask[static_cast<size_t>(p) * st.mask_stride + c / 32] |= 1u << (c % 32);
        }
      if ((e = dev.alloc(&st.mask, words * 4)) != cudaSuccess)
        return cuda_error(e, "sid_trie_build");
      if ((e = cudaMemcpyAsync(st.mask, mask.data(), words * 4, cudaMemcpyHostToDevice,
                               stream)) != cudaSuccess)
        return cuda_error(e, "sid_trie_build");
      if ((e = cudaStreamSynchronize(stream)) != cudaSuccess)
        return cuda_error(e, "sid_trie_build");
      st.bytes += words * 4;
    } else {
      const size_t nb = (static_cast<size_t>(st.n_child) + 8) * 2;
      child_code.resize(static_cast<size_t>(st.n_child) + 8, 0);
      if ((e = dev.alloc(&st.codes, nb)) != cudaSuccess) return cuda_error(e, "sid_trie_build");
      if ((e = cudaMemcpyAsync(st.codes, child_code.data(), nb, cudaMemcpyHostToDevice,
                               stream)) != cudaSuccess)
        return cuda_error(e, "sid_trie_build");
      if ((e = cudaStreamSynchronize(stream)) != cudaSuccess)
        return cuda_error(e, "sid_trie_build");
      st.bytes += nb;
    }
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return cuda_error(e, "sid_trie_build");
  }

  // 4. Leaf tables.
  {
    std::vector<int32_t> rows(leaf_row.begin(), leaf_row.end());
    // Rows of a multiple of 8 codes (16-byte aligned), zero-padded past N: a
    // scorer reads 8 consecutive leaves' codes with one 16-byte load.
    t->leaf_codes_stride = (N + 7) / 8 * 8 + 8;
    std::vector<uint16_t> soa(static_cast<size_t>(depth) * t->leaf_codes_stride, 0);
    for (int64_t j = 0; j < N; ++j)
      for (int l = 0; l < depth; ++l)
        soa[static_cast<size_t>(l) * t->leaf_codes_stride + j] =
            static_cast<uint16_t>(sids[static_cast<int64_t>(leaf_row[j]) * depth + l]);
    if ((e = dev.alloc(&t->leaf_rows, static_cast<size_t>(N) * 4)) != cudaSuccess)
      return cuda_error(e, "sid_trie_build");
    if ((e = dev.alloc(&t->leaf_codes, soa.size() * 2)) != cudaSuccess)
      return cuda_error(e, "sid_trie_build");
    if ((e = cudaMemcpyAsync(t->leaf_rows, rows.data(), static_cast<size_t>(N) * 4,
                             cudaMemcpyHostToDevice, stream)) != cudaSuccess)
      return cuda_error(e, "sid_trie_build");
    if ((e = cudaMemcpyAsync(t->leaf_codes, soa.data(), soa.size() * 2, cudaMemcpyHostToDevice,
                             stream)) != cudaSuccess)
      return cuda_error(e, "sid_trie_build");
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return cuda_error(e, "sid_trie_build");
    t->leaf_bytes = static_cast<size_t>(N) * 4 + soa.size() * 2;
  }
  dev.release();
  *out = t.release();
  return SIDBEAM_OK;
}

extern "C" int sid_trie_info(const sidbeam_trie* t, int level, int64_t* n_nodes, int* layout,
                             size_t* bytes) {
  if (!t) return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_info: NULL trie");
  if (level < 0 || level > t->depth)
    return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_info: level %d outside [0, %d]", level,
                     t->depth);
  if (n_nodes) *n_nodes = t->n_nodes[level];
  if (level < t->depth) {
    if (layout) *layout = t->steps[level].layout;
    if (bytes) *bytes = t->steps[level].bytes;
  } else {
    if (layout) *layout = -1;
    if (bytes) *bytes = t->leaf_bytes;
  }
  return SIDBEAM_OK;
}

extern "C" int sid_trie_leaf_rows(const sidbeam_trie* t, int32_t* out, void* stream) {
  if (!t || !out) return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_leaf_rows: NULL argument");
  const cudaError_t e =
      cudaMemcpyAsync(out, t->leaf_rows, static_cast<size_t>(t->n_leaves) * 4,
                      cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SIDBEAM_OK : cuda_error(e, "sid_trie_leaf_rows");
}

extern "C" int sid_trie_leaf_codes(const sidbeam_trie* t, int32_t* out, void* stream) {
  if (!t || !out) return set_error(SIDBEAM_ERR_INVALID_ARG, "sid_trie_leaf_codes: NULL argument");
  const int64_t total = t->n_leaves * t->depth;
  int64_t g = (total + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  leaf_codes_aos_kernel<<<static_cast<unsigned>(g), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      t->leaf_codes, t->leaf_codes_stride, t->n_leaves, t->depth, out);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SIDBEAM_OK : cuda_error(e, "sid_trie_leaf_codes");
}

extern "C" void sid_trie_free(sidbeam_trie* t) {
  if (!t) return;
  cudaDeviceSynchronize();
  for (int l = 0; l < t->depth; ++l) {
    cudaFree(t->steps[l].off);
    cudaFree(t->steps[l].mask);
    cudaFree(t->steps[l].codes);
  }
  cudaFree(t->leaf_rows);
  cudaFree(t->leaf_codes);
  delete t;
}
