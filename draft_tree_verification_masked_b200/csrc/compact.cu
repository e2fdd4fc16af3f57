// compact.cu -- KV compaction after acceptance (sm_100a).
//
// Under continuous batching every sequence accepts a different number of drafted tokens, and
// handling those per-sequence lengths is the main engineering difficulty of landing tree
// verification in an engine ("Eagle-4 Released: Outpaces DFlash2 and DSpark ...", section
// "Current Limitation").  After the walk, the root's and the accepted nodes' K/V rows (this
// step's tree K/V, in path order) are copied to the request's next cache slots, layer by layer.
//
// The copy is a bit copy and is HBM-bound: every byte moved is read once and written once.
// With a paged cache the destination of each row goes through the request's block table.
#include <algorithm>

#include "kernels.cuh"

namespace etree {


// One CTA per (request, chunk of layers).  Thread 0 reads and validates the request's header
// while the first 64 threads read its path row; the first a + 1 threads then form the source
// rows and the destination slots.  The copy treats the chunk as a flat list of items, one item
// being one moved row (layer, k) for both tensors.  A row is w16 16-byte words for K followed by
// w16 for V; each thread owns every kCompactThreads-th word column and walks the items with
// kUnroll independent loads in flight before their stores, so a copy of a few rows per layer is
// not serialised layer by layer.  The shape (128 threads, 4 loads in flight, about 32 CTAs per
// SM) was the fastest of the swept ones at 64 layers for batches of 64 and 512 requests.
constexpr int kCompactThreads = 128;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kCompactThreads)
    kv_compact_kernel(CompactParams p, int layers_per_cta) {
  __shared__ int path_s[ETREE_PATH_STRIDE], src_s[64];
  __shared__ long long dst_s[64], slot0_s;
  __shared__ int rows_s, code_s, detail_s, bad_s, badpage_s, nbase_s, n_s, L_s;
  pdl_wait();                                      // the accept results (launch_pdl)
  const int r = blockIdx.x;
  const int l0 = blockIdx.y * layers_per_cta;
  const int l1 = min(p.n_layers, l0 + layers_per_cta);
  const int tid = threadIdx.x;
  // One DRAM round trip: the whole path row (it always has ETREE_PATH_STRIDE entries) is read
  // beside the request's header, before the accept length says how much of it is used.
  if (tid < ETREE_PATH_STRIDE) path_s[tid] = p.path[(size_t)r * ETREE_PATH_STRIDE + tid];
  if (tid == 0) {
    const int base = p.cu_nodes[r];
    const int n = p.cu_nodes[r + 1] - base;
    const int a = p.accept_len[r];
    const int L = p.kv_len[r];
    const int cap = p.slot_cap[r];
    const long long sb = p.slot_base[r];
    int code = ETREE_OK, detail = DET_NONE;
    if (n < 1 || n > p.n_max || a < 0 || a >= n || L < 0) {
      code = ETREE_EDEVICE;
      detail = DET_BAD_PATH;
    } else if ((int64_t)L + a + 1 > (int64_t)cap) {
      code = ETREE_ENOSPACE;
      detail = DET_CAPACITY;
    }
    code_s = code;
    detail_s = detail;
    rows_s = code == ETREE_OK ? a + 1 : 0;
    bad_s = 0;
    badpage_s = 0;
    nbase_s = base;
    n_s = n;
    L_s = L;
    slot0_s = sb + L;
  }
  __syncthreads();
  const int rows0 = rows_s;
  if (tid < rows0) {                                   // sources and destinations
    const int j = path_s[tid];
    if (j < 0 || j >= n_s) atomicOr(&bad_s, 1);
    src_s[tid] = nbase_s + j;
    if (!p.block_table) {
      dst_s[tid] = slot0_s + tid;
    } else {
      const long long pos = (long long)L_s + tid;
      const long long pi = pos >> p.page_shift;
      const int page = pi < p.max_pages ? p.block_table[(size_t)r * p.max_pages + pi] : -1;
      const long long slot = ((long long)page << p.page_shift) + (pos & ((1 << p.page_shift) - 1));
      if (page < 0 || slot >= p.cache_slots) atomicOr(&badpage_s, 1);
      dst_s[tid] = slot;
    }
  }
  __syncthreads();
  if (tid == 0 && blockIdx.y == 0) {
    int code = code_s, detail = detail_s;
    if (code == ETREE_OK && bad_s) {
      code = ETREE_EDEVICE;
      detail = DET_BAD_PATH;
    } else if (code == ETREE_OK && badpage_s) {
      code = ETREE_EDEVICE;
      detail = DET_BAD_PAGE;
    }
    if (code != ETREE_OK) report(p.ws, code, detail);
    p.kv_len_out[r] = L_s + (code == ETREE_OK ? rows0 : 0);
  }
  const int rows = (bad_s || badpage_s) ? 0 : rows0;
  if (rows == 0) return;
  const int w16 = p.row16;                            // 16-byte words per row and tensor
  const int cw = 2 * w16;                              // words per item (K row, then V row)
  const int span = min(cw, kCompactThreads);           // threads on one item
  const int groups = kCompactThreads / span;           // items side by side in the CTA
  const int g = tid / span;
  if (g >= groups) return;
  const int items = rows * (l1 - l0);
  for (int c = tid - g * span; c < cw; c += span) {
    const bool isv = c >= w16;
    const int cc = isv ? c - w16 : c;
    const uint4* src = (isv ? p.v_tree : p.k_tree) + cc;
    uint4* dst = (isv ? p.v_cache : p.k_cache) + cc;
    int layer = l0 + g / rows, k = g % rows;           // item g
    for (int i = g; i < items; i += groups * kUnroll) {
      uint4 v[kUnroll];
      size_t to[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (i + u * groups < items) {
          v[u] = __ldg(src + (size_t)layer * p.tree_layer_stride16 + (size_t)src_s[k] * w16);
          to[u] = (size_t)layer * p.cache_layer_stride16 + (size_t)dst_s[k] * w16;
        }
        k += groups;                                   // next item of this thread
        while (k >= rows) {
          k -= rows;
          ++layer;
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (i + u * groups < items) dst[to[u]] = v[u];
    }
  }
}

cudaError_t launch_compact(const CompactParams& p, int ctas, cudaStream_t s) {
  // about `ctas` CTAs over all requests, at least one layer per CTA
  const int want = std::max(1, (ctas + p.B - 1) / p.B);
  const int chunks = std::min(p.n_layers, want);
  const int per = (p.n_layers + chunks - 1) / chunks;
  dim3 grid(p.B, (p.n_layers + per - 1) / per);
  return launch_pdl(kv_compact_kernel, grid, dim3(kCompactThreads), 0, s, p, per);
}

}  // namespace etree
