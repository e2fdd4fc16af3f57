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


// One CTA per (request, chunk of layers).  Its first two warps read the request's accept length
// and path entries in parallel and validate them once; then all 256 threads stream the
// 2 x (a + 1) rows of every layer in the chunk, one 16-byte word per thread per row and
// tensor (K, V), four rows in flight per thread.
__global__ void __launch_bounds__(256) kv_compact_kernel(CompactParams p, int layers_per_cta) {
  __shared__ int src_s[64];
  __shared__ long long dst_s[64];
  __shared__ int rows_s, code_s, detail_s, bad_s, badpage_s;
  const int r = blockIdx.x;
  const int l0 = blockIdx.y * layers_per_cta;
  const int l1 = min(p.n_layers, l0 + layers_per_cta);
  const int tid = threadIdx.x;
  if (tid == 0) {
    const int base = p.cu_nodes[r];
    const int n = p.cu_nodes[r + 1] - base;
    const int a = p.accept_len[r];
    const int L = p.kv_len[r];
    int code = ETREE_OK, detail = DET_NONE;
    if (n < 1 || n > p.n_max || a < 0 || a >= n || L < 0) {
      code = ETREE_EDEVICE;
      detail = DET_BAD_PATH;
    } else if ((int64_t)L + a + 1 > (int64_t)p.slot_cap[r]) {
      code = ETREE_ENOSPACE;
      detail = DET_CAPACITY;
    }
    code_s = code;
    detail_s = detail;
    rows_s = code == ETREE_OK ? a + 1 : 0;
    bad_s = 0;
    badpage_s = 0;
  }
  __syncthreads();
  const int rows0 = rows_s;
  if (tid < rows0) {                                   // path entries and destinations
    const int base = p.cu_nodes[r];
    const int n = p.cu_nodes[r + 1] - base;
    const int j = p.path[(size_t)r * ETREE_PATH_STRIDE + tid];
    if (j < 0 || j >= n) atomicOr(&bad_s, 1);
    src_s[tid] = base + j;
    const long long pos = (long long)p.kv_len[r] + tid;
    if (!p.block_table) {
      dst_s[tid] = p.slot_base[r] + pos;
    } else {
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
    p.kv_len_out[r] = code == ETREE_OK ? p.kv_len[r] + rows0 : p.kv_len[r];
  }
  const int rows = (bad_s || badpage_s) ? 0 : rows0;
  if (rows == 0) return;
  const int w16 = p.row16;                            // 16-byte words per row
  for (int layer = l0; layer < l1; ++layer) {
    const uint4* kt = p.k_tree + (size_t)layer * p.tree_layer_stride16;
    const uint4* vt = p.v_tree + (size_t)layer * p.tree_layer_stride16;
    uint4* kc = p.k_cache + (size_t)layer * p.cache_layer_stride16;
    uint4* vc = p.v_cache + (size_t)layer * p.cache_layer_stride16;
    for (int c = tid; c < 2 * w16; c += blockDim.x) {
      const bool isv = c >= w16;
      const int cc = isv ? c - w16 : c;
      const uint4* src = isv ? vt : kt;
      uint4* dst = isv ? vc : kc;
      int k = 0;
      for (; k + 4 <= rows; k += 4) {
        uint4 v0 = __ldg(src + (size_t)src_s[k] * w16 + cc);
        uint4 v1 = __ldg(src + (size_t)src_s[k + 1] * w16 + cc);
        uint4 v2 = __ldg(src + (size_t)src_s[k + 2] * w16 + cc);
        uint4 v3 = __ldg(src + (size_t)src_s[k + 3] * w16 + cc);
        dst[(size_t)dst_s[k] * w16 + cc] = v0;
        dst[(size_t)dst_s[k + 1] * w16 + cc] = v1;
        dst[(size_t)dst_s[k + 2] * w16 + cc] = v2;
        dst[(size_t)dst_s[k + 3] * w16 + cc] = v3;
      }
      for (; k < rows; ++k) dst[(size_t)dst_s[k] * w16 + cc] = __ldg(src + (size_t)src_s[k] * w16 + cc);
    }
  }
}

cudaError_t launch_compact(const CompactParams& p, int sms, cudaStream_t s) {
  // spread the layers over enough CTAs to give every SM a few, at least one layer per CTA
  const int want = std::max(1, (4 * sms + p.B - 1) / p.B);
  const int chunks = std::min(p.n_layers, want);
  const int per = (p.n_layers + chunks - 1) / chunks;
  dim3 grid(p.B, (p.n_layers + per - 1) / per);
  kv_compact_kernel<<<grid, 256, 0, s>>>(p, per);
  return cudaGetLastError();
}

}  // namespace etree
