// compact.cu -- KV compaction after acceptance (sm_100a).
//
// Under continuous batching every sequence accepts a different number of drafted tokens, and
// handling those per-sequence lengths is the main engineering difficulty of landing tree
// verification in an engine ("Eagle-4 Released: Outpaces DFlash2 and DSpark ...", section
// "Current Limitation").  After the walk, the root's and the accepted nodes' K/V rows (this
// step's tree K/V, in path order) are copied to the request's next cache slots, layer by layer.
//
// One CTA per (request, layer): it validates the request's accept length and path, then streams
// the 2 x (a + 1) rows of hkv * 128 bf16 with 16-byte vector loads and stores.  The copy is a
// bit copy and is HBM-bound.
#include "kernels.cuh"

namespace etree {


__global__ void __launch_bounds__(256) kv_compact_kernel(CompactParams p) {
  __shared__ int src_s[64];
  __shared__ int info_s[2];
  const int r = blockIdx.x;
  const int layer = blockIdx.y;
  if (threadIdx.x == 0) {
    const int base = p.cu_nodes[r];
    const int n = p.cu_nodes[r + 1] - base;
    const int a = p.accept_len[r];
    const int L = p.kv_len[r];
    int ok = 1, detail = DET_NONE, code = ETREE_OK;
    if (n < 1 || n > p.n_max || a < 0 || a >= n || L < 0) {
      ok = 0;
      code = ETREE_EDEVICE;
      detail = DET_BAD_PATH;
    } else if ((int64_t)L + a + 1 > (int64_t)p.slot_cap[r]) {
      ok = 0;
      code = ETREE_ENOSPACE;
      detail = DET_CAPACITY;
    } else {
      for (int k = 0; k <= a; ++k) {
        const int j = p.path[(size_t)r * ETREE_PATH_STRIDE + k];
        if (j < 0 || j >= n) {
          ok = 0;
          code = ETREE_EDEVICE;
          detail = DET_BAD_PATH;
          break;
        }
        src_s[k] = base + j;
      }
    }
    if (!ok && layer == 0) report(p.ws, code, detail);
    if (layer == 0) p.kv_len_out[r] = ok ? L + a + 1 : L;
    info_s[0] = ok ? a + 1 : 0;
  }
  __syncthreads();
  const int rows = info_s[0];
  if (rows == 0) return;
  const int64_t dst0 = p.slot_base[r] + p.kv_len[r];
  const uint4* kt = p.k_tree + (size_t)layer * p.tree_layer_stride16;
  const uint4* vt = p.v_tree + (size_t)layer * p.tree_layer_stride16;
  uint4* kc = p.k_cache + (size_t)layer * p.cache_layer_stride16;
  uint4* vc = p.v_cache + (size_t)layer * p.cache_layer_stride16;
  const int per = rows * p.row16;
  // K and V interleaved in one index space so both streams are in flight together
  for (int i = threadIdx.x; i < 2 * per; i += blockDim.x) {
    const int which = i >= per;
    const int e = which ? i - per : i;
    const int k = e / p.row16, c = e - k * p.row16;
    const size_t src = (size_t)src_s[k] * p.row16 + c;
    const size_t dst = (size_t)(dst0 + k) * p.row16 + c;
    if (which)
      vc[dst] = __ldg(vt + src);
    else
      kc[dst] = __ldg(kt + src);
  }
}

cudaError_t launch_compact(const CompactParams& p, cudaStream_t s) {
  dim3 grid(p.B, p.n_layers);
  kv_compact_kernel<<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace etree
