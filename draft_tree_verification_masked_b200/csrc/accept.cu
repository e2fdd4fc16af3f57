// accept.cu -- per-row reductions of the LM-head partials and the acceptance walk (sm_100a).
//
// The target accepts the drafted prefix that is consistent with its own distribution and adds
// one token of its own after the first rejection ("Eagle-4 Released: Outpaces DFlash2 and DSpark
// ...", section "Technical Background").  With a tree, the accepted prefix is a root-to-node
// path (same section: a draft tree lets one verification cover several paths).  T = 0 is the
// deterministic greedy setting ("EAGLE-4 ... 961.6 tokens/s是怎么测出来的", whatsnewx.com);
// at T > 0 verification keeps the target's output distribution ("EAGLE-4 官方推理代码发布 ...",
// arex-research.com, paragraph on the repository's positioning), which the min(1, p/q) test
// with a residual resample achieves.
//
// One warp per node row reduces the row across the LM head's partial summaries; the warp that
// completes a request's last row then takes the request's acceptance step (a ballot walk over
// the <= 64 nodes at T = 0, the sequential accept test along the chain at T > 0).
#include "kernels.cuh"
#include "philox.cuh"

namespace etree {


// Merge (top1, id, top2) summaries: the larger top1 wins (lower id on equal values); the
// merged top2 is the larger of the winner's top2 and the loser's top1.
__device__ __forceinline__ void merge_top2(float& t1, int& id, float& t2, float o1, int oid,
                                           float o2) {
  const bool other_wins = (o1 > t1) || (o1 == t1 && oid >= 0 && (id < 0 || oid < id));
  if (other_wins) {
    t2 = fmaxf(o2, t1);
    t1 = o1;
    id = oid;
  } else {
    t2 = fmaxf(t2, o1);
  }
}

__device__ __forceinline__ void merge_key(float& k, int& id, float ok, int oid) {
  if (oid < 0) return;
  if (id < 0 || ok > k || (ok == k && oid < id)) {
    k = ok;
    id = oid;
  }
}

// Merge two (max, sum 2^(x - max)) summaries in log2 units; an empty side has max = -inf.
__device__ __forceinline__ void merge_lse(float& m, float& s, float om, float os) {
  if (om == -INFINITY) return;
  if (m == -INFINITY) {
    m = om;
    s = os;
    return;
  }
  const float nm = fmaxf(m, om);
  s = s * exp2f(m - nm) + os * exp2f(om - nm);
  m = nm;
}

// ---------------------------------------------------------------------------- row ownership
// Node rows are reduced one warp per row across many CTAs; the warp that finishes the last row
// of a request (a per-request arrival counter, zeroed by the LM-head GEMM that runs first) then
// takes that request's acceptance step.  Warps past the last row check one request each and
// answer malformed ones, which no row ever completes.

__device__ __forceinline__ bool request_ok(const AcceptParams& p, int r, int& base, int& n) {
  base = __ldg(p.cu_nodes + r);
  const int end = __ldg(p.cu_nodes + r + 1);
  n = end - base;
  return base >= 0 && end <= p.n_total && n >= 1 && n <= p.n_max;
}

// The well-formed request that holds node row `row`, or -1.
__device__ __forceinline__ int row_owner(const AcceptParams& p, int row, int& base, int& n) {
  int lo = 0, hi = p.B - 1;                      // largest r with cu_nodes[r] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.cu_nodes + mid) <= row) lo = mid; else hi = mid - 1;
  }
  if (!request_ok(p, lo, base, n) || row < base || row >= base + n) return -1;
  return lo;
}

// True in every lane of the warp that brings request r's arrivals to n; that warp then sees
// every other row's results (fence, atomic, fence).
__device__ __forceinline__ bool last_arrival(int32_t* cnt, int r, int n, int lane) {
  int last = 0;
  if (lane == 0) {
    __threadfence();
    last = atomicAdd(cnt + r, 1) == n - 1;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) __threadfence();
  return last != 0;
}

// ------------------------------------------------------------------------------------ T == 0
// Greedy walk of one request: from the root, follow the lowest-index child that carries
// argmax(current node); the node where no child matches gives the bonus token.
__device__ void walk_greedy(const AcceptParams& p, const int32_t* arg_ws, int r, int base, int n,
                            int lane, int* am, int* par, int* tok, int* pth) {
  int32_t* path = p.path + (size_t)r * ETREE_PATH_STRIDE;
  int32_t* outt = p.out_tokens + (size_t)r * ETREE_OUT_STRIDE;
  bool ok = true;
  for (int j = lane; j < 64; j += 32) {
    if (j < n) {
      const int pj = p.parent[base + j];
      ok = ok && ((j == 0) ? pj == -1 : (pj >= 0 && pj < j));
      par[j] = pj;
      tok[j] = p.tokens[base + j];
      am[j] = __ldcg(arg_ws + base + j);
    } else {
      par[j] = -2;
      tok[j] = -1;
      am[j] = -1;
    }
  }
  ok = __all_sync(0xffffffffu, ok);
  __syncwarp();
  if (!ok && lane == 0) report(p.ws, ETREE_EDEVICE, DET_BAD_PARENT);
  int u = 0, a = 0;
  if (lane == 0) pth[0] = 0;
  if (ok) {
    for (int step = 0; step < 64; ++step) {
      const int want = am[u];
      const bool m0 = lane >= 1 && par[lane] == u && tok[lane] == want;
      const bool m1 = par[lane + 32] == u && tok[lane + 32] == want;
      const unsigned b0 = __ballot_sync(0xffffffffu, m0);
      const unsigned b1 = __ballot_sync(0xffffffffu, m1);
      if (b0 == 0 && b1 == 0) break;
      const int c = b0 ? (__ffs(b0) - 1) : (32 + __ffs(b1) - 1);
      ++a;
      if (lane == 0) pth[a] = c;
      u = c;
    }
  }
  __syncwarp();
  const int bonus = am[u];
  for (int k = lane; k < 64; k += 32) path[k] = (k <= a) ? pth[k] : -1;
  for (int k = lane; k < 65; k += 32)
    outt[k] = (k < a) ? tok[pth[k + 1]] : (k == a ? bonus : -1);
  if (lane == 0) p.accept_len[r] = a;
}

// Outputs of a request with no valid tree: nothing accepted, no bonus.
__device__ void answer_malformed(const AcceptParams& p, int r, int lane) {
  int32_t* path = p.path + (size_t)r * ETREE_PATH_STRIDE;
  int32_t* outt = p.out_tokens + (size_t)r * ETREE_OUT_STRIDE;
  if (lane == 0) {
    report(p.ws, ETREE_EDEVICE, DET_BAD_NODES);
    p.accept_len[r] = 0;
  }
  path[lane] = -1;
  path[lane + 32] = -1;
  outt[lane] = -1;
  outt[lane + 32] = -1;
  if (lane == 0) outt[64] = -1;
}

// One warp per node row merges the row's (top1, id, top2) summaries into its argmax and
// top1 - top2 gap; the last row of a request walks it.
__global__ void __launch_bounds__(256) greedy_accept_kernel(AcceptParams p, int32_t* arg_ws,
                                                            int32_t* cnt) {
  __shared__ int am_s[8][64], par_s[8][64], tok_s[8][64], pth_s[8][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x * 8 + warp;
  if (item >= p.n_total + p.B) return;
  int base, n;
  if (item >= p.n_total) {
    const int r = item - p.n_total;
    if (!request_ok(p, r, base, n)) answer_malformed(p, r, lane);
    return;
  }
  const int row = item;
  const float4* part = p.part + (size_t)row * p.n_tiles;
  float t1 = -INFINITY, t2 = -INFINITY;
  int id = -1;
  int t = lane;
  for (; t + 96 < p.n_tiles; t += 128) {             // four loads in flight per lane
    const float4 a = part[t], b = part[t + 32], c = part[t + 64], d = part[t + 96];
    merge_top2(t1, id, t2, a.x, __float_as_int(a.y), a.z);
    merge_top2(t1, id, t2, b.x, __float_as_int(b.y), b.z);
    merge_top2(t1, id, t2, c.x, __float_as_int(c.y), c.z);
    merge_top2(t1, id, t2, d.x, __float_as_int(d.y), d.z);
  }
  for (; t < p.n_tiles; t += 32) {
    const float4 a = part[t];
    merge_top2(t1, id, t2, a.x, __float_as_int(a.y), a.z);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o1 = __shfl_xor_sync(0xffffffffu, t1, off);
    const int oid = __shfl_xor_sync(0xffffffffu, id, off);
    const float o2 = __shfl_xor_sync(0xffffffffu, t2, off);
    merge_top2(t1, id, t2, o1, oid, o2);
  }
  if (lane == 0) {
    arg_ws[row] = id;
    if (p.node_argmax) p.node_argmax[row] = id;
    if (p.node_gap) p.node_gap[row] = t1 - t2;
  }
  const int r = row_owner(p, row, base, n);
  if (r < 0 || !last_arrival(cnt, r, n, lane)) return;
  walk_greedy(p, arg_ws, r, base, n, lane, am_s[warp], par_s[warp], tok_s[warp], pth_s[warp]);
}

// ------------------------------------------------------------------------------------- T > 0
// Chain check and the child token of every row (read by the LM-head epilogue).
__global__ void chain_prep_kernel(AcceptParams p, int32_t* child_tok) {
  __shared__ int flag_s;
  const int r = blockIdx.x;
  const int base = p.cu_nodes[r];
  const int n = p.cu_nodes[r + 1] - base;
  if (n < 1 || n > p.n_max) return;
  if (threadIdx.x == 0) flag_s = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int pi = p.parent[base + i];
    if (i == 0 ? pi != -1 : pi != i - 1) atomicOr(&flag_s, 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    int ct = -1;
    if (flag_s == 0 && i + 1 < n) {
      ct = p.tokens[base + i + 1];
      if (ct < 0 || ct >= p.V) ct = -1;
    }
    child_tok[base + i] = ct;
  }
}

// The acceptance chain of one request (one warp): node k is kept while U_k q(x_k) < p(x_k),
// with p from the row's logit of x_k and its log-sum-exp; then the stop row's hidden state is
// copied out for the second (draw) pass.
__device__ void accept_chain(const AcceptParams& p, int r, int base, int n, int lane) {
  int32_t* path = p.path + (size_t)r * ETREE_PATH_STRIDE;
  int32_t* outt = p.out_tokens + (size_t)r * ETREE_OUT_STRIDE;
  bool chain = true;
  for (int i = lane; i < n; i += 32) {
    const int pi = p.parent[base + i];
    if (i == 0 ? pi != -1 : pi != i - 1) chain = false;
  }
  chain = __all_sync(0xffffffffu, chain);
  int a = 0, rejected = 0;
  if (!chain) {
    if (lane == 0) report(p.ws, ETREE_EUNSUPPORTED, DET_NOT_CHAIN);
  } else if (lane == 0) {
    for (int k = 1; k < n; ++k) {
      const int u = k - 1;
      const int x = p.tokens[base + k];
      if (x < 0 || x >= p.V) {
        report(p.ws, ETREE_EDEVICE, DET_BAD_TOKEN);
        rejected = 1;
        break;
      }
      const float px = exp2f(p.zchild[base + u] * p.k_log2 - __ldcg(p.lse2 + base + u));
      const float qx = __ldg(p.q_draft + (size_t)(base + u) * p.V + x);
      float U[8];
      uniforms8(p.seed, p.step, 0u, (uint32_t)k, (uint32_t)r, 1u, U);
      if (U[0] * qx < px) {
        ++a;
      } else {
        rejected = 1;
        break;
      }
    }
  }
  a = __shfl_sync(0xffffffffu, a, 0);
  rejected = __shfl_sync(0xffffffffu, rejected, 0);
  for (int k = lane; k < 64; k += 32) path[k] = (chain && k <= a) ? k : (k == 0 ? 0 : -1);
  for (int k = lane; k < 65; k += 32) outt[k] = (chain && k < a) ? p.tokens[base + k + 1] : -1;
  const int src = chain ? base + a : base;
  if (lane == 0) {
    p.accept_len[r] = chain ? a : 0;
    p.stop_row[r] = src;
    p.stop_node[r] = chain ? a : 0;
    p.mode[r] = chain ? rejected : 0;
  }
  const uint4* hs = reinterpret_cast<const uint4*>(p.hidden + (size_t)src * p.H);
  uint4* hd = reinterpret_cast<uint4*>(p.hid2 + (size_t)r * p.H);
  for (int i = lane; i < p.H / 8; i += 32) hd[i] = hs[i];
}

// One warp per node row merges the row's (max, sum) summaries into log2 sum 2^(z log2(e) / T);
// the last row of a request runs its acceptance chain.  Malformed requests accept nothing and
// draw from row 0 so that the second pass reads defined data.
__global__ void __launch_bounds__(256) chain_accept_kernel(AcceptParams p, int32_t* cnt) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x * 8 + warp;
  if (item >= p.n_total + p.B) return;
  int base, n;
  if (item >= p.n_total) {
    const int r = item - p.n_total;
    if (request_ok(p, r, base, n)) return;
    answer_malformed(p, r, lane);
    if (lane == 0) {
      p.stop_row[r] = 0;
      p.stop_node[r] = 0;
      p.mode[r] = 0;
    }
    const uint4* hs = reinterpret_cast<const uint4*>(p.hidden);
    uint4* hd = reinterpret_cast<uint4*>(p.hid2 + (size_t)r * p.H);
    for (int i = lane; i < p.H / 8; i += 32) hd[i] = hs[i];
    return;
  }
  const int row = item;
  const float4* part = p.part + (size_t)row * p.n_tiles;
  float m = -INFINITY, s = 0.f;
  int t = lane;
  for (; t + 96 < p.n_tiles; t += 128) {
    const float4 a = part[t], b = part[t + 32], c = part[t + 64], d = part[t + 96];
    merge_lse(m, s, a.x, a.y);
    merge_lse(m, s, b.x, b.y);
    merge_lse(m, s, c.x, c.y);
    merge_lse(m, s, d.x, d.y);
  }
  for (; t < p.n_tiles; t += 32) {
    const float4 a = part[t];
    merge_lse(m, s, a.x, a.y);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, off);
    const float os = __shfl_xor_sync(0xffffffffu, s, off);
    merge_lse(m, s, om, os);
  }
  if (lane == 0) p.lse2[row] = m + log2f(s);
  const int r = row_owner(p, row, base, n);
  if (r < 0 || !last_arrival(cnt, r, n, lane)) return;
  accept_chain(p, r, base, n, lane);
}

// The first level of the two-level draw, per request: the exponential race among the 128-id
// block totals (key W_b / E_b with E_b = -log U_b, stream 2), ties to the lowest block; the
// bonus is the inverse-CDF pick the GEMM epilogue made inside the winning block.  A residual
// with no positive weight anywhere (p <= q everywhere: p = q up to rounding) gives the argmax
// of p instead, taken from the per-block logit maxima.
__global__ void bonus_kernel(AcceptParams p) {
  const int r = blockIdx.x;
  const int lane = threadIdx.x;
  const int node = p.stop_node[r];
  const float4* row = p.part2 + (size_t)r * p.n_tiles2;
  float kb = -INFINITY, zm = -INFINITY;
  int ib = -1, iz = -1;
  for (int g = lane; g * 8 < p.n_tiles2; g += 32) {
    float u[8];
    uniforms8(p.seed, p.step, (uint32_t)g, (uint32_t)node, (uint32_t)r, 2u, u);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int b = g * 8 + e;
      if (b < p.n_tiles2) {
        const float4 v = row[b];
        if (v.x > 0.f) merge_key(kb, ib, __fdividef(v.x, -logf(u[e])), __float_as_int(v.y));
        merge_key(zm, iz, v.z, __float_as_int(v.w));
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float okb = __shfl_xor_sync(0xffffffffu, kb, off);
    const int oib = __shfl_xor_sync(0xffffffffu, ib, off);
    const float ozm = __shfl_xor_sync(0xffffffffu, zm, off);
    const int oiz = __shfl_xor_sync(0xffffffffu, iz, off);
    merge_key(kb, ib, okb, oib);
    merge_key(zm, iz, ozm, oiz);
  }
  if (lane == 0) {
    const int base = p.cu_nodes[r];
    const int n = p.cu_nodes[r + 1] - base;
    if (n < 1 || n > p.n_max) return;
    const int a = p.accept_len[r];
    p.out_tokens[(size_t)r * ETREE_OUT_STRIDE + a] = ib >= 0 ? ib : iz;
  }
}

cudaError_t launch_accept_greedy(const AcceptParams& p, int32_t* arg_ws, int32_t* cnt,
                                 cudaStream_t s) {
  greedy_accept_kernel<<<(p.n_total + p.B + 7) / 8, 256, 0, s>>>(p, arg_ws, cnt);
  return cudaGetLastError();
}

cudaError_t launch_chain_prep(const AcceptParams& p, int32_t* child_tok, cudaStream_t s) {
  chain_prep_kernel<<<p.B, 64, 0, s>>>(p, child_tok);
  return cudaGetLastError();
}

cudaError_t launch_accept_chain(const AcceptParams& p, int32_t* cnt, cudaStream_t s) {
  chain_accept_kernel<<<(p.n_total + p.B + 7) / 8, 256, 0, s>>>(p, cnt);
  return cudaGetLastError();
}

cudaError_t launch_bonus(const AcceptParams& p, cudaStream_t s) {
  bonus_kernel<<<p.B, 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace etree
