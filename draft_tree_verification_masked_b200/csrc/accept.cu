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
#include <algorithm>

#include "kernels.cuh"
#include "philox.cuh"
#include "race.cuh"

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
  if (!ok) {                                       // no valid tree: nothing accepted, no bonus
    if (lane == 0) {
      report(p.ws, ETREE_EDEVICE, DET_BAD_PARENT);
      p.accept_len[r] = 0;
    }
    for (int k = lane; k < 64; k += 32) path[k] = -1;
    for (int k = lane; k < 65; k += 32) outt[k] = -1;
    return;
  }
  int u = 0, a = 0;
  if (lane == 0) pth[0] = 0;
  {
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
  pdl_wait();                                      // the LM-head summaries (launch_pdl)
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
  for (; t + 224 < p.n_tiles; t += 256) {            // eight loads in flight per lane
    float4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = part[t + 32 * u];
#pragma unroll
    for (int u = 0; u < 8; ++u) merge_top2(t1, id, t2, x[u].x, __float_as_int(x[u].y), x[u].z);
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
    p.cval[r] = (chain && rejected) ? 1.f : 0.f;
    p.rfloor[2 * r] = 0u;
    p.rfloor[2 * r + 1] = 0u;
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
      p.cval[r] = 0.f;
      p.rfloor[2 * r] = 0u;
      p.rfloor[2 * r + 1] = 0u;
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
  for (; t + 224 < p.n_tiles; t += 256) {            // eight loads in flight, merged in order
    float4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = part[t + 32 * u];
#pragma unroll
    for (int u = 0; u < 8; ++u) merge_lse(m, s, x[u].x, x[u].y);
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

// ---------------------------------------------------------------- T > 0 on branching trees
// Multi-candidate speculative sampling (the multi-step rule of SpecInfer, Miao et al. 2023): the
// children of node u are candidates drafted independently from q_u and are tested in index
// order against a running target r that starts at p_u; a rejection replaces r by
// norm(max(0, r - q_u)).  Each residual is r_i = max(0, p_u - c_i q_u) / N(c_i) with
// N(c) = sum_v max(0, p_u(v) - c q_u(v)), c_0 = 0, N(c_0) = 1, c_{i+1} = c_i + N(c_i), so the
// walk needs, per rejection that is followed by another sibling, one pass over row u's logits
// (materialised by the LM-head pass for rows with two or more children) and its q row.

// One CTA: per-node child counts, then a row of the caller's logit buffer for every node with
// two or more children (in node order).  Nodes past zbuf_rows get none: their requests are
// answered as malformed by the walk and the status reports ETREE_ENOSPACE.  With a buffer of at
// least n_total rows every node gets its own row (row g for node g), and the bonus draw reads the
// stop row's logits there instead of recomputing them.
__global__ void __launch_bounds__(1024) tree_prep_kernel(AcceptParams p, int32_t* ccount,
                                                         int32_t* zrow, int zbuf_rows) {
  __shared__ int32_t part_s[1024];
  const int tid = threadIdx.x, nt = blockDim.x;
  if (zbuf_rows >= p.n_total) {                       // every row materialised: row g is node g
    for (int g = tid; g < p.n_total; g += nt) zrow[g] = g;
    return;
  }
  for (int g = tid; g < p.n_total; g += nt) ccount[g] = 0;
  __syncthreads();
  for (int g = tid; g < p.n_total; g += nt) {
    int base, n;
    if (row_owner(p, g, base, n) < 0) continue;
    const int local = g - base, pl = p.parent[g];
    if (local >= 1 && pl >= 0 && pl < local) atomicAdd(ccount + base + pl, 1);
  }
  __syncthreads();
  // exclusive scan of the branching flags: each thread owns a contiguous segment
  const int seg = (p.n_total + nt - 1) / nt;
  const int g0 = min(p.n_total, tid * seg), g1 = min(p.n_total, g0 + seg);
  int cnt = 0;
  for (int g = g0; g < g1; ++g) cnt += ccount[g] >= 2;
  part_s[tid] = cnt;
  __syncthreads();
  for (int off = 1; off < nt; off <<= 1) {            // Hillis-Steele inclusive scan
    const int v = tid >= off ? part_s[tid - off] : 0;
    __syncthreads();
    part_s[tid] += v;
    __syncthreads();
  }
  int next = part_s[tid] - cnt;
  bool over = false;
  for (int g = g0; g < g1; ++g) {
    int zr = -1;
    if (ccount[g] >= 2) {
      if (next < zbuf_rows) zr = next; else over = true;
      ++next;
    }
    zrow[g] = zr;
  }
  if (over) report(p.ws, ETREE_ENOSPACE, DET_ZBUF);
}

// One warp per non-root node: the parent row's logit of the node's token,
// z = hidden[parent] . W[token], in fp32 (the acceptance test's p(x) needs it for every child,
// and siblings may share a row).  Invalid tokens get -inf and report ETREE_EDEVICE.
__global__ void __launch_bounds__(256) child_logit_kernel(AcceptParams p,
                                                          const __nv_bfloat16* w_lm, float* zc) {
  const int g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (g >= p.n_total) return;
  int base, n;
  float z = -INFINITY;
  if (row_owner(p, g, base, n) >= 0 && g > base) {
    const int pl = p.parent[g], x = p.tokens[g];
    if (pl >= 0 && pl < g - base && x >= 0 && x < p.V) {
      const uint4* h = reinterpret_cast<const uint4*>(p.hidden + (size_t)(base + pl) * p.H);
      const uint4* w = reinterpret_cast<const uint4*>(w_lm + (size_t)x * p.H);
      float acc = 0.f;
      for (int i = lane; i < p.H / 8; i += 32) {
        const uint4 a = h[i], b = __ldg(w + i);
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 fa = __bfloat1622float2(a2[k]), fb = __bfloat1622float2(b2[k]);
          acc = fmaf(fa.x, fb.x, acc);
          acc = fmaf(fa.y, fb.y, acc);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      z = acc;
    } else if (lane == 0 && (x < 0 || x >= p.V)) {
      report(p.ws, ETREE_EDEVICE, DET_BAD_TOKEN);
    }
  }
  if (lane == 0) zc[g] = z;
}

// One warp per node row: log2 sum 2^(z log2(e) / T) from the LM head's (max, sum) summaries.
__global__ void __launch_bounds__(256) row_lse_kernel(AcceptParams p) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.n_total) return;
  const float4* part = p.part + (size_t)row * p.n_tiles;
  float m = -INFINITY, s = 0.f;
  int t = lane;
  for (; t + 224 < p.n_tiles; t += 256) {            // eight loads in flight, merged in order
    float4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = part[t + 32 * u];
#pragma unroll
    for (int u = 0; u < 8; ++u) merge_lse(m, s, x[u].x, x[u].y);
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
}

// The part of N(c) = sum_v max(0, p_u(v) - c q_u(v)) over one materialised logit row that falls
// in slice `part` of `parts` (whole float4 groups when vocab is a multiple of 4), by the whole
// CTA: p_u(v) = 2^(z_v log2(e) / T - lse2_u) and the difference in fp32, summed in fp32 over 16
// terms, then in fp64 (each thread's partials, then the CTA's).
__device__ double residual_mass(const AcceptParams& p, const float* zr, const float* qr, float L2,
                                double c, double* red, int part, int parts) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const float cf = (float)c, kl = p.k_log2;
  double acc = 0.0;
  if ((p.V & 3) == 0) {
    const int all4 = p.V / 4, per = (all4 + parts - 1) / parts;
    const int o4 = min(all4, part * per);
    const float4* z4 = reinterpret_cast<const float4*>(zr) + o4;
    const float4* q4 = reinterpret_cast<const float4*>(qr) + o4;
    const int n4 = min(all4, o4 + per) - o4;
    int i = tid;
    for (; i + 3 * nt < n4; i += 4 * nt) {            // four float4 pairs in flight per thread
      float4 z[4], q[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        z[k] = z4[i + k * nt];
        q[k] = __ldg(q4 + i + k * nt);
      }
      float part = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        part += fmaxf(exp2f(z[k].x * kl - L2) - cf * q[k].x, 0.f);
        part += fmaxf(exp2f(z[k].y * kl - L2) - cf * q[k].y, 0.f);
        part += fmaxf(exp2f(z[k].z * kl - L2) - cf * q[k].z, 0.f);
        part += fmaxf(exp2f(z[k].w * kl - L2) - cf * q[k].w, 0.f);
      }
      acc += (double)part;
    }
    for (; i < n4; i += nt) {
      const float4 z = z4[i], q = __ldg(q4 + i);
      const float zz[4] = {z.x, z.y, z.z, z.w}, qq[4] = {q.x, q.y, q.z, q.w};
      float part = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) part += fmaxf(exp2f(zz[k] * kl - L2) - cf * qq[k], 0.f);
      acc += (double)part;
    }
  } else {
    const int per = (p.V + parts - 1) / parts;
    const int v1 = min(p.V, (part + 1) * per);
    for (int v = part * per + tid; v < v1; v += nt)
      acc += (double)fmaxf(exp2f(zr[v] * kl - L2) - cf * __ldg(qr + v), 0.f);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((tid & 31) == 0) red[tid >> 5] = acc;
  __syncthreads();
  double tot = 0.0;
  for (int w = 0; w < (nt >> 5); ++w) tot += red[w];
  __syncthreads();
  return tot;
}

// The multi-candidate walk, CS CTAs (a thread-block cluster) per request.  Thread 0 of every CTA
// takes the same decisions from the same data, so the CTAs move in step; each CTA evaluates its
// slice of N(c) when a rejected child has a younger sibling still to test.  It publishes the slice
// in its shared memory (a release store of the pass number), and every CTA adds the CS slices in
// rank order, so N(c) is the same in all of them.  Reading the other CTAs' slices polls a bounded
// number of times.  Rank 0 writes accept_len, path, the accepted tokens, the stop row / node, the
// draw offset cval (negative: the residual has no positive weight and the bonus is drawn from p)
// and the stop row's hidden state for the draw pass.  A child's logit under its parent's row comes
// from child_logit_kernel (zc), or, with zc null (every row materialised), from the parent's
// stored row.
__device__ __forceinline__ uint32_t walk_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void walk_cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t walk_mapa(const void* p, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(p)), "r"(rank));
  return ra;
}

constexpr uint32_t kWalkPollCap = 1u << 22;     // polls of a peer's pass number (a few seconds)

template <int CS, int NT>
__global__ void __cluster_dims__(CS, 1, 1) __launch_bounds__(NT)
    tree_walk_kernel(AcceptParams p, const float* zc, const int32_t* zrow, const float* zbuf) {
  __shared__ int par_s[64], tok_s[64];
  __shared__ double red_s[NT / 32];
  __shared__ int act_s, u_s, ok_s, fell_s, bad_s;
  __shared__ double c_s;
  __shared__ double slice_s[2], got_s[CS];     // this CTA's N(c) slice by pass parity; gathered
  __shared__ uint32_t pass_s;                  // passes published so far
  __shared__ int late_s;
  __shared__ float qx_s[64], zx_s[64], l2_s[64], uni_s[64];   // per child: its test's inputs
  const int r = blockIdx.x / CS, tid = threadIdx.x;
  const int rank = CS > 1 ? (int)walk_cluster_rank() : 0;
  const bool lead = rank == 0;
  int32_t* path = p.path + (size_t)r * ETREE_PATH_STRIDE;
  int32_t* outt = p.out_tokens + (size_t)r * ETREE_OUT_STRIDE;
  int base, n;
  const bool n_ok = request_ok(p, r, base, n);
  if (tid == 0) {
    ok_s = n_ok ? 1 : 0;
    bad_s = 0;                                          // malformed input (not a full buffer)
    pass_s = 0u;
    late_s = 0;
  }
  if (n_ok && tid < n) {
    par_s[tid] = p.parent[base + tid];
    tok_s[tid] = p.tokens[base + tid];
  }
  __syncthreads();
  if constexpr (CS > 1) walk_cluster_sync();           // every pass counter starts at 0
  if (n_ok && tid < n) {
    const int pj = par_s[tid];
    const bool good = tid == 0 ? pj == -1 : (pj >= 0 && pj < tid);
    bool fits = true;                                   // a branching node without a logit row
    int kids = 0;
    for (int j = tid + 1; j < n; ++j) kids += par_s[j] == tid;
    if (kids >= 2 && zrow[base + tid] < 0) fits = false;
    if (!good) {
      if (lead) report(p.ws, ETREE_EDEVICE, DET_BAD_PARENT);
      atomicAnd(&ok_s, 0);
      atomicOr(&bad_s, 1);
    }
    if (tid >= 1 && (tok_s[tid] < 0 || tok_s[tid] >= p.V)) {
      if (!zc && lead) report(p.ws, ETREE_EDEVICE, DET_BAD_TOKEN);   // else child_logit did
      atomicAnd(&ok_s, 0);
      atomicOr(&bad_s, 1);
    }
    if (!fits) atomicAnd(&ok_s, 0);                      // reported by tree_prep_kernel
  }
  __syncthreads();
  if (!ok_s) {
    // accept nothing.  A request without a logit row for a branching node (a full buffer) draws
    // its bonus from the root's p; a malformed one gets no bonus (stop node -1, which the draws
    // skip), so a caller that emits tokens before reading the status emits none.
    if (lead) {
      if (!n_ok && tid == 0) report(p.ws, ETREE_EDEVICE, DET_BAD_NODES);
      for (int k = tid; k < 64; k += NT) path[k] = (n_ok && k == 0) ? 0 : -1;
      for (int k = tid; k < 65; k += NT) outt[k] = -1;
      if (tid == 0) {
        p.accept_len[r] = 0;
        p.stop_row[r] = n_ok ? base : 0;
        p.stop_node[r] = (n_ok && !bad_s) ? 0 : -1;
        p.cval[r] = 0.f;
        p.rfloor[2 * r] = 0u;
        p.rfloor[2 * r + 1] = 0u;
      }
    }
    if (tid == 0) u_s = n_ok ? base : 0;
  } else {
    // Each child's test inputs do not depend on the walk's state: its parent row's log-sum-exp,
    // q and logit of its token, and its uniform.  They are read (and the uniform drawn) by one
    // thread per child up front, so thread 0's serial walk reads shared memory only.
    if (tid >= 1 && tid < n) {
      const int pu = par_s[tid], x = tok_s[tid];
      qx_s[tid] = __ldg(p.q_draft + (size_t)(base + pu) * p.V + x);
      zx_s[tid] = zc ? zc[base + tid] : zbuf[(size_t)zrow[base + pu] * p.V + x];
      l2_s[tid] = p.lse2[base + pu];
      float U[8];
      uniforms8(p.seed, p.step, 0u, (uint32_t)tid, (uint32_t)r, 1u, U);
      uni_s[tid] = U[0];
    }
    // thread 0's walk state: node u, last child tested, c and N(c) of the current residual
    int u = 0, j = 0, a = 0;
    double c = 0.0, N = 1.0;
    uint32_t npass = 0u;                                // residual passes so far (every thread)
    if (tid == 0) {
      if (lead) path[0] = 0;
      fell_s = 0;
    }
    for (int it = 0; it < 2 * 64 + 2; ++it) {          // each node is tested once: bounded
      __syncthreads();                                  // the previous round's values are read
      if (tid == 0) {
        int act = 2;                                    // 0: moved on, 1: need N(c), 2: stop
        for (j = j + 1; j < n && par_s[j] != u; ++j) {}
        if (j < n) {
          const int x = tok_s[j];
          const double qx = (double)qx_s[j];
          // the parent row's logit of x: from the materialised row itself when every row is
          // kept (the same fp32 accumulator the row's log-sum-exp came from), else child_logit's
          const double pz = (double)exp2f(zx_s[j] * p.k_log2 - l2_s[j]);
          const double rx = pz - c * qx > 0.0 ? (pz - c * qx) / N : 0.0;
          if ((double)uni_s[j] * qx < rx) {             // accepted: the walk moves to child j
            ++a;
            if (lead) {
              path[a] = j;
              outt[a - 1] = x;
            }
            u = j;
            c = 0.0;
            N = 1.0;
            act = 0;
          } else {                                      // rejected: r <- norm(max(0, r - q))
            c += N;
            int k = j + 1;
            while (k < n && par_s[k] != u) ++k;
            act = k < n ? 1 : 2;                        // N(c) only if a sibling remains
          }
        }
        act_s = act;
        u_s = u;
        c_s = c;
      }
      __syncthreads();
      const int act = act_s;
      if (act == 2) break;
      if (act == 1) {
        const int ur = base + u_s;
        const double mine = residual_mass(p, zbuf + (size_t)zrow[ur] * p.V,
                                          p.q_draft + (size_t)ur * p.V, p.lse2[ur], c_s, red_s,
                                          rank, CS);
        double Nn = mine;
        if constexpr (CS > 1) {
          const uint32_t k = npass++;                   // this pass, the same in every CTA
          if (tid == 0) {
            slice_s[k & 1] = mine;
            asm volatile("st.release.cluster.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(&pass_s)),
                         "r"(k + 1u)
                         : "memory");
          }
          if (tid < CS) {                               // thread q reads CTA q's slice
            const uint32_t ra = walk_mapa(&pass_s, (uint32_t)tid);
            uint32_t seen = 0u, tries = 0u;
            do {
              asm volatile("ld.acquire.cluster.shared::cluster.u32 %0, [%1];"
                           : "=r"(seen)
                           : "r"(ra)
                           : "memory");
              if (seen > k) break;
              __nanosleep(32);
            } while (++tries < kWalkPollCap);
            double v = __longlong_as_double(0x7ff8000000000000ll);   // NaN: gave up
            if (seen > k) {
              asm volatile("ld.shared::cluster.f64 %0, [%1];"
                           : "=d"(v)
                           : "r"(walk_mapa(&slice_s[k & 1], (uint32_t)tid))
                           : "memory");
            } else {
              atomicOr(&late_s, 1);
            }
            got_s[tid] = v;
          }
          __syncthreads();
          Nn = 0.0;
          for (int q = 0; q < CS; ++q) Nn += got_s[q];  // rank order: the same sum everywhere
        }
        if (tid == 0) {
          N = Nn;
          if (!(N > 0.0)) fell_s = 1;                   // no positive residual: draw from p
        }
        __syncthreads();
        if (fell_s) break;
      }
    }
    if (tid == 0 && late_s) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_WALK);
    if (tid == 0 && lead) {
      for (int k = a + 1; k < 64; ++k) path[k] = -1;
      for (int k = a; k < 65; ++k) outt[k] = -1;
      p.accept_len[r] = a;
      p.stop_row[r] = base + u;
      p.stop_node[r] = u;
      p.cval[r] = fell_s ? -1.f : (float)c;
      p.rfloor[2 * r] = 0u;
      p.rfloor[2 * r + 1] = 0u;
    }
    if (tid == 0) u_s = base + u;
  }
  __syncthreads();
  if (lead) {
    const uint4* hs = reinterpret_cast<const uint4*>(p.hidden + (size_t)u_s * p.H);
    uint4* hd = reinterpret_cast<uint4*>(p.hid2 + (size_t)r * p.H);
    for (int i = tid; i < p.H / 8; i += NT) hd[i] = hs[i];
  }
  if constexpr (CS > 1) walk_cluster_sync();           // no CTA leaves while its slice is read
}

// The bonus draw's last step, one warp per request: the largest race key over the draw pass's
// summaries (ties to the lower id), for the residual weights and for p.  The bonus is the
// residual's winner, or p's when the residual has no positive weight (or no rejection happened,
// in which case the draw weights are p and only p's race ran).
__global__ void __launch_bounds__(256) bonus_kernel(AcceptParams p) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= p.B) return;
  const float4* row = p.part2 + (size_t)r * p.n_tiles2;
  float kr = -INFINITY, kp = -INFINITY;
  int ir = -1, ip = -1;
  int t = lane;
  for (; t + 96 < p.n_tiles2; t += 128) {             // four loads in flight per lane
    float4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = row[t + 32 * u];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      merge_key(kr, ir, x[u].x, __float_as_int(x[u].y));
      merge_key(kp, ip, x[u].z, __float_as_int(x[u].w));
    }
  }
  for (; t < p.n_tiles2; t += 32) {
    const float4 x = row[t];
    merge_key(kr, ir, x.x, __float_as_int(x.y));
    merge_key(kp, ip, x.z, __float_as_int(x.w));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float okr = __shfl_xor_sync(0xffffffffu, kr, off);
    const int oir = __shfl_xor_sync(0xffffffffu, ir, off);
    const float okp = __shfl_xor_sync(0xffffffffu, kp, off);
    const int oip = __shfl_xor_sync(0xffffffffu, ip, off);
    merge_key(kr, ir, okr, oir);
    merge_key(kp, ip, okp, oip);
  }
  if (lane == 0) {
    const int base = p.cu_nodes[r];
    const int n = p.cu_nodes[r + 1] - base;
    if (n < 1 || n > p.n_max || p.stop_node[r] < 0) return;   // malformed: no bonus
    const int a = p.accept_len[r];
    p.out_tokens[(size_t)r * ETREE_OUT_STRIDE + a] = ir >= 0 ? ir : ip;
  }
}

// The bonus draw from materialised logits: the races of race.cuh over the stop row's stored
// logits and its draft row (the same fp32 logits the first GEMM pass produced, so the tokens
// equal those of a second pass over W).  A request's vocabulary is split into `parts` ranges of
// whole 8-id groups, one CTA each, so that small batches still fill the SMs.  Thread t of a CTA
// takes the groups t, t + blockDim, ... of its range; a CTA-wide floor in shared memory (keys of
// real ids) sharpens each thread's screen.  Leaders are merged by a total order (larger key, then
// lower id), so the result does not depend on the mapping: within the CTA by shuffles, across
// the parts by the CTA that arrives last (a per-request counter that the first GEMM pass zeroed)
// over the parts' summaries.
constexpr int kDrawThreads = 256;

__global__ void __launch_bounds__(kDrawThreads) draw_rows_kernel(AcceptParams p,
                                                                 const int32_t* zrow,
                                                                 const float* zbuf, int parts,
                                                                 float4* dpart, int32_t* dcnt) {
  __shared__ unsigned fl_s[2];                        // floors (fp32 bits of positive keys)
  __shared__ float kr_s[kDrawThreads / 32], kp_s[kDrawThreads / 32];
  __shared__ int ir_s[kDrawThreads / 32], ip_s[kDrawThreads / 32];
  const int r = blockIdx.x / parts, part = blockIdx.x % parts;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int base, n;
  if (!request_ok(p, r, base, n) || p.stop_node[r] < 0) return;   // answered by the walk
  if (tid == 0) fl_s[0] = fl_s[1] = 0u;
  __syncthreads();
  const int srow = p.stop_row[r];
  const int zr = zrow[srow];
  const float c = p.cval[r];
  const float L2 = p.lse2[srow];
  const float* z = zbuf + (size_t)(zr < 0 ? 0 : zr) * p.V;
  const float* q = p.q_draft + (size_t)srow * p.V;
  const uint32_t node = (uint32_t)p.stop_node[r];
  float kr = -INFINITY, kp = -INFINITY;
  int ir = -1, ip = -1;
  float thr_r = 0.f, thr_p = 0.f;
  const int groups = (p.V + 7) / 8;
  const int per = (groups + parts - 1) / parts;
  const int g1 = min(groups, (part + 1) * per);
  for (int g = part * per + tid; zr >= 0 && g < g1; g += kDrawThreads) {
    const int c0 = g * 8;
    float zz[8], qq[8];
    if ((p.V & 7) == 0) {
      const float4 a = *reinterpret_cast<const float4*>(z + c0);
      const float4 b = *reinterpret_cast<const float4*>(z + c0 + 4);
      zz[0] = a.x; zz[1] = a.y; zz[2] = a.z; zz[3] = a.w;
      zz[4] = b.x; zz[5] = b.y; zz[6] = b.z; zz[7] = b.w;
      if (c > 0.f) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(q + c0));
        const float4 y = __ldg(reinterpret_cast<const float4*>(q + c0 + 4));
        qq[0] = x.x; qq[1] = x.y; qq[2] = x.z; qq[3] = x.w;
        qq[4] = y.x; qq[5] = y.y; qq[6] = y.z; qq[7] = y.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        zz[e] = c0 + e < p.V ? z[c0 + e] : 0.f;
        qq[e] = (c > 0.f && c0 + e < p.V) ? __ldg(q + c0 + e) : 0.f;
      }
    }
    thr_r = fmaxf(thr_r, __uint_as_float(fl_s[0]) * kRaceShrink);
    thr_p = fmaxf(thr_p, __uint_as_float(fl_s[1]) * kRaceShrink);
    const float kr0 = kr, kp0 = kp;
    race8(zz, qq, c0, p.V, p.k_log2, L2, c, p.seed, p.step, node, (uint32_t)r, thr_r, thr_p, kr,
          ir, kp, ip);
    if (kr > kr0 && kr > 0.f) atomicMax(&fl_s[0], __float_as_uint(kr));
    if (kp > kp0 && kp > 0.f) atomicMax(&fl_s[1], __float_as_uint(kp));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float okr = __shfl_xor_sync(0xffffffffu, kr, off);
    const int oir = __shfl_xor_sync(0xffffffffu, ir, off);
    const float okp = __shfl_xor_sync(0xffffffffu, kp, off);
    const int oip = __shfl_xor_sync(0xffffffffu, ip, off);
    merge_key(kr, ir, okr, oir);
    merge_key(kp, ip, okp, oip);
  }
  if (lane == 0) {
    kr_s[warp] = kr;
    ir_s[warp] = ir;
    kp_s[warp] = kp;
    ip_s[warp] = ip;
  }
  __syncthreads();
  if (tid != 0) return;
  for (int w = 1; w < kDrawThreads / 32; ++w) {
    merge_key(kr, ir, kr_s[w], ir_s[w]);
    merge_key(kp, ip, kp_s[w], ip_s[w]);
  }
  if (parts > 1) {
    dpart[(size_t)r * parts + part] =
        make_float4(kr, __int_as_float(ir), kp, __int_as_float(ip));
    __threadfence();
    if (atomicAdd(dcnt + r, 1) != parts - 1) return;   // not the last part to finish
    __threadfence();
    for (int q2 = 0; q2 < parts; ++q2) {
      const float4 x = __ldcg(dpart + (size_t)r * parts + q2);
      merge_key(kr, ir, x.x, __float_as_int(x.y));
      merge_key(kp, ip, x.z, __float_as_int(x.w));
    }
  }
  const int a = p.accept_len[r];
  p.out_tokens[(size_t)r * ETREE_OUT_STRIDE + a] = ir >= 0 ? ir : ip;
}

// Parts per request: about 8 CTAs per SM in all, at most 32 per request, at least one 8-id group
// per thread of each part, and no more parts than summary slots (max_parts).
int draw_parts(int B, int V, int sms, int max_parts) {
  const int groups = (V + 7) / 8;
  int parts = (8 * sms + B - 1) / std::max(1, B);
  parts = std::min(parts, 32);
  parts = std::min(parts, std::max(1, groups / kDrawThreads));
  parts = std::min(parts, max_parts);
  return std::max(1, parts);
}

cudaError_t launch_draw_rows(const AcceptParams& p, const int32_t* zrow, const float* zbuf,
                             int parts, float4* dpart, int32_t* dcnt, cudaStream_t s) {
  draw_rows_kernel<<<p.B * parts, kDrawThreads, 0, s>>>(p, zrow, zbuf, parts, dpart, dcnt);
  return cudaGetLastError();
}

cudaError_t launch_accept_greedy(const AcceptParams& p, int32_t* arg_ws, int32_t* cnt,
                                 cudaStream_t s) {
  return launch_pdl(greedy_accept_kernel, dim3((p.n_total + p.B + 7) / 8), dim3(256), 0, s, p,
                    arg_ws, cnt);
}

cudaError_t launch_chain_prep(const AcceptParams& p, int32_t* child_tok, cudaStream_t s) {
  chain_prep_kernel<<<p.B, 64, 0, s>>>(p, child_tok);
  return cudaGetLastError();
}

cudaError_t launch_accept_chain(const AcceptParams& p, int32_t* cnt, cudaStream_t s) {
  chain_accept_kernel<<<(p.n_total + p.B + 7) / 8, 256, 0, s>>>(p, cnt);
  return cudaGetLastError();
}

cudaError_t launch_tree_prep(const AcceptParams& p, const __nv_bfloat16* w_lm, int32_t* ccount,
                             int32_t* zrow, int zbuf_rows, float* zc, cudaStream_t s) {
  tree_prep_kernel<<<1, 1024, 0, s>>>(p, ccount, zrow, zbuf_rows);
  if (zbuf_rows >= p.n_total) return cudaGetLastError();   // the walk reads the kept rows
  child_logit_kernel<<<(p.n_total + 7) / 8, 256, 0, s>>>(p, w_lm, zc);
  return cudaGetLastError();
}

cudaError_t launch_tree_walk(const AcceptParams& p, const float* zc, const int32_t* zrow,
                             const float* zbuf, int sms, cudaStream_t s) {
  row_lse_kernel<<<(p.n_total + 7) / 8, 256, 0, s>>>(p);
  // small batches: a cluster of 8 CTAs per request splits each residual pass; large batches
  // already fill the SMs with one CTA per request
  if (p.B * 8 <= 4 * sms)
    tree_walk_kernel<8, 256><<<p.B * 8, 256, 0, s>>>(p, zc, zrow, zbuf);
  else
    tree_walk_kernel<1, 1024><<<p.B, 1024, 0, s>>>(p, zc, zrow, zbuf);
  return cudaGetLastError();
}

cudaError_t launch_bonus(const AcceptParams& p, cudaStream_t s) {
  bonus_kernel<<<(p.B + 7) / 8, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace etree
