// attn_combine.cu -- the two small kernels around the tree attention (sm_100a): the
// log-sum-exp merge of KV-split partials and the longest-first dispatch order of requests.
//
// Tree attention splits a request's keys over several CTAs when there are too few (request, KV
// head, row block) work items to fill the SMs; each split leaves an unnormalised output with its
// running maximum and sum, and the merge below combines them exactly (every tree node attends
// to its request's cached keys and to its ancestors: "Eagle-4 Released: Outpaces DFlash2 and
// DSpark ...", section "Technical Background").
#include "kernels.cuh"

namespace etree {

// Merge the split partials of each (node, head) row by log-sum-exp: one warp per row, each lane
// owning 4 of the 128 output dims.  The row's split maxima and sums are loaded together with its
// request's header (lane s holds split s), so the partials are read in two dependent rounds:
// the (m, l) pairs, then every used split's 512-byte output slice, BATCH splits in flight (8 when
// there are at most 8 splits, which keeps the kernel's registers and its occupancy high).
template <int BATCH>
__global__ void attn_combine_kernel(AttnParams p, int n_total) {
  pdl_wait();                                      // the split partials of the attention kernel
  pdl_trigger();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= n_total * p.hq) return;
  const float2* mlp = p.ml_part + (size_t)gw * p.nsplit;
  const float4* op = reinterpret_cast<const float4*>(p.o_part + (size_t)gw * p.nsplit * 128);
  float2 ml = lane < p.nsplit ? mlp[lane] : make_float2(-INFINITY, 0.f);
  const int node = gw / p.hq;
  int lo = 0, hi = p.B - 1;                        // request of this node
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.cu_nodes[mid] <= node) lo = mid; else hi = mid - 1;
  }
  const int L = p.kv_len[lo];
  const int n = p.cu_nodes[lo + 1] - p.cu_nodes[lo];
  if (n < 1 || n > p.n_max || L < 0 || L > p.kv_len_max) return;   // reported by the main kernel
  const int total = (L + p.keys - 1) / p.keys + (n + p.keys - 1) / p.keys;
  const int used = min(p.nsplit, (total + p.tps - 1) / p.tps);     // splits that ran (the rest
                                                                   // hold stale values)
  // the maximum over the used splits, 32 at a time across the lanes
  float M = -INFINITY;
  for (int s0 = 0; s0 < used; s0 += 32) {
    const float2 x = s0 == 0 ? ml : (s0 + lane < used ? mlp[s0 + lane] : ml);
    if (s0 + lane < used) M = fmaxf(M, x.x);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float Mb = (M == -INFINITY) ? 0.f : M;
  // the weighted sums in split order; the weights come from the lane that holds the split
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  for (int s0 = 0; s0 < used; s0 += 32) {
    const float2 x = s0 == 0 ? ml : (s0 + lane < used ? mlp[s0 + lane] : make_float2(-INFINITY, 0.f));
    const float wl = s0 + lane < used ? exp2f(x.x - Mb) : 0.f;   // split s0 + lane's weight
    const float ll = wl * x.y;
    const int cnt = min(32, used - s0);
    for (int b0 = 0; b0 < cnt; b0 += BATCH) {
      float4 v[BATCH];
#pragma unroll
      for (int i = 0; i < BATCH; ++i)
        v[i] = b0 + i < cnt ? op[(size_t)(s0 + b0 + i) * 32 + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {
        const float w = __shfl_sync(0xffffffffu, wl, (b0 + i) & 31);
        const float lw = __shfl_sync(0xffffffffu, ll, (b0 + i) & 31);
        if (b0 + i < cnt) {
          lsum += lw;
          acc.x += v[i].x * w;
          acc.y += v[i].y * w;
          acc.z += v[i].z * w;
          acc.w += v[i].w * w;
        }
      }
    }
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  uint2 packed;
  packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(p.out + (size_t)gw * 128)[lane] = packed;
  if (p.lse && lane == 0) p.lse[gw] = (M + log2f(lsum)) * 0.69314718055994531f;
}

// Longest-first dispatch order: request r's rank is the number of requests with a longer KV
// cache (ties by index), so order[rank] lists requests by decreasing length.  CTAs are
// dispatched roughly in block order, and starting the long work first shortens the tail of a
// batch with mixed lengths.
__global__ void attn_order_kernel(const int32_t* kv_len, int B, int32_t* order) {
  extern __shared__ int32_t len_s[];
  for (int i = threadIdx.x; i < B; i += blockDim.x) len_s[i] = kv_len[i];
  __syncthreads();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= B) return;
  const int L = len_s[r];
  int rank = 0;
  for (int i = 0; i < B; ++i) {
    const int Li = len_s[i];
    rank += (Li > L) || (Li == L && i < r);
  }
  order[rank] = r;
}

cudaError_t launch_attn_order(const int32_t* kv_len, int B, int32_t* order, cudaStream_t stream) {
  attn_order_kernel<<<(B + 255) / 256, 256, B * sizeof(int32_t), stream>>>(kv_len, B, order);
  return cudaGetLastError();
}

cudaError_t launch_attn_combine(const AttnParams& p, int n_total, cudaStream_t stream) {
  const int rows = n_total * p.hq;
  const int threads = 256;
  const int blocks = (rows * 32 + threads - 1) / threads;
  if (p.nsplit <= 8)
    return launch_pdl(attn_combine_kernel<8>, dim3(blocks), dim3(threads), 0, stream, p, n_total);
  return launch_pdl(attn_combine_kernel<16>, dim3(blocks), dim3(threads), 0, stream, p, n_total);
}

}  // namespace etree
