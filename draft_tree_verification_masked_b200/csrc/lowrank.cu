// lowrank.cu -- the low-rank candidate head (sm_100a).
//
// EAGLE-4's draft replaces its vocabulary projection by a low-rank candidate head: a small
// factorised product screens the vocabulary for candidate tokens, and only those few are scored
// exactly; the pages credit it with cutting a draft forward from 574 us (65.4% in the vocab
// head) to 326 us at rank 512 and 255 us at rank 128 ("EAGLE-4 是什麼？...", aiposthub.com,
// section "EAGLE-4 是什麼？先看推測解碼為什麼能變快", Fig. 2).  For M hidden rows h:
//
//   g  = h D^T        D [r][H]: split-K over H on the CUDA cores (lr_down_kernel), the
//                     partials summed in a fixed order and rounded to bf16 (lr_reduce_kernel);
//   z~ = g U^T        U [V][r]: the LM-head GEMM on tcgen05 with the EPI_TOPK epilogue, which
//                     keeps each thread's 16 largest (value, id) per row -- z~ never reaches HBM;
//   C  = top-k of z~  topk_merge_kernel: one CTA per row merges the sorted 16-lists;
//   z_c = h . W_c     lr_rescore_kernel: one warp per candidate, then the k are ordered by z_c.
//
// The screen streams |U| = V r 2 bytes (155 MB at r = 512, 39 MB at r = 128) instead of the full
// head's |W| = V H 2 (1.56 GB at H = 5120), plus k rows of W per hidden row.
#include "kernels.cuh"

namespace etree {

namespace {
constexpr int kDT = 64;        // rows (m) and columns (j) per CTA tile
constexpr int kDK = 128;       // H per CTA (the split-K chunk)
constexpr int kDPad = 8;       // bf16 padding per smem row (breaks the 512-byte bank stride)
}  // namespace

// part[kc][m][j] = sum_{h in chunk kc} A[m][h] B[j * bstride][h], fp32 (A [M][K], B rows of K;
// j < N).  The down projection has A = hidden, B = D; the screen's sample has A = g and B = every
// bstride-th row of U.  CTA tile 64 m x 64 j x 128 h staged in padded shared memory (row
// stride 272 bytes: the 8 rows an ldmatrix reads fall in distinct banks).
__global__ void __launch_bounds__(256) lr_down_kernel(const __nv_bfloat16* __restrict__ hid,
                                                      const __nv_bfloat16* __restrict__ D, int M,
                                                      int H, int r, int bstride,
                                                      float* __restrict__ part) {
  __shared__ __align__(16) __nv_bfloat16 hs[kDT][kDK + kDPad];
  __shared__ __align__(16) __nv_bfloat16 ds[kDT][kDK + kDPad];
  const int j0 = blockIdx.x * kDT, kc = blockIdx.y, m0 = blockIdx.z * kDT;
  const int h0 = kc * kDK;
  const int tid = threadIdx.x;
  // stage the two tiles, 16 bytes per thread per step (zeros past M, r or H)
  for (int e = tid; e < kDT * (kDK / 8); e += 256) {
    const int row = e / (kDK / 8), c8 = (e % (kDK / 8)) * 8;
    uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
    if (m0 + row < M && h0 + c8 < H)
      a = *reinterpret_cast<const uint4*>(hid + (size_t)(m0 + row) * H + h0 + c8);
    if (j0 + row < r && h0 + c8 < H)
      b = __ldg(reinterpret_cast<const uint4*>(D + (size_t)(j0 + row) * bstride * H + h0 + c8));
    *reinterpret_cast<uint4*>(&hs[row][c8]) = a;
    *reinterpret_cast<uint4*>(&ds[row][c8]) = b;
  }
  __syncthreads();
  // 8 warps: warp (wm, wn) computes rows wm*16 .. +15 and columns wn*32 .. +31 with
  // mma.m16n8k16 (bf16 in, fp32 accumulate), fragments loaded by ldmatrix
  const int warp = tid >> 5, lane = tid & 31;
  const int wm = warp & 3, wn = warp >> 2;
  float acc[4][4] = {};
#pragma unroll
  for (int kk = 0; kk < kDK / 16; ++kk) {
    uint32_t a[4];
    ldmatrix_x4(smem_u32(&hs[wm * 16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]), a[0], a[1],
                a[2], a[3]);
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(smem_u32(&ds[wn * 32 + np * 16 + (lane & 7) + ((lane >> 4) << 3)]
                              [kk * 16 + ((lane >> 3) & 1) * 8]),
                  b0, b1, b2, b3);
      mma_bf16_16816(acc[2 * np], a, b0, b1);
      mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
    }
  }
#pragma unroll
  for (int t = 0; t < 4; ++t) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int m = m0 + wm * 16 + (lane >> 2) + 8 * hf;
      const int j = j0 + wn * 32 + t * 8 + (lane & 3) * 2;
      if (m < M) {
        if (j < r) part[((size_t)kc * M + m) * r + j] = acc[t][2 * hf];
        if (j + 1 < r) part[((size_t)kc * M + m) * r + j + 1] = acc[t][2 * hf + 1];
      }
    }
  }
}

// g[m][j] = bf16(sum over chunks, in chunk order); also resets the screen's per-row bounds.
__global__ void lr_reduce_kernel(const float* __restrict__ part, int nk, int M, int r,
                                 __nv_bfloat16* __restrict__ g, uint32_t* __restrict__ tkth) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < M) tkth[t] = enc_order(-INFINITY);
  if (t >= M * r) return;
  float s = 0.f;
  for (int k = 0; k < nk; ++k) s += part[(size_t)k * M * r + t];
  g[t] = __float2bfloat16_rn(s);
}

// zs[m][j] = sum over the chunk partials (in chunk order) of the sampled approximate logits.
__global__ void sample_sum_kernel(const float* __restrict__ part, int nk, int MS,
                                  float* __restrict__ zs) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= MS) return;
  float x = 0.f;
  for (int k = 0; k < nk; ++k) x += part[(size_t)k * MS + t];
  zs[t] = x;
}

// (va, ia) ranks before (vb, ib): larger value first, then the lower id; empty entries (id < 0)
// rank last.
__device__ __forceinline__ bool before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia >= 0 && (ib < 0 || ia < ib));
}

// One CTA per row: a floor for the screen.  Each thread takes the maximum of its sampled
// approximate logits; the 16th largest of these 256 maxima is a value that 16 distinct logits
// reach (each maximum is one), so no logit below it can be among the k <= 16 selected.  For a
// sample of 8192 it sits near the row's 99.8th percentile.  It is lowered by a rounding margin
// that covers the sample's fp32 sums differing from the tensor-core sums of the same values.
__global__ void __launch_bounds__(256) sample_floor_kernel(const float* __restrict__ zs, int S,
                                                           uint32_t* __restrict__ tkth) {
  __shared__ float mx[256];
  const int m = blockIdx.x, tid = threadIdx.x;
  const float* row = zs + (size_t)m * S;
  float best = -INFINITY;
  for (int j0 = tid; j0 < S; j0 += 256 * 8) {
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = j0 + u * 256 < S ? row[j0 + u * 256] : -INFINITY;
#pragma unroll
    for (int u = 0; u < 8; ++u) best = fmaxf(best, x[u]);
  }
  mx[tid] = best;
  __syncthreads();
  int rank = 0;                                       // maxima ranked before this thread's
  for (int j = 0; j < 256; ++j) rank += mx[j] > best || (mx[j] == best && j < tid);
  if (rank == 15) {                                   // exactly one thread (ranks are distinct)
    const float floor = best == -INFINITY ? -INFINITY : best - 1e-3f * (1.f + fabsf(best));
    tkth[m] = enc_order(floor);
  }
}

// One CTA per row.  The screen published a lower bound T of the row's 16th largest value, so
// only list entries >= T can be selected: each thread scans its share of the 16 x nlists
// entries (8 loads in flight) and appends the survivors (usually a few hundred) to shared
// memory, where a bitonic sort orders them and the first k go to cand[m][0..k).  More than
// kGather survivors (not seen in practice) fall back to ranking them in passes over the lists.
constexpr int kGather = 2048;

__global__ void __launch_bounds__(256) topk_merge_kernel(const float2* __restrict__ lists,
                                                         int nlists, const uint32_t* tkth, int k,
                                                         int32_t* __restrict__ cand) {
  __shared__ float gv[kGather];
  __shared__ int gi[kGather];
  __shared__ int gn;
  const int m = blockIdx.x, tid = threadIdx.x;
  const float T = dec_order(tkth[m]);
  const float2* rowl = lists + (size_t)m * nlists * 16;
  const int total = nlists * 16;
  if (tid == 0) gn = 0;
  __syncthreads();
  for (int e0 = tid; e0 < total; e0 += 256 * 8) {
    float2 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      x[u] = e0 + u * 256 < total ? rowl[e0 + u * 256] : make_float2(-INFINITY, __int_as_float(-1));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int xi = __float_as_int(x[u].y);
      if (xi >= 0 && x[u].x >= T) {
        const int at = atomicAdd(&gn, 1);
        if (at < kGather) {
          gv[at] = x[u].x;
          gi[at] = xi;
        }
      }
    }
  }
  __syncthreads();
  const int n = gn;
  if (n <= kGather) {
    // bitonic sort of the survivors (padded with empty entries to a power of two), best first
    int P = 16;
    while (P < n) P <<= 1;
    for (int e = n + tid; e < P; e += 256) {
      gv[e] = -INFINITY;
      gi[e] = -1;
    }
    __syncthreads();
    for (int size = 2; size <= P; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < P / 2; i += 256) {
          const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
          const bool best_first = (lo & size) == 0;
          const bool swap = best_first ? before(gv[hi], gi[hi], gv[lo], gi[lo])
                                       : before(gv[lo], gi[lo], gv[hi], gi[hi]);
          if (swap) {
            const float tv = gv[lo];
            const int ti = gi[lo];
            gv[lo] = gv[hi];
            gi[lo] = gi[hi];
            gv[hi] = tv;
            gi[hi] = ti;
          }
        }
        __syncthreads();
      }
    }
    if (tid < k) cand[(size_t)m * 16 + tid] = gi[tid];
    return;
  }
  // fallback: every entry >= T is ranked against every other by a pass over the lists
  for (int e = tid; e < total; e += 256) {
    const float2 x = rowl[e];
    const int xi = __float_as_int(x.y);
    if (xi < 0 || x.x < T) continue;
    int rank = 0;
    for (int f = 0; f < total && rank < k; ++f) {
      const float2 y = rowl[f];
      rank += before(y.x, __float_as_int(y.y), x.x, xi);
    }
    if (rank < k) cand[(size_t)m * 16 + rank] = xi;
  }
}

// One CTA per row, one warp per candidate: z_c = h . W_c in fp32 (the row staged in shared
// memory, ten W loads in flight per lane); then the k candidates are ordered by z_c descending
// (lower id first on equal values).
__global__ void __launch_bounds__(512) lr_rescore_kernel(const __nv_bfloat16* __restrict__ hid,
                                                         const __nv_bfloat16* __restrict__ W,
                                                         int H, int V, int k,
                                                         const int32_t* __restrict__ cand,
                                                         int32_t* __restrict__ out_ids,
                                                         float* __restrict__ out_logit) {
  __shared__ uint4 hsm[1024];                     // H <= 8192
  __shared__ float zs[16];
  __shared__ int cs[16];
  const int m = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4* hrow = reinterpret_cast<const uint4*>(hid + (size_t)m * H);
  for (int i = threadIdx.x; i < H / 8; i += blockDim.x) hsm[i] = hrow[i];
  __syncthreads();
  if (warp < k) {
    const int c = cand[(size_t)m * 16 + warp];
    float acc = 0.f;
    if (c >= 0 && c < V) {
      const uint4* w = reinterpret_cast<const uint4*>(W + (size_t)c * H);
#pragma unroll 10
      for (int i = lane; i < H / 8; i += 32) {
        const uint4 a = hsm[i], b = __ldg(w + i);
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 fa = __bfloat1622float2(a2[q]), fb = __bfloat1622float2(b2[q]);
          acc = fmaf(fa.x, fb.x, acc);
          acc = fmaf(fa.y, fb.y, acc);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    } else {
      acc = -INFINITY;
    }
    if (lane == 0) {
      zs[warp] = acc;
      cs[warp] = c;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < k; ++i) {                    // insertion sort of <= 16
      const float x = zs[i];
      const int ci = cs[i];
      int j = i - 1;
      while (j >= 0 && (zs[j] < x || (zs[j] == x && cs[j] > ci))) {
        zs[j + 1] = zs[j];
        cs[j + 1] = cs[j];
        --j;
      }
      zs[j + 1] = x;
      cs[j + 1] = ci;
    }
    for (int i = 0; i < k; ++i) {
      out_ids[(size_t)m * k + i] = cs[i];
      out_logit[(size_t)m * k + i] = zs[i];
    }
  }
}

int lowrank_down_chunks(int H) { return (H + kDK - 1) / kDK; }

cudaError_t launch_lowrank_down(const __nv_bfloat16* hid, const __nv_bfloat16* D, int M, int H,
                                int r, float* part, __nv_bfloat16* g, uint32_t* tkth,
                                cudaStream_t s) {
  const int nk = lowrank_down_chunks(H);
  dim3 grid((r + kDT - 1) / kDT, nk, (M + kDT - 1) / kDT);
  lr_down_kernel<<<grid, 256, 0, s>>>(hid, D, M, H, r, 1, part);
  lr_reduce_kernel<<<(M * r + 255) / 256, 256, 0, s>>>(part, nk, M, r, g, tkth);
  return cudaGetLastError();
}

int lowrank_sample_cols(int V) { return V < 8192 ? V : 8192; }

cudaError_t launch_lowrank_sample(const __nv_bfloat16* g, const __nv_bfloat16* U, int M, int r,
                                  int V, float* part, uint32_t* tkth, cudaStream_t s) {
  const int S = lowrank_sample_cols(V), stride = V / S;
  const int nk = (r + kDK - 1) / kDK;
  dim3 grid((S + kDT - 1) / kDT, nk, (M + kDT - 1) / kDT);
  lr_down_kernel<<<grid, 256, 0, s>>>(g, U, M, r, S, stride, part);
  float* zs = part + (size_t)nk * M * S;
  sample_sum_kernel<<<(M * S + 255) / 256, 256, 0, s>>>(part, nk, M * S, zs);
  sample_floor_kernel<<<M, 256, 0, s>>>(zs, S, tkth);
  return cudaGetLastError();
}

cudaError_t launch_lowrank_finish(const float2* lists, int nlists, const uint32_t* tkth, int M,
                                  int k, int32_t* cand, const __nv_bfloat16* hid,
                                  const __nv_bfloat16* W, int H, int V, int32_t* out_ids,
                                  float* out_logit, cudaStream_t s) {
  topk_merge_kernel<<<M, 256, 0, s>>>(lists, nlists, tkth, k, cand);
  lr_rescore_kernel<<<M, 32 * k, 0, s>>>(hid, W, H, V, k, cand, out_ids, out_logit);
  return cudaGetLastError();
}

}  // namespace etree
