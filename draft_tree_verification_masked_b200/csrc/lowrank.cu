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
  // Every kernel here is launched with launch_pdl.  Only the floor kernel signals its dependent
  // early: the screen GEMM after it has set-up and U tiles to load before it waits.  An early
  // signal to a dependent with nothing to overlap measured slower than none.
  pdl_wait();
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

// g[m][j] = bf16(sum over chunks, in chunk order); also resets the screen's per-row bounds and
// the floor kernel's per-row counters.
__global__ void lr_reduce_kernel(const float* __restrict__ part, int nk, int M, int r,
                                 __nv_bfloat16* __restrict__ g, uint32_t* __restrict__ tkth,
                                 int32_t* __restrict__ fcnt) {
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < M) {
    tkth[t] = enc_order(-INFINITY);
    fcnt[t] = 0;
  }
  if (t >= M * r) return;
  float s = 0.f;
  for (int k = 0; k < nk; ++k) s += part[(size_t)k * M * r + t];
  g[t] = __float2bfloat16_rn(s);
}

// (va, ia) ranks before (vb, ib): larger value first, then the lower id; empty entries (id < 0)
// rank last.
__device__ __forceinline__ bool before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia >= 0 && (ib < 0 || ia < ib));
}

// A floor for the screen, kFloorParts CTAs per row.  Each sampled approximate logit is the sum
// of the split-K partials part[kc][m][j] in chunk order.  Thread t of every CTA of a row covers
// a fixed set of sampled columns; the maximum over its columns in all parts is one logit of the
// row, so the 16th largest of the 256 thread maxima is a value that 16 distinct logits reach, and
// no logit below it can be among the k <= 16 selected.  For a sample of 8192 it sits near the
// row's 99.8th percentile.  The CTA that completes a row (per-row counter, fence, atomic, fence)
// ranks the maxima.  The floor is lowered by a rounding margin that covers the sample's fp32 sums
// differing from the tensor-core sums of the same values.
constexpr int kFloorParts = 8;

__global__ void __launch_bounds__(256) sample_floor_kernel(const float* __restrict__ part,
                                                           int nk, int M, int S,
                                                           float* __restrict__ fmax,
                                                           int32_t* __restrict__ fcnt,
                                                           uint32_t* __restrict__ tkth) {
  __shared__ float mx[256];
  __shared__ int last_s;
  pdl_wait();
  pdl_trigger();
  const int m = blockIdx.x / kFloorParts, q = blockIdx.x % kFloorParts, tid = threadIdx.x;
  const int span = (S + kFloorParts - 1) / kFloorParts;
  const int c0 = q * span, c1 = min(S, c0 + span);
  const size_t cs = (size_t)M * S;                    // stride between chunk partials
  const float* row = part + (size_t)m * S;
  float best = -INFINITY;
  for (int j0 = c0 + tid; j0 < c1; j0 += 256 * 4) {
    float x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = 0.f;
    for (int kc = 0; kc < nk; ++kc) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (j0 + u * 256 < c1) x[u] += row[kc * cs + j0 + u * 256];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (j0 + u * 256 < c1) best = fmaxf(best, x[u]);
  }
  fmax[((size_t)m * kFloorParts + q) * 256 + tid] = best;
  __threadfence();
  __syncthreads();
  if (tid == 0) last_s = atomicAdd(fcnt + m, 1) == kFloorParts - 1;
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  best = -INFINITY;
  for (int q2 = 0; q2 < kFloorParts; ++q2)
    best = fmaxf(best, __ldcg(fmax + ((size_t)m * kFloorParts + q2) * 256 + tid));
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
// entries (8 loads in flight) and each warp appends its survivors (150-500 per row measured on
// the rank-128 and rank-512 workloads) to shared memory together.  A bitonic sort on the first
// 256 threads orders them and the first k go to cand[m][0..k).  (Counting ranks, a bisection for
// the k-th key over the CTA or one warp, and a register tournament in one warp all measured
// within -1 .. +5 us of it.)  More than kGather survivors fall back to ranking them in passes
// over the lists.
constexpr int kGather = 2048;
constexpr int kMergeThreads = 1024;
constexpr int kSortThreads = 256;

// Barrier 1 among the first kSortThreads threads of the CTA (barrier 0 is __syncthreads).
__device__ __forceinline__ void sort_barrier() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSortThreads) : "memory");
}

__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(const float2* __restrict__ lists,
                                                                   int nlists, const uint32_t* tkth,
                                                                   int k,
                                                                   int32_t* __restrict__ cand) {
  __shared__ float gv[kGather];
  __shared__ int gi[kGather];
  __shared__ int gn;
  pdl_wait();
  const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const float T = dec_order(tkth[m]);
  const float2* rowl = lists + (size_t)m * nlists * 16;
  const int total = nlists * 16;
  if (tid == 0) gn = 0;
  __syncthreads();
  // every lane of a warp runs the same iterations, so survivors are appended a warp at a time
  for (int eb = tid - lane; eb < total; eb += kMergeThreads * 8) {
    float2 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = eb + lane + u * kMergeThreads;
      x[u] = e < total ? rowl[e] : make_float2(-INFINITY, __int_as_float(-1));
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int xi = __float_as_int(x[u].y);
      const bool sv = xi >= 0 && x[u].x >= T;
      const unsigned b = __ballot_sync(0xffffffffu, sv);
      if (b) {
        int at = 0;
        if (lane == 0) at = atomicAdd(&gn, __popc(b));
        at = __shfl_sync(0xffffffffu, at, 0) + __popc(b & ((1u << lane) - 1u));
        if (sv && at < kGather) {
          gv[at] = x[u].x;
          gi[at] = xi;
        }
      }
    }
  }
  __syncthreads();
  const int n = gn;
  if (n <= kGather) {
    // The sort runs on the first kSortThreads threads only, synchronised by a named barrier of
    // that many threads (the rest of the CTA leaves); strides are powers of two, so the pair
    // indices are bit operations.
    if (tid >= kSortThreads) return;
    int P = 16;
    while (P < n) P <<= 1;
    for (int e = n + tid; e < P; e += kSortThreads) {
      gv[e] = -INFINITY;
      gi[e] = -1;
    }
    sort_barrier();
    for (int size = 2; size <= P; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < P / 2; i += kSortThreads) {
          const int lo = ((i & ~(stride - 1)) << 1) | (i & (stride - 1)), hi = lo + stride;
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
        sort_barrier();
      }
    }
    if (tid < k) cand[(size_t)m * 16 + tid] = gi[tid];
    return;
  }
  // fallback: every entry >= T is ranked against every other by a pass over the lists
  for (int e = tid; e < total; e += kMergeThreads) {
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

constexpr int kRescoreLoads = 20;        // 16-byte words of W per lane requested up front

// One CTA per row, one warp per candidate: z_c = h . W_c in fp32 (the row staged in shared
// memory, the lane's W words requested first); then the k candidates are ordered by z_c descending
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
  pdl_wait();
  const int m = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4* hrow = reinterpret_cast<const uint4*>(hid + (size_t)m * H);
  // this lane's first kRescoreLoads words of the candidate's W row (all of it at H <= 5120) are
  // requested before the hidden row is staged, so both loads are in flight together
  const int c = warp < k ? cand[(size_t)m * 16 + warp] : -1;
  const bool live = warp < k && c >= 0 && c < V;
  uint4 wv[kRescoreLoads];
  {
    const uint4* w = reinterpret_cast<const uint4*>(W + (size_t)(live ? c : 0) * H);
#pragma unroll
    for (int u = 0; u < kRescoreLoads; ++u) {
      const int i = lane + 32 * u;
      wv[u] = (live && i < H / 8) ? __ldg(w + i) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  for (int i = threadIdx.x; i < H / 8; i += blockDim.x) hsm[i] = hrow[i];
  __syncthreads();
  if (warp < k) {
    float acc = 0.f;
    if (live) {
#pragma unroll
      for (int u = 0; u < kRescoreLoads; ++u) {
        const int i = lane + 32 * u;
        if (i >= H / 8) break;
        const uint4 a = hsm[i], b = wv[u];
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 fa = __bfloat1622float2(a2[q]), fb = __bfloat1622float2(b2[q]);
          acc = fmaf(fa.x, fb.x, acc);
          acc = fmaf(fa.y, fb.y, acc);
        }
      }
      const uint4* w = reinterpret_cast<const uint4*>(W + (size_t)c * H);
      for (int i = lane + 32 * kRescoreLoads; i < H / 8; i += 32) {   // H > 5120
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
                                int32_t* fcnt, cudaStream_t s) {
  const int nk = lowrank_down_chunks(H);
  dim3 grid((r + kDT - 1) / kDT, nk, (M + kDT - 1) / kDT);
  cudaError_t e = launch_pdl(lr_down_kernel, grid, dim3(256), 0, s, hid, D, M, H, r, 1, part);
  if (e != cudaSuccess) return e;
  return launch_pdl(lr_reduce_kernel, dim3((M * r + 255) / 256), dim3(256), 0, s, part, nk, M, r,
                    g, tkth, fcnt);
}

int lowrank_sample_cols(int V) { return V < 8192 ? V : 8192; }

int lowrank_floor_maxima(int M) { return M * kFloorParts * 256; }

cudaError_t launch_lowrank_sample(const __nv_bfloat16* g, const __nv_bfloat16* U, int M, int r,
                                  int V, float* part, float* fmax, int32_t* fcnt, uint32_t* tkth,
                                  cudaStream_t s) {
  const int S = lowrank_sample_cols(V), stride = V / S;
  const int nk = (r + kDK - 1) / kDK;
  dim3 grid((S + kDT - 1) / kDT, nk, (M + kDT - 1) / kDT);
  cudaError_t e = launch_pdl(lr_down_kernel, grid, dim3(256), 0, s, g, U, M, r, S, stride, part);
  if (e != cudaSuccess) return e;
  return launch_pdl(sample_floor_kernel, dim3(M * kFloorParts), dim3(256), 0, s, part, nk, M, S,
                    fmax, fcnt, tkth);
}

cudaError_t launch_lowrank_finish(const float2* lists, int nlists, const uint32_t* tkth, int M,
                                  int k, int32_t* cand, const __nv_bfloat16* hid,
                                  const __nv_bfloat16* W, int H, int V, int32_t* out_ids,
                                  float* out_logit, cudaStream_t s) {
  cudaError_t e = launch_pdl(topk_merge_kernel, dim3(M), dim3(kMergeThreads), 0, s, lists,
                             nlists, tkth, k, cand);
  if (e != cudaSuccess) return e;
  return launch_pdl(lr_rescore_kernel, dim3(M), dim3(32 * k), 0, s, hid, W, H, V, k, cand,
                    out_ids, out_logit);
}

}  // namespace etree
