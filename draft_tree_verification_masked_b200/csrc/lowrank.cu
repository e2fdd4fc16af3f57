// lowrank.cu -- the low-rank candidate head (sm_100a).
//
// EAGLE-4's draft replaces its vocabulary projection by a low-rank candidate head: a small
// factorised product screens the vocabulary for candidate tokens, and only those few are scored
// exactly; the pages credit it with cutting a draft forward from 574 us (65.4% in the vocab
// head) to 326 us at rank 512 and 255 us at rank 128 ("EAGLE-4 是什麼？...", aiposthub.com,
// section "EAGLE-4 是什麼？先看推測解碼為什麼能變快", Fig. 2).  For M hidden rows h:
//
//   g  = h D^T        D [r][H]: lr_splitk_kernel, tcgen05 tiles of 64 x 64 with K split in
//                     chunks of 128 over many CTAs; lr_reduce_kernel sums the chunk partials in
//                     chunk order (the same order every call) and rounds g to bf16;
//   floor             the same split-K kernel on every stride-th row of U (8192 samples per
//                     row), and sample_floor_kernel: a lower bound of each row's 16th largest z~;
//   z~ = g U^T        U [V][r]: the LM-head GEMM on tcgen05 with the EPI_TOPK epilogue, which
//                     keeps each thread's 16 largest (value, id) per row above the floor -- z~
//                     never reaches HBM;
//   C  = top-k of z~  topk_select_kernel: one CTA per row finds the k-th largest list entry by
//                     a radix select over all the lists and keeps the entries ranked above it;
//   z_c = h . W_c     in the same CTA: one warp per candidate, then the k are ordered by z_c.
//
// The screen streams |U| = V r 2 bytes (155 MB at r = 512, 39 MB at r = 128) instead of the full
// head's |W| = V H 2 (1.56 GB at H = 5120), plus k rows of W per hidden row.
#include "kernels.cuh"

namespace etree {


// part[kc][m][j] = sum over k in chunk kc of A[m][k] B[j][k], fp32, for m < M and j < N; chunk
// kc covers k in [128 kc, 128 kc + 128) of K (a multiple of 64).  The down projection has A =
// hidden, B = D; the screen's sample has A = g and B = every stride-th row of U (a tensor map
// whose rows step over the others).  One CTA = 64 m x 64 j x 128 k, many CTAs in flight: thread 0
// issues the chunk's (at most) two K steps of 128-byte-swizzled boxes {64 k, 64 rows} of A and B
// on one barrier, thread 32 issues tcgen05.mma M=64 N=64 K=16 into 64 TMEM columns, and the four
// warps store their accumulator rows (lanes 0..15 of each TMEM lane quarter) as fp32.
constexpr int kSkTile = 64;     // m and j per CTA
constexpr int kSkChunk = 128;   // k per CTA

__global__ void __launch_bounds__(128) lr_splitk_kernel(const __grid_constant__ CUtensorMap tm_a,
                                                        const __grid_constant__ CUtensorMap tm_b,
                                                        int M, int K, int N,
                                                        float* __restrict__ part, WsHeader* ws) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));   // [step][A 8 KB, B 8 KB]
  __shared__ uint64_t full, done;
  __shared__ uint32_t tmem_s;
  const int j0 = blockIdx.x * kSkTile, kc = blockIdx.y, m0 = blockIdx.z * kSkTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int steps = min(kSkChunk / 64, K / 64 - kc * (kSkChunk / 64));
  if (threadIdx.x == 0) {
    mbar_init(&full, 1);
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_s, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  pdl_wait();                                           // A (hidden or g) of an earlier kernel
  bool ok = true;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    mbar_arrive_expect_tx(&full, steps * 16384);
    for (int s = 0; s < steps; ++s) {
      const int k = (kc * (kSkChunk / 64) + s) * 64;
      tma_load_2d(tiles + s * 16384, &tm_a, &full, k, m0);
      tma_load_2d(tiles + s * 16384 + 8192, &tm_b, &full, k, j0);
    }
  } else if (threadIdx.x == 32) {
    ok = mbar_wait(&full, 0);
    tc_fence_after();
    if (ok) {
      const uint32_t idesc = idesc_bf16_f32(kSkTile, kSkTile);
      for (int s = 0; s < steps; ++s) {
        const uint64_t da = smem_desc_sw128(tiles + s * 16384);
        const uint64_t db = smem_desc_sw128(tiles + s * 16384 + 8192);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, (s > 0 || kk > 0) ? 1u : 0u);
      }
    }
    tc_commit(&done);
  }
  __syncwarp();
  const bool got = mbar_wait(&done, 0);
  __syncwarp();
  tc_fence_after();
  float v0[32], v1[32];
  tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), v0);
  tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32, v1);
  const int m = m0 + 16 * warp + lane;
  if (ok && got && lane < 16 && m < M) {
    float* dst = part + ((size_t)kc * M + m) * N + j0;
    if (j0 + kSkTile <= N && (N & 3) == 0) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(dst)[q] = make_float4(v0[4 * q], v0[4 * q + 1], v0[4 * q + 2],
                                                        v0[4 * q + 3]);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(dst + 32)[q] = make_float4(v1[4 * q], v1[4 * q + 1],
                                                             v1[4 * q + 2], v1[4 * q + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j0 + j < N) dst[j] = v0[j];
        if (j0 + 32 + j < N) dst[32 + j] = v1[j];
      }
    }
  }
  if (threadIdx.x == 0) {                               // the boxes have landed before exit
    if (!mbar_wait(&full, 0)) ok = false;
  }
  if (!ok || !got) report(ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
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

// (va, ia) ranks before (vb, ib): larger value first, then the lower id.
__device__ __forceinline__ bool before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// The top k of a row from its screen lists.  Each vocab id appears in at most one list, and
// every list holds its thread's 16 largest values, so the row's k <= 16 largest values are
// among the list entries: the k-th largest entry, with equal values ranked by the lower id,
// splits them exactly.  One CTA per row finds it by a radix select on order-preserving 32-bit
// codes of the values (-0 counted as +0, empty entries excluded): each pass histograms the next
// 8 bits of the entries that match the digits fixed so far, and one warp finds the digit that
// holds the k-th largest.  The select stops early when every entry of that digit is needed.
// Entries above the final prefix are taken, then those on it (all of them, or the lowest ids
// when the k-th value is shared), and one warp orders the k by (value desc, id asc).
constexpr int kSelThreads = 1024;
constexpr int kSelRegs = 8;              // entries per thread kept in registers (8192 per row)

__device__ __forceinline__ uint32_t sel_code(float2 x) {
  if (__float_as_int(x.y) < 0) return 0u;            // empty entry
  return enc_order(x.x == 0.f ? 0.f : x.x);          // >= 0x007fffff for every non-NaN value
}

__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(
    const float2* __restrict__ lists, int nlists, int k, int32_t* __restrict__ cand,
    const __nv_bfloat16* __restrict__ hid,
    const __nv_bfloat16* __restrict__ W, int H, int V, int32_t* __restrict__ out_ids,
    float* __restrict__ out_logit) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_digit, s_above, s_count, s_n;
  __shared__ int s_min[kSelThreads / 32];
  __shared__ float sv[16], zs[16];
  __shared__ int si[16], cs[16];
  __shared__ uint4 hsm[1024];                          // the hidden row (H <= 8192)
  pdl_wait();
  const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  {                                                    // staged for the rescoring at the end
    const uint4* hrow = reinterpret_cast<const uint4*>(hid + (size_t)m * H);
    for (int i = tid; i < H / 8; i += kSelThreads) hsm[i] = hrow[i];
  }
  const float2* rowl = lists + (size_t)m * nlists * 16;
  const int total = nlists * 16;
  const int in_regs = kSelRegs * kSelThreads;
  uint32_t code[kSelRegs];
#pragma unroll
  for (int u = 0; u < kSelRegs; ++u) {
    const int e = tid + u * kSelThreads;
    code[u] = e < total ? sel_code(__ldg(rowl + e)) : 0u;
  }
  uint32_t prefix = 0u, pmask = 0u;
  uint32_t krem = (uint32_t)k;            // entries still to take among those on the prefix
  bool whole = false;                     // every entry on the prefix is taken
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kSelRegs; ++u)
      if (code[u] && (code[u] & pmask) == prefix) atomicAdd(&hist[(code[u] >> shift) & 255u], 1u);
    for (int e = in_regs + tid; e < total; e += kSelThreads) {
      const uint32_t cc = sel_code(__ldg(rowl + e));
      if (cc && (cc & pmask) == prefix) atomicAdd(&hist[(cc >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255 - 8l down to 248 - 8l; counts are scanned from the top digit
      uint32_t cnt[8], sum = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - 8 * lane - i];
        sum += cnt[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const uint32_t excl = incl - sum;
      if (excl < krem && krem <= incl) {
        uint32_t run = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (run + cnt[i] >= krem) {
            s_digit = 255u - 8u * lane - i;
            s_above = run;
            s_count = cnt[i];
            break;
          }
          run += cnt[i];
        }
      }
      if (lane == 31 && incl < krem) {                  // fewer than k entries in the lists
        s_digit = 256u;
        s_above = incl;
        s_count = 0u;
      }
    }
    __syncthreads();
    const uint32_t d = s_digit;
    if (d > 255u) {                                     // take every entry (first pass only)
      whole = true;
      break;
    }
    prefix |= d << shift;
    pmask |= 255u << shift;
    krem -= s_above;
    if (s_count == krem) {
      whole = true;
      break;
    }
  }
  if (tid == 0) s_n = 0u;
  __syncthreads();
  // entries above the prefix (fewer than k), and all entries on it when `whole`
  auto take = [&](uint32_t cc, int e) {
    const uint32_t cm = cc & pmask;
    if (cc && (cm > prefix || (whole && cm == prefix))) {
      const uint32_t at = atomicAdd(&s_n, 1u);
      const float2 x = __ldg(rowl + e);
      if (at < 16u) {
        sv[at] = x.x;
        si[at] = __float_as_int(x.y);
      }
    }
  };
#pragma unroll
  for (int u = 0; u < kSelRegs; ++u) take(code[u], tid + u * kSelThreads);
  for (int e = in_regs + tid; e < total; e += kSelThreads) take(sel_code(__ldg(rowl + e)), e);
  __syncthreads();
  if (!whole) {
    // the k-th value is shared by more entries than are still needed: the krem lowest ids
    // among the entries whose code is exactly the prefix, one block-wide minimum at a time
    int last = -1;
    for (uint32_t t = 0; t < krem; ++t) {
      int best = 0x7fffffff;
#pragma unroll
      for (int u = 0; u < kSelRegs; ++u) {
        if (code[u] == prefix) {
          const int id = __float_as_int(__ldg(rowl + tid + u * kSelThreads).y);
          if (id > last && id < best) best = id;
        }
      }
      for (int e = in_regs + tid; e < total; e += kSelThreads) {
        const float2 x = __ldg(rowl + e);
        const int id = __float_as_int(x.y);
        if (sel_code(x) == prefix && id > last && id < best) best = id;
      }
      best = __reduce_min_sync(0xffffffffu, best);
      if (lane == 0) s_min[warp] = best;
      __syncthreads();
      if (warp == 0) {
        int b = lane < kSelThreads / 32 ? s_min[lane] : 0x7fffffff;
        b = __reduce_min_sync(0xffffffffu, b);
        if (lane == 0) {
          const uint32_t at = s_n++;
          if (at < 16u) {
            sv[at] = dec_order(prefix);
            si[at] = b;
          }
          s_min[0] = b;
        }
      }
      __syncthreads();
      last = s_min[0];
      __syncthreads();
    }
  }
  if (warp == 0) {                                     // the candidates in screen order
    float v = -INFINITY;
    int id = 0x7fffffff;
    const int nn = min((int)s_n, k);
    if (lane < nn) {
      v = sv[lane];
      id = si[lane];
    }
    int rank = 0;
    for (int j = 0; j < nn; ++j) rank += before(sv[j], si[j], v, id);
    if (lane < nn) cand[(size_t)m * 16 + rank] = id;
    else if (lane < k) cand[(size_t)m * 16 + lane] = -1;
  }
  // The exact logits z_c = h . W_c of the k candidates, one warp each (fp32, the hidden row from
  // shared memory, four W words per lane in flight), then the k ordered by z_c descending, the
  // lower id first on equal values.  Missing candidates (fewer than k entries) are (-1, -inf).
  const int n = min((int)s_n, k);
  if (warp < k) {
    const int c = warp < n ? si[warp] : -1;
    float acc = -INFINITY;
    if (c >= 0 && c < V) {
      const uint4* w = reinterpret_cast<const uint4*>(W + (size_t)c * H);
      acc = 0.f;
      for (int i0 = lane; i0 < H / 8; i0 += 32 * 4) {
        uint4 wv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + 32 * u;
          wv[u] = i < H / 8 ? __ldg(w + i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + 32 * u;
          if (i >= H / 8) break;
          const uint4 a = hsm[i];
          const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&wv[u]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 fa = __bfloat1622float2(a2[q]), fb = __bfloat1622float2(b2[q]);
            acc = fmaf(fa.x, fb.x, acc);
            acc = fmaf(fa.y, fb.y, acc);
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    }
    if (lane == 0) {
      zs[warp] = acc;
      cs[warp] = c;
    }
  }
  __syncthreads();
  if (tid == 0) {
    for (int i = 1; i < k; ++i) {                    // insertion sort of <= 16
      const float x = zs[i];
      const int ci = cs[i];
      int j = i - 1;
      while (j >= 0 && (zs[j] < x || (zs[j] == x && (unsigned)cs[j] > (unsigned)ci))) {
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
int lowrank_down_chunks(int H) { return (H + kSkChunk - 1) / kSkChunk; }

static const int kSkSmem = 1024 + 2 * 16384;     // two K steps of A and B boxes, 1 KB aligned

static cudaError_t launch_splitk(const CUtensorMap& ta, const CUtensorMap& tb, int M, int K, int N,
                                 float* part, WsHeader* ws, cudaStream_t s) {
  dim3 grid((N + kSkTile - 1) / kSkTile, (K + kSkChunk - 1) / kSkChunk, (M + kSkTile - 1) / kSkTile);
  return launch_pdl(lr_splitk_kernel, grid, dim3(128), (size_t)kSkSmem, s, ta, tb, M, K, N, part,
                    ws);
}

cudaError_t launch_lowrank_down(const CUtensorMap& tm_h, const CUtensorMap& tm_d, int M, int H,
                                int r, float* part, __nv_bfloat16* g, uint32_t* tkth,
                                int32_t* fcnt, WsHeader* ws, cudaStream_t s) {
  cudaError_t e = launch_splitk(tm_h, tm_d, M, H, r, part, ws, s);
  if (e != cudaSuccess) return e;
  return launch_pdl(lr_reduce_kernel, dim3((M * r + 255) / 256), dim3(256), 0, s, part,
                    lowrank_down_chunks(H), M, r, g, tkth, fcnt);
}

int lowrank_sample_cols(int V) { return V < 8192 ? V : 8192; }

int lowrank_floor_maxima(int M) { return M * kFloorParts * 256; }

cudaError_t launch_lowrank_sample(const CUtensorMap& tm_g, const CUtensorMap& tm_us, int M, int r,
                                  int V, float* part, float* fmax, int32_t* fcnt, uint32_t* tkth,
                                  WsHeader* ws, cudaStream_t s) {
  const int S = lowrank_sample_cols(V);
  cudaError_t e = launch_splitk(tm_g, tm_us, M, r, S, part, ws, s);
  if (e != cudaSuccess) return e;
  return launch_pdl(sample_floor_kernel, dim3(M * kFloorParts), dim3(256), 0, s, part,
                    lowrank_down_chunks(r), M, S, fmax, fcnt, tkth);
}

cudaError_t launch_lowrank_finish(const float2* lists, int nlists, int M, int k, int32_t* cand,
                                  const __nv_bfloat16* hid, const __nv_bfloat16* W, int H, int V,
                                  int32_t* out_ids, float* out_logit, cudaStream_t s) {
  return launch_pdl(topk_select_kernel, dim3(M), dim3(kSelThreads), 0, s, lists, nlists, k, cand,
                    hid, W, H, V, out_ids, out_logit);
}

}  // namespace etree
