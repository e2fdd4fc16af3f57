// attn_tree.cu -- tree-masked GQA attention for draft-tree verification (sm_100a).
//
// Every draft-tree node attends to its request's cached keys and to the tree nodes that are its
// ancestors or itself: the target verifies all drafted tokens in one parallel forward, and a
// draft tree lets one verification cover several candidate paths ("Eagle-4 Released: Outpaces
// DFlash2 and DSpark ...", section "Technical Background").  Single-request decoding moves data
// rather than computing ("EAGLE-4 是什麼？...", aiposthub.com, opening section), so the kernel is
// built around reading each KV byte from HBM once for all tree nodes and all query heads of a
// KV-head group.
//
// Design.  One CTA = (request, KV head, row chunk, KV split).  Its query rows are the
// (node, group head) pairs of one KV head: row = node * G + g, so one staged K/V tile serves
// n * G query rows.  A producer warp streams 64-key K/V tiles with TMA (128-byte swizzle) into a
// STAGES-deep shared-memory ring guarded by mbarriers; NW consumer warps own 16 query rows each
// and run QK^T and PV on the tensor cores (m16n8k16, fp32 accumulate) with an online softmax
// whose row max / sum reductions are quad shuffles.  The tree's own keys form one extra tile at
// the end of the request's work list; its mask is each row's uint64 ancestor bitmask, held in a
// register.  Split partials (unnormalised O, running max, running sum) are merged by a
// log-sum-exp combine kernel.
#include "kernels.cuh"

namespace etree {

constexpr int kTileKeys = 64;
constexpr int kStageBytes = 4 * 8192;   // K lo/hi + V lo/hi boxes of [64 keys][64 dims] bf16


__device__ __forceinline__ uint32_t swz(uint32_t box, int key, int chunk) {
  return box + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
}

template <int NW, int STAGES>
__global__ void __launch_bounds__((NW + 1) * 32)
attn_tree_kernel(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                 const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_vt,
                 AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* anc_s = empty + STAGES;              // [64] ancestor masks of the request's nodes
  int* flags = reinterpret_cast<int*>(anc_s + 64);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_req = p.hkv * p.mchunks;
  const int r = p.order ? p.order[blockIdx.x / per_req] : blockIdx.x / per_req;
  const int kvh = (blockIdx.x % per_req) / p.mchunks;
  const int mc = blockIdx.x % p.mchunks;
  const int s = blockIdx.y;

  const int base = p.cu_nodes[r];
  const int n = p.cu_nodes[r + 1] - base;
  const int L = p.kv_len[r];
  const int64_t sbase = p.slot_base[r];
  if (n < 1 || n > p.n_max || L < 0 || L > p.kv_len_max || sbase < 0 ||
      sbase + L > p.cache_slots) {
    if (threadIdx.x == 0 && s == 0 && mc == 0 && kvh == 0)
      report(p.ws, ETREE_EDEVICE, (n < 1 || n > p.n_max) ? DET_BAD_NODES : DET_KV_LEN);
    return;
  }
  const int R = n * p.G;
  const int row0 = mc * NW * 16;
  if (row0 >= R) return;
  const int nt_cache = (L + kTileKeys - 1) / kTileKeys;
  const int total = nt_cache + 1;                  // the tree tile comes last
  const int t0 = s * p.tps;
  const int t1 = min(total, t0 + p.tps);
  if (t0 >= t1) return;
  const bool has_tree = (t1 == total);

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    flags[0] = 0;
    fence_barrier_init();
  }
  if (has_tree) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      uint64_t m = 0;
      int j = i, steps = 0;
      bool ok = true;
      while (j >= 0 && steps <= 64) {
        m |= 1ull << j;
        int pj = p.parent[base + j];
        if ((j == 0 && pj != -1) || (j > 0 && (pj < 0 || pj >= j))) { ok = false; break; }
        j = pj;
        ++steps;
      }
      if (!ok) {
        m = 1ull << i;                             // a malformed tree: each node sees itself
        report(p.ws, ETREE_EDEVICE, DET_BAD_PARENT);
      }
      anc_s[i] = m;
    }
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------------------------------------------- TMA producer warp
    if (lane == 0) {
      prefetch_tmap(&tm_kc);
      prefetch_tmap(&tm_vc);
      for (int t = t0, it = 0; t < t1; ++t, ++it) {
        const int st = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (it >= STAGES && !mbar_wait(&empty[st], ph ^ 1)) {
          report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
          break;
        }
        uint8_t* dst = smem + st * kStageBytes;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        if (t < nt_cache) {
          const int32_t slot = static_cast<int32_t>(sbase + (int64_t)t * kTileKeys);
          tma_load_3d(dst, &tm_kc, &full[st], 0, kvh, slot);
          tma_load_3d(dst + 8192, &tm_kc, &full[st], 64, kvh, slot);
          tma_load_3d(dst + 16384, &tm_vc, &full[st], 0, kvh, slot);
          tma_load_3d(dst + 24576, &tm_vc, &full[st], 64, kvh, slot);
        } else {
          tma_load_3d(dst, &tm_kt, &full[st], 0, kvh, base);
          tma_load_3d(dst + 8192, &tm_kt, &full[st], 64, kvh, base);
          tma_load_3d(dst + 16384, &tm_vt, &full[st], 0, kvh, base);
          tma_load_3d(dst + 24576, &tm_vt, &full[st], 64, kvh, base);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------------ consumer warps
    const int quad = lane >> 2, qc = lane & 3;
    const int rA = row0 + warp * 16 + quad, rB = rA + 8;
    const bool vA = rA < R, vB = rB < R;
    const int iA = vA ? rA / p.G : 0, iB = vB ? rB / p.G : 0;
    const int hA = kvh * p.G + (vA ? rA % p.G : 0), hB = kvh * p.G + (vB ? rB % p.G : 0);
    const uint64_t ancA = (has_tree && vA) ? anc_s[iA] : 0ull;
    const uint64_t ancB = (has_tree && vB) ? anc_s[iB] : 0ull;

    // Q fragments of this warp's 16 rows (A operand, row-major): 8 k-steps of 16 dims.
    uint32_t qf[8][4];
    {
      const uint32_t* qa = reinterpret_cast<const uint32_t*>(
          p.q + ((size_t)(base + iA) * p.hq + hA) * 128);
      const uint32_t* qb = reinterpret_cast<const uint32_t*>(
          p.q + ((size_t)(base + iB) * p.hq + hB) * 128);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        qf[kk][0] = vA ? __ldg(qa + kk * 8 + qc) : 0u;
        qf[kk][1] = vB ? __ldg(qb + kk * 8 + qc) : 0u;
        qf[kk][2] = vA ? __ldg(qa + kk * 8 + 4 + qc) : 0u;
        qf[kk][3] = vB ? __ldg(qb + kk * 8 + 4 + qc) : 0u;
      }
    }

    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;

    for (int t = t0, it = 0; t < t1; ++t, ++it) {
      const int st = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      if (!mbar_wait(&full[st], ph)) {
        report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
        break;
      }
      const uint32_t k0 = smem_u32(smem + st * kStageBytes);
      const uint32_t k1 = k0 + 8192, v0 = k0 + 16384, v1 = k0 + 24576;

      // S = Q K^T over this tile's 64 keys
      float sc[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int cidx = 2 * kk + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(swz(cidx < 8 ? k0 : k1, key, cidx), b0, b1, b2, b3);
          mma_bf16_16816(sc[2 * np], qf[kk], b0, b1);
          mma_bf16_16816(sc[2 * np + 1], qf[kk], b2, b3);
        }
      }

      // mask, scale into log2 units, online softmax
      const bool tree_tile = (t == nt_cache);
      float tmA = -INFINITY, tmB = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = nt * 8 + qc * 2 + (e & 1);
          bool ok;
          if (tree_tile) {
            const uint64_t a = (e < 2) ? ancA : ancB;
            ok = col < n && ((a >> col) & 1ull);
          } else {
            ok = t * kTileKeys + col < L;
          }
          const float v = ok ? sc[nt][e] * p.scale_log2 : -INFINITY;
          sc[nt][e] = v;
          if (e < 2) tmA = fmaxf(tmA, v); else tmB = fmaxf(tmB, v);
        }
      }
      tmA = fmaxf(tmA, __shfl_xor_sync(0xffffffffu, tmA, 1));
      tmA = fmaxf(tmA, __shfl_xor_sync(0xffffffffu, tmA, 2));
      tmB = fmaxf(tmB, __shfl_xor_sync(0xffffffffu, tmB, 1));
      tmB = fmaxf(tmB, __shfl_xor_sync(0xffffffffu, tmB, 2));
      const float nmA = fmaxf(mA, tmA), nmB = fmaxf(mB, tmB);
      const float baseA = (nmA == -INFINITY) ? 0.f : nmA;
      const float baseB = (nmB == -INFINITY) ? 0.f : nmB;
      const float cA = exp2f(mA - baseA), cB = exp2f(mB - baseB);
      mA = nmA;
      mB = nmB;
      float sA = 0.f, sB = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        sc[nt][0] = exp2f(sc[nt][0] - baseA);
        sc[nt][1] = exp2f(sc[nt][1] - baseA);
        sc[nt][2] = exp2f(sc[nt][2] - baseB);
        sc[nt][3] = exp2f(sc[nt][3] - baseB);
        sA += sc[nt][0] + sc[nt][1];
        sB += sc[nt][2] + sc[nt][3];
      }
      lA = lA * cA + sA;
      lB = lB * cB + sB;
#pragma unroll
      for (int dt = 0; dt < 16; ++dt) {
        o[dt][0] *= cA;
        o[dt][1] *= cA;
        o[dt][2] *= cB;
        o[dt][3] *= cB;
      }

      // O += P V  (P from the score registers, V via transposed ldmatrix)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2(sc[2 * j][0], sc[2 * j][1]);
        pa[1] = pack_bf16x2(sc[2 * j][2], sc[2 * j][3]);
        pa[2] = pack_bf16x2(sc[2 * j + 1][0], sc[2 * j + 1][1]);
        pa[3] = pack_bf16x2(sc[2 * j + 1][2], sc[2 * j + 1][3]);
#pragma unroll
        for (int dp = 0; dp < 8; ++dp) {
          const int key = 16 * j + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int cidx = dp * 2 + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(swz(cidx < 8 ? v0 : v1, key, cidx), b0, b1, b2, b3);
          mma_bf16_16816(o[2 * dp], pa, b0, b1);
          mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }

    lA += __shfl_xor_sync(0xffffffffu, lA, 1);
    lA += __shfl_xor_sync(0xffffffffu, lA, 2);
    lB += __shfl_xor_sync(0xffffffffu, lB, 1);
    lB += __shfl_xor_sync(0xffffffffu, lB, 2);

    const size_t gA = (size_t)(base + iA) * p.hq + hA;
    const size_t gB = (size_t)(base + iB) * p.hq + hB;
    if (p.nsplit == 1) {
      const float invA = lA > 0.f ? 1.f / lA : 0.f, invB = lB > 0.f ? 1.f / lB : 0.f;
#pragma unroll
      for (int dt = 0; dt < 16; ++dt) {
        const int col = dt * 8 + qc * 2;
        if (vA)
          *reinterpret_cast<uint32_t*>(p.out + gA * 128 + col) =
              pack_bf16x2(o[dt][0] * invA, o[dt][1] * invA);
        if (vB)
          *reinterpret_cast<uint32_t*>(p.out + gB * 128 + col) =
              pack_bf16x2(o[dt][2] * invB, o[dt][3] * invB);
      }
      if (p.lse && qc == 0) {
        if (vA) p.lse[gA] = (mA + log2f(lA)) * 0.69314718055994531f;
        if (vB) p.lse[gB] = (mB + log2f(lB)) * 0.69314718055994531f;
      }
    } else {
      float* opA = p.o_part + (gA * p.nsplit + s) * 128;
      float* opB = p.o_part + (gB * p.nsplit + s) * 128;
#pragma unroll
      for (int dt = 0; dt < 16; ++dt) {
        const int col = dt * 8 + qc * 2;
        if (vA) *reinterpret_cast<float2*>(opA + col) = make_float2(o[dt][0], o[dt][1]);
        if (vB) *reinterpret_cast<float2*>(opB + col) = make_float2(o[dt][2], o[dt][3]);
      }
      if (qc == 0) {
        if (vA) p.ml_part[gA * p.nsplit + s] = make_float2(mA, lA);
        if (vB) p.ml_part[gB * p.nsplit + s] = make_float2(mB, lB);
      }
    }
  }
  __syncthreads();
}

// Merge the split partials of each (node, head) row by log-sum-exp: one warp per row, each lane
// owning 4 of the 128 output dims.
__global__ void attn_combine_kernel(AttnParams p, int n_total) {
  pdl_wait();                                      // the split partials of the attention kernel
  pdl_trigger();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= n_total * p.hq) return;
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
  const int used = min(p.nsplit, (total + p.tps - 1) / p.tps);
  const float2* mlp = p.ml_part + (size_t)gw * p.nsplit;
  const float4* op = reinterpret_cast<const float4*>(p.o_part + (size_t)gw * p.nsplit * 128);
  // the maximum: one split per lane, then across the warp
  float M = -INFINITY;
  for (int s = lane; s < used; s += 32) M = fmaxf(M, mlp[s].x);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float Mb = (M == -INFINITY) ? 0.f : M;
  // the weighted sums in split order, eight splits' loads in flight at a time
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  for (int s0 = 0; s0 < used; s0 += 8) {
    float2 ml[8];
    float4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool in = s0 + i < used;
      ml[i] = in ? mlp[s0 + i] : make_float2(-INFINITY, 0.f);
      v[i] = in ? op[(size_t)(s0 + i) * 32 + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float w = s0 + i < used ? exp2f(ml[i].x - Mb) : 0.f;
      lsum += ml[i].y * w;
      acc.x += v[i].x * w;
      acc.y += v[i].y * w;
      acc.z += v[i].z * w;
      acc.w += v[i].w * w;
    }
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  uint2 packed;
  packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(p.out + (size_t)gw * 128)[lane] = packed;
  if (p.lse && lane == 0) p.lse[gw] = (M + log2f(lsum)) * 0.69314718055994531f;
}

// ------------------------------------------------------------------------------- host launcher
template <int NW>
static cudaError_t launch_attn_nw(const CUtensorMap& kc, const CUtensorMap& vc,
                                  const CUtensorMap& kt, const CUtensorMap& vt,
                                  const AttnParams& p, int stages, cudaStream_t stream) {
  dim3 grid(p.B * p.hkv * p.mchunks, p.nsplit);
  dim3 block((NW + 1) * 32);
  if (stages == 4) {
    const size_t smem = 4 * kStageBytes + 1024 + 2 * 4 * 8 + 64 * 8 + 64;
    auto k = attn_tree_kernel<NW, 4>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, block, smem, stream>>>(kc, vc, kt, vt, p);
  } else {
    const size_t smem = 3 * kStageBytes + 1024 + 2 * 3 * 8 + 64 * 8 + 64;
    auto k = attn_tree_kernel<NW, 3>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, block, smem, stream>>>(kc, vc, kt, vt, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_attn(const CUtensorMap& kc, const CUtensorMap& vc, const CUtensorMap& kt,
                        const CUtensorMap& vt, const AttnParams& p, int nw, int stages,
                        int n_total, cudaStream_t stream) {
  cudaError_t e;
  switch (nw) {
    case 1: e = launch_attn_nw<1>(kc, vc, kt, vt, p, stages, stream); break;
    case 2: e = launch_attn_nw<2>(kc, vc, kt, vt, p, stages, stream); break;
    case 3: e = launch_attn_nw<3>(kc, vc, kt, vt, p, stages, stream); break;
    case 4: e = launch_attn_nw<4>(kc, vc, kt, vt, p, stages, stream); break;
    case 5: e = launch_attn_nw<5>(kc, vc, kt, vt, p, stages, stream); break;
    case 6: e = launch_attn_nw<6>(kc, vc, kt, vt, p, stages, stream); break;
    case 7: e = launch_attn_nw<7>(kc, vc, kt, vt, p, stages, stream); break;
    default: e = launch_attn_nw<8>(kc, vc, kt, vt, p, stages, stream); break;
  }
  if (e != cudaSuccess || p.nsplit == 1) return e;
  return launch_attn_combine(p, n_total, stream);
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
  return launch_pdl(attn_combine_kernel, dim3(blocks), dim3(threads), 0, stream, p, n_total);
}

}  // namespace etree
