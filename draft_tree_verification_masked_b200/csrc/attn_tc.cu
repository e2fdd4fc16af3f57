// attn_tc.cu -- tree-masked GQA attention on tcgen05 / TMEM (sm_100a).
//
// Same computation as the split-KV kernel in attn_tree.cu (every tree node attends to its
// request's cached keys and to its tree ancestors and itself: "Eagle-4 Released: Outpaces
// DFlash2 and DSpark ...", section "Technical Background"), with both matrix products on the
// 5th-generation tensor cores:
//
//   S  = Q K^T   tcgen05.mma M=128 (query rows) x N=64 (keys) x K=128, fp32 into TMEM;
//   O += P V     tcgen05.mma M=128 x N=128 (head dims) x K=64 (keys), fp32 accumulated in TMEM.
//
// One CTA = (request, KV head, 128-row block, KV split).  The query rows are the (node, group
// head) pairs of one KV head, row = node * G + g; one TMA box {64 dims, G heads, NB nodes} of the
// [n_total][hq][128] query tensor lands them in exactly that order (NB = floor(128 / G)).
// Warp 0 streams Q once and the 64-key K/V tiles through a STAGES-deep ring; warp 1 issues the
// MMAs; warps 2-5 own one query row per thread (= one TMEM lane): they read S from TMEM, apply
// the key mask (cache length, or the row's ancestor bitmask on the tree tile), run the online
// softmax in log2 units, and write P (bf16, 128-byte swizzle) to shared memory for the PV
// product.  S is double-buffered in TMEM so QK^T of tile j+1 overlaps the softmax of tile j.
// O is rescaled lazily: only when a row's running maximum grows by more than 2^8 does the
// softmax read-modify-write O in TMEM, so P stays below 256 and the usual case has no O traffic.
#include "kernels.cuh"

namespace etree {

namespace {
constexpr int kKeys = 64;
constexpr int kKV = 4 * 8192;               // K lo/hi + V lo/hi boxes of [64 keys][64 dims]
constexpr int kQBytes = 2 * 16384;          // Q lo/hi boxes of [128 rows][64 dims]
constexpr int kPBytes = 16384;              // one P buffer: [128 rows][64 keys] bf16
constexpr float kLazy = 8.0f;               // rescale O only when the max grows by > 2^8

struct TcSmem {
  // barriers and small arrays, placed after the 1024-aligned tile area
  uint64_t kv_full[4], kv_empty[4], q_full, s_full[2], s_free[2], p_full[2], p_free[2];
  uint64_t anc[64];
  int32_t par[64];
  uint32_t tmem;
};
}  // namespace

template <int STAGES>
__global__ void __launch_bounds__(192, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
               const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kt,
               const __grid_constant__ CUtensorMap tm_vt, AttnParams p, int NB) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                                   // 32 KB
  uint8_t* sKV = smem + kQBytes;                        // STAGES x 32 KB
  uint8_t* sP = sKV + STAGES * kKV;                     // 2 x 16 KB (double buffer)
  TcSmem* sh = reinterpret_cast<TcSmem*>(sP + 2 * kPBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_req = p.hkv * p.mchunks;
  const int r = blockIdx.x / per_req;
  const int kvh = (blockIdx.x % per_req) / p.mchunks;
  const int mb = blockIdx.x % p.mchunks;
  const int s = blockIdx.y;
  const int G = p.G;

  const int base = p.cu_nodes[r];
  const int n = p.cu_nodes[r + 1] - base;
  const int L = p.kv_len[r];
  const int64_t sbase = p.slot_base[r];
  if (n < 1 || n > p.n_max || L < 0 || L > p.kv_len_max || sbase < 0 ||
      sbase + L > p.cache_slots) {
    if (threadIdx.x == 0 && s == 0 && mb == 0 && kvh == 0)
      report(p.ws, ETREE_EDEVICE, (n < 1 || n > p.n_max) ? DET_BAD_NODES : DET_KV_LEN);
    return;
  }
  const int node0 = mb * NB;
  if (node0 >= n) return;
  const int nt_cache = (L + kKeys - 1) / kKeys;
  const int total = nt_cache + 1;                       // the tree tile comes last
  const int t0 = s * p.tps;
  const int t1 = min(total, t0 + p.tps);
  if (t0 >= t1) return;
  const int T = t1 - t0;
  const bool has_tree = (t1 == total);
  const int qrows = NB * G;                             // rows the Q box fills

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&sh->kv_full[i], 1);
      mbar_init(&sh->kv_empty[i], 1);
    }
    mbar_init(&sh->q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->s_full[b], 1);
      mbar_init(&sh->s_free[b], 4);
      mbar_init(&sh->p_full[b], 4);
      mbar_init(&sh->p_free[b], 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem, 256);
    tmem_relinquish();
  }
  if (has_tree) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) sh->par[i] = p.parent[base + i];
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      uint64_t m = 0;
      int j = i, steps = 0;
      bool ok = true;
      while (j >= 0 && steps <= 64) {
        m |= 1ull << j;
        const int pj = sh->par[j];
        if ((j == 0 && pj != -1) || (j > 0 && (pj < 0 || pj >= j))) { ok = false; break; }
        j = pj;
        ++steps;
      }
      if (!ok) {
        m = 1ull << i;                                  // a malformed tree: each node sees itself
        report(p.ws, ETREE_EDEVICE, DET_BAD_PARENT);
      }
      sh->anc[i] = m;
    }
  }
  // rows past the Q box are zero so that their (unused) products stay finite
  for (int i = threadIdx.x; i < (128 - qrows) * 16; i += blockDim.x) {
    const int row = qrows + i / 16, c = i % 16;
    uint4* dst = reinterpret_cast<uint4*>(sQ + (c >> 3) * 16384 + row * 128 + (c & 7) * 16);
    *dst = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem;

  if (warp == 0) {
    // ------------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_kc);
      prefetch_tmap(&tm_vc);
      mbar_arrive_expect_tx(&sh->q_full, 2 * qrows * 128);
      tma_load_3d(sQ, &tm_q, &sh->q_full, 0, kvh * G, base + node0);
      tma_load_3d(sQ + 16384, &tm_q, &sh->q_full, 64, kvh * G, base + node0);
      for (int j = 0; j < T; ++j) {
        const int t = t0 + j;
        const int st = j % STAGES;
        const uint32_t ph = (j / STAGES) & 1;
        if (j >= STAGES && !mbar_wait(&sh->kv_empty[st], ph ^ 1)) {
          report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
          break;
        }
        uint8_t* dst = sKV + st * kKV;
        mbar_arrive_expect_tx(&sh->kv_full[st], kKV);
        if (t < nt_cache) {
          const int32_t slot = static_cast<int32_t>(sbase + (int64_t)t * kKeys);
          tma_load_3d(dst, &tm_kc, &sh->kv_full[st], 0, kvh, slot);
          tma_load_3d(dst + 8192, &tm_kc, &sh->kv_full[st], 64, kvh, slot);
          tma_load_3d(dst + 16384, &tm_vc, &sh->kv_full[st], 0, kvh, slot);
          tma_load_3d(dst + 24576, &tm_vc, &sh->kv_full[st], 64, kvh, slot);
        } else {
          tma_load_3d(dst, &tm_kt, &sh->kv_full[st], 0, kvh, base);
          tma_load_3d(dst + 8192, &tm_kt, &sh->kv_full[st], 64, kvh, base);
          tma_load_3d(dst + 16384, &tm_vt, &sh->kv_full[st], 0, kvh, base);
          tma_load_3d(dst + 24576, &tm_vt, &sh->kv_full[st], 64, kvh, base);
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, kKeys);
      const uint32_t idO = idesc_bf16_f32(128, 128) | (1u << 16);   // B (V) is MN-major
      bool ok = mbar_wait(&sh->q_full, 0);
      tc_fence_after();
      const uint64_t dq0 = smem_desc_sw128(sQ), dq1 = smem_desc_sw128(sQ + 16384);
      auto pv = [&](int jj) -> bool {
        const int pb = jj & 1;
        if (!mbar_wait(&sh->p_full[pb], (jj >> 1) & 1)) return false;
        tc_fence_after();
        const uint64_t dp = smem_desc_sw128(sP + pb * kPBytes);
        const uint8_t* v0 = sKV + (jj % STAGES) * kKV + 16384;
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k)
          tc_mma_bf16(tmem + 128, dp + 2 * k, smem_desc_sw128_mn(v0 + k * 2048, 8192), idO,
                      (jj > 0 || k > 0) ? 1u : 0u);
        tc_commit(&sh->p_free[pb]);
        tc_commit(&sh->kv_empty[jj % STAGES]);
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % STAGES;
        const int sb = j & 1;
        if (!mbar_wait(&sh->kv_full[st], (j / STAGES) & 1)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&sh->s_free[sb], ((j >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint8_t* k0 = sKV + st * kKV;
        const uint64_t dk0 = smem_desc_sw128(k0), dk1 = smem_desc_sw128(k0 + 8192);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc_mma_bf16(tmem + sb * kKeys, (k < 4 ? dq0 : dq1) + 2 * (k & 3),
                      (k < 4 ? dk0 : dk1) + 2 * (k & 3), idS, k > 0 ? 1u : 0u);
        tc_commit(&sh->s_full[sb]);
        if (j >= 1 && !pv(j - 1)) { ok = false; break; }
      }
      if (ok && !pv(T - 1)) ok = false;
      if (!ok) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
    }
  } else {
    // ------------------------------------------------------------------- softmax warpgroup
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int node_l = row / G, g = row - node_l * G;
    const int node = node0 + node_l;
    const bool valid = row < qrows && node < n;
    const uint64_t anc = (has_tree && valid) ? sh->anc[node] : 0ull;
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int t = t0 + j;
      const int sb = j & 1;
      if (!mbar_wait(&sh->s_full[sb], (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      float sc[64];
      {
        float a[32], b[32];
        tmem_ld32(lane_base + sb * kKeys, a);
        tmem_ld32(lane_base + sb * kKeys + 32, b);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sc[c] = a[c];
          sc[32 + c] = b[c];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->s_free[sb]);

      // keep-mask of this row's 64 keys: the cache positions below kv_len, or on the tree
      // tile the row's ancestor bits
      uint32_t klo, khi;
      if (!valid) {
        klo = khi = 0u;
      } else if (t == nt_cache) {
        klo = static_cast<uint32_t>(anc);
        khi = static_cast<uint32_t>(anc >> 32);
      } else {
        const int lim = L - t * kKeys;                  // >= 1 on a cache tile
        klo = lim >= 32 ? 0xffffffffu : ((1u << lim) - 1u);
        khi = lim >= 64 ? 0xffffffffu : (lim > 32 ? ((1u << (lim - 32)) - 1u) : 0u);
      }
      const float sl = p.scale_log2;
      float t0m = -INFINITY, t1m = -INFINITY, t2m = -INFINITY, t3m = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        const uint32_t w = c < 32 ? klo : khi;
        const int b0 = c & 31;
        const float v0 = ((w >> b0) & 1u) ? sc[c] * sl : -INFINITY;
        const float v1 = ((w >> (b0 + 1)) & 1u) ? sc[c + 1] * sl : -INFINITY;
        const float v2 = ((w >> (b0 + 2)) & 1u) ? sc[c + 2] * sl : -INFINITY;
        const float v3 = ((w >> (b0 + 3)) & 1u) ? sc[c + 3] * sl : -INFINITY;
        sc[c] = v0;
        sc[c + 1] = v1;
        sc[c + 2] = v2;
        sc[c + 3] = v3;
        t0m = fmaxf(t0m, v0);
        t1m = fmaxf(t1m, v1);
        t2m = fmaxf(t2m, v2);
        t3m = fmaxf(t3m, v3);
      }
      const float tmax = fmaxf(fmaxf(t0m, t1m), fmaxf(t2m, t3m));
      const bool need = tmax > m_ref + kLazy;           // also true for the first finite max
      const bool any = __any_sync(0xffffffffu, need);
      const float m_new = need ? tmax : m_ref;
      const float off = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = need ? exp2f(m_ref - m_new) : 1.f;
      float ls0 = 0.f, ls1 = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float e0 = ex2_approx(sc[2 * c] - off), e1 = ex2_approx(sc[2 * c + 1] - off);
        ls0 += e0;
        ls1 += e1;
        pk[c] = pack_bf16x2(e0, e1);
      }
      l = l * corr + (ls0 + ls1);
      m_ref = m_new;
      // A rescale of O needs every earlier PV product finished (the last one wrote O).
      if (any && j >= 1) {
        if (!mbar_wait(&sh->p_free[(j - 1) & 1], ((j - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(lane_base + 128 + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= corr;
          tmem_st32(lane_base + 128 + c * 32, o);
        }
      }
      // P buffer j % 2 is free once PV(j - 2) has completed
      const int pb = j & 1;
      if (j >= 2) {
        if (!mbar_wait(&sh->p_free[pb], ((j >> 1) & 1) ^ 1)) { ok = false; break; }
      }
      uint8_t* prow = sP + pb * kPBytes + row * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = v;
      }
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->p_full[pb]);
    }
    if (ok && !mbar_wait(&sh->p_free[(T - 1) & 1], ((T - 1) >> 1) & 1)) ok = false;
    if (!ok) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
    tc_fence_after();
    const size_t gidx = (size_t)(base + (valid ? node : 0)) * p.hq + kvh * G + g;
    if (p.nsplit == 1) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(lane_base + 128 + c * 32, o);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + gidx * 128 + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                                pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
        }
      }
      if (valid && p.lse) p.lse[gidx] = (m_ref + log2f(l)) * 0.69314718055994531f;
    } else {
      float* op = p.o_part + (gidx * p.nsplit + s) * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(lane_base + 128 + c * 32, o);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(op + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
      }
      if (valid) p.ml_part[gidx * p.nsplit + s] = make_float2(m_ref, l);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

size_t attn_tc_smem_bytes(int stages) {
  return 1024 + kQBytes + (size_t)stages * kKV + 2 * kPBytes + sizeof(TcSmem);
}

cudaError_t launch_attn_tc(const CUtensorMap& q, const CUtensorMap& kc, const CUtensorMap& vc,
                           const CUtensorMap& kt, const CUtensorMap& vt, const AttnParams& p,
                           int nb, int stages, int n_total, cudaStream_t stream) {
  dim3 grid(p.B * p.hkv * p.mchunks, p.nsplit);
  cudaError_t e;
  if (stages >= 4) {
    auto k = attn_tc_kernel<4>;
    const size_t smem = attn_tc_smem_bytes(4);
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 192, smem, stream>>>(q, kc, vc, kt, vt, p, nb);
  } else {
    auto k = attn_tc_kernel<3>;
    const size_t smem = attn_tc_smem_bytes(3);
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 192, smem, stream>>>(q, kc, vc, kt, vt, p, nb);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || p.nsplit == 1) return e;
  return launch_attn_combine(p, n_total, stream);
}

}  // namespace etree
