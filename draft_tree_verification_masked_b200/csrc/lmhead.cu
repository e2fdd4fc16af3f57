// lmhead.cu -- LM-head GEMM on tcgen05 / TMEM with fused per-row reductions (sm_100a).
//
// Verification scores every tree node with the target's own output distribution: the target
// keeps the drafted prefix that agrees with it and emits one token of its own after the first
// rejection ("Eagle-4 Released: Outpaces DFlash2 and DSpark ...", section "Technical
// Background").  The vocabulary projection is the largest single matrix of that pass (on the
// draft side the pages measure the vocab head at 65.4% of a draft forward: "EAGLE-4 是什麼？...",
// aiposthub.com, Fig. 2 paragraph), so z = hidden W^T runs on the 5th-generation tensor cores and
// its N x vocab logits are never written to memory: each 128 x 256 accumulator tile is reduced
// in the epilogue, straight out of tensor memory, to a few numbers per row.
//
// Kernel shape.  Persistent: one CTA per SM walks the (row tile, vocab tile) list, vocab-major
// so that concurrently running CTAs share W tiles through L2.  Warp 0 streams 128x64 hidden
// tiles and 256x64 W tiles with TMA (128-byte swizzle) into a 4-deep shared-memory ring; warp 1
// issues tcgen05.mma (M=128, N=256, K=16, bf16 in, fp32 out) into one of two 256-column TMEM
// accumulators; warps 2-5 drain the other accumulator with tcgen05.ld, one TMEM lane (= one
// output row) per thread, and apply the epilogue:
//   EPI_ARGMAX  per row and tile: top-1 value, its vocab id (lowest on ties) and top-2 value;
//   EPI_LSE     per row and tile: m = max z*log2(e)/T and sum 2^(z*log2(e)/T - m), plus the
//               logit of the row's child token when it falls in the tile;
//   EPI_RACE    per row and tile: the exponential-race winners log w_v - log(-log U_v) for
//               w = max(0, p - q) and for w = p, with Philox4x64-10 uniforms.
#include "kernels.cuh"
#include "philox.cuh"

namespace etree {

constexpr int kBM = 128, kBN = 256, kBK = 64, kGStages = 4;
constexpr int kABytes = kBM * kBK * 2, kBBytes = kBN * kBK * 2;
enum Epi { EPI_ARGMAX = 0, EPI_LSE = 1, EPI_RACE = 2 };


template <int EPI>
__global__ void __launch_bounds__(192, 1)
lmhead_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kGStages * kBBytes);
  uint64_t* empty = full + kGStages;
  uint64_t* accf = empty + kGStages;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ----------------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int st = it % kGStages;
          const uint32_t ph = (it / kGStages) & 1;
          if (!mbar_wait(&empty[st], ph ^ 1)) {
            report(p.ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[st], kABytes + kBBytes);
          tma_load_2d(sA + st * kABytes, &tm_a, &full[st], kb * kBK, mt * kBM);
          tma_load_2d(sB + st * kBBytes, &tm_b, &full[st], kb * kBK, nt * kBN);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      int it = 0, ai = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++ai) {
        const int buf = ai & 1;
        const uint32_t aph = (ai >> 1) & 1;
        if (!mbar_wait(&acce[buf], aph ^ 1)) {
          report(p.ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + buf * kBN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int st = it % kGStages;
          const uint32_t ph = (it / kGStages) & 1;
          if (!mbar_wait(&full[st], ph)) {
            report(p.ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_sw128(sA + st * kABytes);
          const uint64_t bd = smem_desc_sw128(sB + st * kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            tc_mma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) ? 1u : 0u);
          tc_commit(&empty[st]);
        }
        tc_commit(&accf[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------------------ epilogue warps
    const int wq = warp & 3;                 // this warp may read TMEM lanes 32*wq .. 32*wq+31
    int ai = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++ai) {
      const int buf = ai & 1;
      const uint32_t aph = (ai >> 1) & 1;
      if (!mbar_wait(&accf[buf], aph)) {
        report(p.ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
        break;
      }
      tc_fence_after();
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      const int row = wq * 32 + lane;
      const int grow = mt * kBM + row;
      const bool active = grow < p.M;
      const uint32_t tbase = tmem + ((uint32_t)(wq * 32) << 16) + buf * kBN;

      float r0 = -INFINITY, r2 = -INFINITY, r1f = 0.f;
      int r1 = -1, r3 = -1;
      // EPI_LSE extras
      int ct = -1;
      float zc = 0.f;
      bool found = false;
      // EPI_RACE extras
      int g = 0, unode = 0, md = 0;
      float L2 = 0.f;
      const float* qrow = nullptr;
      if (EPI == EPI_LSE && active) ct = p.child_tok[grow];
      if (EPI == EPI_RACE && active) {
        g = p.stop_row[grow];
        unode = p.stop_node[grow];
        md = p.mode[grow];
        L2 = p.lse2[g];
        qrow = p.q_draft + (size_t)g * p.V;
      }

#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        float v[32];
        tmem_ld32(tbase + c * 32, v);
        const int col0 = nt * kBN + c * 32;
        if (!active) continue;
        if (EPI == EPI_ARGMAX) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float x = v[j];
            if (col0 + j < p.V) {
              if (x > r0) {
                r2 = r0;
                r0 = x;
                r1 = col0 + j;
              } else if (x > r2) {
                r2 = x;
              }
            }
          }
        } else if (EPI == EPI_LSE) {
          float cm = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < p.V) cm = fmaxf(cm, v[j] * p.k_log2);
          if (cm > r0) {
            r1f *= exp2f(r0 - cm);
            r0 = cm;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < p.V) r1f += exp2f(v[j] * p.k_log2 - r0);
          if (ct >= col0 && ct < col0 + 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j == ct) zc = v[j];
            found = true;
          }
        } else {  // EPI_RACE
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int cb = col0 + 4 * jj;
            if (cb >= p.V) break;
            float u[4];
            uniforms4(p.seed, p.step, (uint32_t)(cb >> 2), (uint32_t)unode, (uint32_t)grow, 0u,
                      u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int cc = cb + e;
              if (cc < p.V) {
                const float lp2 = v[4 * jj + e] * p.k_log2 - L2;
                const float gum = -logf(-logf(u[e]));
                const float kp = lp2 * 0.69314718055994531f + gum;
                if (kp > r2) {
                  r2 = kp;
                  r3 = cc;
                }
                if (md) {
                  const float w = exp2f(lp2) - __ldg(qrow + cc);
                  if (w > 0.f) {
                    const float kr = logf(w) + gum;
                    if (kr > r0) {
                      r0 = kr;
                      r1 = cc;
                    }
                  }
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
      if (active) {
        float4 out;
        if (EPI == EPI_ARGMAX)
          out = make_float4(r0, __int_as_float(r1), r2, 0.f);
        else if (EPI == EPI_LSE)
          out = make_float4(r0, r1f, 0.f, 0.f);
        else
          out = make_float4(r0, __int_as_float(r1), r2, __int_as_float(r3));
        p.part[(size_t)grow * p.n_tiles + nt] = out;
        if (EPI == EPI_LSE && found) p.zchild[grow] = zc;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

size_t lmhead_smem_bytes() {
  return (size_t)kGStages * (kABytes + kBBytes) + 1024 + (2 * kGStages + 4) * 8 + 16;
}

cudaError_t launch_lmhead(int epi, const CUtensorMap& ta, const CUtensorMap& tb,
                          const GemmParams& p, int grid, cudaStream_t stream) {
  const size_t smem = lmhead_smem_bytes();
  cudaError_t e;
  if (epi == EPI_ARGMAX) {
    auto k = lmhead_gemm_kernel<EPI_ARGMAX>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 192, smem, stream>>>(ta, tb, p);
  } else if (epi == EPI_LSE) {
    auto k = lmhead_gemm_kernel<EPI_LSE>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 192, smem, stream>>>(ta, tb, p);
  } else {
    auto k = lmhead_gemm_kernel<EPI_RACE>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 192, smem, stream>>>(ta, tb, p);
  }
  return cudaGetLastError();
}

}  // namespace etree
