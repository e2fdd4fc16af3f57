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
// so that concurrently running CTAs share W tiles through L2.  Warp 0 streams BMx64 hidden tiles
// (BM = 128, or 64 when all rows fit) and BNx64 W tiles with TMA (128-byte swizzle) into a
// shared-memory ring of as many stages as fit (4 at 128x256, 6 at 64x208); warp 1 issues
// tcgen05.mma (M=BM, N=BN, K=16, bf16 in, fp32 out) into one of two BN-column TMEM accumulators;
// eight epilogue warps drain the other accumulator with tcgen05.ld, one TMEM lane (= one output
// row) per thread, two warps per lane quarter, and apply the epilogue:
//   EPI_ARGMAX  per row and tile: top-1 value, its vocab id (lowest on ties) and top-2 value;
//   EPI_LSE     per row and tile: m = max z*log2(e)/T and sum 2^(z*log2(e)/T - m), plus the
//               logit of the row's child token when it falls in the tile; rows of branching tree
//               nodes also write their logits out (the sibling residuals need whole rows);
//   EPI_TOPK    per row and tile half: the 16 largest values and their ids (the low-rank
//               candidate head's screen, lowrank.cu);
//   EPI_RACE    per row and tile half: the leading entries of two exponential races over the
//               vocabulary (key w_v / E_v, E_v = -log U_v), one over the draw's weights
//               max(0, p - c q) (c = 1 after one rejection, larger c after sibling rejections)
//               and one over p itself (used when c = 0, or when the residual has no positive
//               weight); bonus_kernel takes the largest key over the tiles.
#include "kernels.cuh"
#include "philox.cuh"
#include "race.cuh"

namespace etree {

constexpr int kBK = 64;

// Stage count of the smem ring for a (BM, BN) tile: as many as fit in ~210 KB, at most 6.
__host__ __device__ constexpr int gemm_stages(int bm, int bn) {
  return (210 * 1024) / ((bm + bn) * kBK * 2) < 6 ? (210 * 1024) / ((bm + bn) * kBK * 2) : 6;
}
enum Epi { EPI_ARGMAX = 0, EPI_LSE = 1, EPI_RACE = 2, EPI_TOPK = 3 };

// EPI_TOPK: the 16 largest values seen by one thread, sorted descending (equal values: lower id
// first); empty entries are (-inf, -1).
struct TopK16 {
  float v[16];
  int id[16];
  __device__ __forceinline__ void clear() {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      v[i] = -INFINITY;
      id[i] = -1;
    }
  }
  // Columns arrive in increasing id, so a value equal to the 16th never displaces it.
  __device__ __forceinline__ void insert(float x, int c) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {                  // one compare-exchange pass down the list
      const bool in = x > v[i];
      const float tv = v[i];
      const int tc = id[i];
      v[i] = in ? x : tv;
      id[i] = in ? c : tc;
      x = in ? tv : x;
      c = in ? tc : c;
    }
  }
  // W consecutive columns: the values above the current 16th are staged (in column order) and
  // inserted by one rolled loop, so the insertion code appears once instead of W times.
  // Values below `floor` (a lower bound of the row's k-th largest over the whole vocabulary)
  // cannot be selected and are skipped.
  template <int W>
  __device__ __forceinline__ void push_chunk(const float (&x)[W], int col0, int V, float floor) {
    const float t = v[15];
    bool any = false;
#pragma unroll
    for (int j = 0; j < W; ++j) any |= x[j] > t && x[j] >= floor && col0 + j < V;
    if (!any) return;
    float2 buf[W];
    int n = 0;
#pragma unroll
    for (int j = 0; j < W; ++j)
      if (x[j] > t && x[j] >= floor && col0 + j < V)
        buf[n++] = make_float2(x[j], __int_as_float(col0 + j));
#pragma unroll 1
    for (int i = 0; i < n; ++i)
      if (buf[i].x > v[15]) insert(buf[i].x, __float_as_int(buf[i].y));
  }
};

// Per-row running state of the epilogue over one vocab tile.
struct EpiRow {
  float r0 = -INFINITY, r2 = -INFINITY, r1f = 0.f;   // ARGMAX: top1, top2 | LSE: max, sum
                                                     // RACE: best keys (residual, p)
  int r1 = -1, r3 = -1;                              // ARGMAX: id | RACE: ids (residual, p)
  int ct = -1;                                       // LSE: child token of the row
  float zc = 0.f;                                    // LSE: its logit
  bool found = false;
  int unode = 0, req = 0;                            // RACE: stop node, request
  float c = 0.f;                                     // RACE: residual offset (cval)
  float L2 = 0.f;                                    // RACE: log2 sum 2^(z k)
  float fr = 0.f, fp = 0.f;                          // RACE: the row's published floors
  const float* qrow = nullptr;                       // RACE: q_draft row
};

// The exponential race (race.cuh) over W consecutive ids (col0 a multiple of 8).  The screening
// threshold is the larger of this thread's best key and the floor other threads published for
// the row (keys of real ids, so never above the row's final maximum).
template <int W>
__device__ __forceinline__ void race_chunk(const GemmParams& p, EpiRow& st, const float (&z)[W],
                                           const float (&q)[W], int col0) {
  float thr_p = fmaxf(st.fp, st.r2 > 0.f ? st.r2 : 0.f) * kRaceShrink;
  float thr_r = fmaxf(st.fr, st.r0 > 0.f ? st.r0 : 0.f) * kRaceShrink;
#pragma unroll
  for (int g = 0; g < W / 8; ++g) {
    const int c0 = col0 + 8 * g;
    if (c0 >= p.V) break;
    race8(z + 8 * g, q + 8 * g, c0, p.V, p.k_log2, st.L2, st.c, p.seed, p.step,
          (uint32_t)st.unode, (uint32_t)st.req, thr_r, thr_p, st.r0, st.r1, st.r2, st.r3);
  }
}

// Folds W consecutive logits v (columns col0 .. col0+W-1) into the row state.
template <int EPI, int W>
__device__ __forceinline__ void epi_chunk(const GemmParams& p, EpiRow& st, const float (&v)[W],
                                          int col0) {
  if constexpr (EPI == EPI_ARGMAX) {
#pragma unroll
    for (int j = 0; j < W; ++j) {
      const float x = v[j];
      if (col0 + j < p.V) {
        if (x > st.r0) {
          st.r2 = st.r0;
          st.r0 = x;
          st.r1 = col0 + j;
        } else if (x > st.r2) {
          st.r2 = x;
        }
      }
    }
  } else if constexpr (EPI == EPI_LSE) {
    float cm = -INFINITY;
#pragma unroll
    for (int j = 0; j < W; ++j)
      if (col0 + j < p.V) cm = fmaxf(cm, v[j] * p.k_log2);
    if (cm > st.r0) {
      st.r1f *= exp2f(st.r0 - cm);
      st.r0 = cm;
    }
#pragma unroll
    for (int j = 0; j < W; ++j)
      if (col0 + j < p.V) st.r1f += exp2f(v[j] * p.k_log2 - st.r0);
    if (st.ct >= col0 && st.ct < col0 + W) {
#pragma unroll
      for (int j = 0; j < W; ++j)
        if (col0 + j == st.ct) st.zc = v[j];
      st.found = true;
    }
  }
}

// W consecutive logits of one row to its materialised copy (columns past the vocab dropped).
template <int W>
__device__ __forceinline__ void store_logits(const GemmParams& p, float* zdst, const float (&v)[W],
                                             int col0) {
  if ((p.V & 3) == 0) {
#pragma unroll
    for (int j = 0; j < W; j += 4)
      if (col0 + j < p.V)
        *reinterpret_cast<float4*>(zdst + col0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < W; ++j)
      if (col0 + j < p.V) zdst[col0 + j] = v[j];
  }
}

// Draft probabilities of W consecutive ids (zero past the vocabulary).
template <int W>
__device__ __forceinline__ void load_q(const GemmParams& p, const float* qrow, int col0,
                                       float (&q)[W]) {
  if ((p.V & 3) == 0) {
#pragma unroll
    for (int j = 0; j < W; j += 4) {
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col0 + j < p.V) t = __ldg(reinterpret_cast<const float4*>(qrow + col0 + j));
      q[j] = t.x;
      q[j + 1] = t.y;
      q[j + 2] = t.z;
      q[j + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < W; ++j) q[j] = col0 + j < p.V ? __ldg(qrow + col0 + j) : 0.f;
  }
}

// One 16-column slice of a warp's 32 rows to the materialised logit rows by a TMA store: each
// lane writes its row's 16 values (from v[off ..]) into the warp's staging box in the tensor
// map's 64-byte swizzle (16-byte chunk k of row r sits at chunk k ^ ((r >> 1) & 3)), then lane 0
// stores the box at (col0, row0).  Rows past n_total and columns past the vocabulary lie outside
// the tensor and are not written.  zpend: lane 0 has a store in flight that may still read zbox.
template <int W, int N>
__device__ __forceinline__ void stage_z(const CUtensorMap* tm, float* zbox, const float (&v)[N],
                                        int off, int col0, int row0, int lane, bool& zpend,
                                        int V, int M) {
  static_assert(W == 16, "16-column boxes");
  if (col0 >= V || row0 >= M) return;                 // wholly outside the tensor: nothing to store
  if (lane == 0 && zpend) tma_store_wait_read();
  __syncwarp();
  float4* rowp = reinterpret_cast<float4*>(zbox + lane * 16);
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    rowp[k ^ sw] = make_float4(v[off + 4 * k], v[off + 4 * k + 1], v[off + 4 * k + 2],
                               v[off + 4 * k + 3]);
  fence_proxy_async();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm, zbox, col0, row0);
    tma_store_commit();
    zpend = true;
  }
}

constexpr int kEpiWarps = 8;                 // two warps per TMEM lane quarter
constexpr int kGemmThreads = 32 * (2 + kEpiWarps);

template <int EPI, int BN, int BM>
__global__ void __launch_bounds__(kGemmThreads, 1)
lmhead_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_z, GemmParams p) {
  constexpr int kABytes = BM * kBK * 2;
  constexpr int kBBytes = BN * kBK * 2;
  constexpr int kGStages = gemm_stages(BM, BN);
  constexpr int kBM = BM;
  constexpr bool kZTma = EPI == EPI_LSE && BM == 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kGStages * kBBytes);
  uint64_t* empty = full + kGStages;
  uint64_t* accf = empty + kGStages;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;                // the MMA issuer's last commit, waited on at exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  // EPI_LSE at BM = 128: one 32-row x 16-column fp32 staging box per epilogue warp (64-byte
  // swizzle) for the TMA stores of materialised logit rows, 1024-aligned after the barriers
  float* zstage = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(tmem_slot + 4) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], kEpiWarps);
    }
    mbar_init(drain, 1);
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
  // Everything above overlaps the previous kernel of the stream (launch_pdl); the weight tiles
  // of the first stages are requested before waiting too, since no kernel of the step writes W.
  // No early signal to dependents: the kernels after the GEMM have no set-up to overlap, and an
  // early signal measured slower.
  if (warp != 0) {
    pdl_wait();
    if (p.cnt && blockIdx.x == 0)
      for (int i = threadIdx.x - 32; i < p.cnt_n; i += blockDim.x - 32) p.cnt[i] = 0;
  }

  if (warp == 0) {
    // ----------------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      // W tiles of this CTA's first kGStages k-blocks, each stage armed for its full bytes
      const int pre = blockIdx.x < p.num_tiles ? min(kGStages, p.k_blocks) : 0;
      {
        const int nt0 = blockIdx.x / p.m_tiles;
        for (int kb = 0; kb < pre; ++kb) {
          mbar_arrive_expect_tx(&full[kb], kABytes + kBBytes);
          tma_load_2d(sB + kb * kBBytes, &tm_b, &full[kb], kb * kBK, nt0 * BN);
        }
      }
      pdl_wait();
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int st = it % kGStages;
          const uint32_t ph = (it / kGStages) & 1;
          if (it < pre) {                             // W already requested, stage armed
            tma_load_2d(sA + st * kABytes, &tm_a, &full[st], kb * kBK, mt * kBM);
            continue;
          }
          if (!mbar_wait(&empty[st], ph ^ 1)) {
            report(p.ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[st], kABytes + kBBytes);
          tma_load_2d(sA + st * kABytes, &tm_a, &full[st], kb * kBK, mt * kBM);
          tma_load_2d(sB + st * kBBytes, &tm_b, &full[st], kb * kBK, nt * BN);
        }
      }
      // Before the CTA may exit, the last kGStages loads have landed (earlier ones were
      // consumed, which implies landed).  Bounded, like every wait here.
      bool drained = true;
      for (int j = it > kGStages ? it - kGStages : 0; j < it; ++j)
        drained = mbar_wait(&full[j % kGStages], (j / kGStages) & 1) && drained;
      if (!drained) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN);
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
        const uint32_t d = tmem + buf * BN;
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
      // every MMA issued above completes before TMEM is released
      tc_commit(drain);
      if (!mbar_wait(drain, 0)) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
    }
  } else {
    // ------------------------------------------------------------------------ epilogue warps
    // Warp w reads TMEM lanes 32*(w%4) .. +31 (one output row per thread); the two warps of a
    // lane quarter take alternate 32-column chunks of the tile and write separate summaries.
    const int wq = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int kChunks = BN / 32;
    constexpr int kTailHalf = (kChunks & 1) ? 1 : 0;   // the 16-column tail goes to the half
                                                        // with fewer full chunks
    int ai = 0;
    EpiRow st;
    TopK16 tk;
    tk.clear();
    float* zbox = zstage + (warp - 2) * (32 * 16);    // this warp's staging box
    bool zpend = false;                               // a TMA store from zbox may be reading it
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++ai) {
      const int buf = ai & 1;
      const uint32_t aph = (ai >> 1) & 1;
      if (!mbar_wait(&accf[buf], aph)) {
        report(p.ws, ETREE_ETIMEOUT, DET_WAIT_GEMM);
        break;
      }
      tc_fence_after();
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      // M=128: row r sits in TMEM lane r.  M=64: rows 16q .. 16q+15 sit in the first 16 lanes of
      // lane quarter q, the other 16 lanes of the quarter hold no output.
      const int row = BM == 128 ? wq * 32 + lane : wq * 16 + (lane & 15);
      const int grow = mt * kBM + row;
      const bool active = (BM == 128 || lane < 16) && grow < p.M;
      const uint32_t tbase = tmem + ((uint32_t)(wq * 32) << 16) + buf * BN;

      if (!p.per_cta) {
        st = EpiRow();
        if (EPI == EPI_TOPK) tk.clear();
      }
      // EPI_TOPK: the largest 16th-best published so far by any thread bounds the row's k-th
      float tfloor = -INFINITY;
      if (EPI == EPI_TOPK && active) tfloor = dec_order(__ldcg(p.tkth + grow));
      if (EPI == EPI_LSE && active && p.child_tok) st.ct = p.child_tok[grow];
      const int zr = (EPI == EPI_LSE && active && p.zrow && !p.z_tma) ? p.zrow[grow] : -1;
      float* zdst = zr >= 0 ? p.zbuf + (size_t)zr * p.V : nullptr;
      const int row0 = mt * kBM + wq * 32;            // first row of this warp's TMA boxes
      if (EPI == EPI_RACE && active) {
        const int g = p.stop_row[grow];
        st.unode = p.stop_node[grow];
        st.c = p.cval[grow];
        st.req = grow;
        st.L2 = p.lse2[g];
        st.qrow = p.q_draft + (size_t)g * p.V;
        st.fr = __uint_as_float(__ldcg(p.rfloor + 2 * grow));
        st.fp = __uint_as_float(__ldcg(p.rfloor + 2 * grow + 1));
      }
      {
#pragma unroll 1
        for (int c = half; c < kChunks; c += 2) {
          float v[32];
          tmem_ld32(tbase + c * 32, v);
          if constexpr (EPI == EPI_TOPK) {
            if (active) tk.push_chunk<32>(v, nt * BN + c * 32, p.V, tfloor);
          } else if constexpr (EPI == EPI_RACE) {
            if (active) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {          // two 16-id halves keep registers low
                const int col0 = nt * BN + c * 32 + 16 * hh;
                float q[16];
                if (st.c > 0.f) load_q<16>(p, st.qrow, col0, q);
                race_chunk<16>(p, st, *reinterpret_cast<const float(*)[16]>(v + 16 * hh), q,
                               col0);
              }
            }
          } else {
            if (active) epi_chunk<EPI, 32>(p, st, v, nt * BN + c * 32);
          }
          if constexpr (kZTma) {
            if (p.z_tma) {
              stage_z<16>(&tm_z, zbox, v, 0, nt * BN + c * 32, row0, lane, zpend, p.V, p.M);
              stage_z<16>(&tm_z, zbox, v, 16, nt * BN + c * 32 + 16, row0, lane, zpend, p.V, p.M);
            } else if (zdst) {
              store_logits<32>(p, zdst, v, nt * BN + c * 32);
            }
          } else {
            if (EPI == EPI_LSE && zdst) store_logits<32>(p, zdst, v, nt * BN + c * 32);
          }
        }
        if constexpr (BN % 32 == 16) {
          if (half == kTailHalf) {
            float v[16];
            tmem_ld16(tbase + kChunks * 32, v);
            if constexpr (EPI == EPI_TOPK) {
              if (active) tk.push_chunk<16>(v, nt * BN + kChunks * 32, p.V, tfloor);
            } else if constexpr (EPI == EPI_RACE) {
              if (active) {
                float q[16];
                if (st.c > 0.f) load_q<16>(p, st.qrow, nt * BN + kChunks * 32, q);
                race_chunk<16>(p, st, v, q, nt * BN + kChunks * 32);
              }
            } else {
              if (active) epi_chunk<EPI, 16>(p, st, v, nt * BN + kChunks * 32);
            }
            if constexpr (kZTma) {
              if (p.z_tma)
                stage_z<16>(&tm_z, zbox, v, 0, nt * BN + kChunks * 32, row0, lane, zpend, p.V, p.M);
              else if (zdst)
                store_logits<16>(p, zdst, v, nt * BN + kChunks * 32);
            } else {
              if (EPI == EPI_LSE && zdst) store_logits<16>(p, zdst, v, nt * BN + kChunks * 32);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
      // per_cta: the row state runs on over this CTA's tiles (increasing ids, so first-seen
      // still means lowest id) and is written once, after the CTA's last tile.
      if (EPI == EPI_TOPK && active && tk.v[15] > tfloor)   // 16 values >= it: a valid bound
        atomicMax(p.tkth + grow, enc_order(tk.v[15]));
      if (EPI == EPI_RACE && active) {                  // positive keys order as their bits
        if (st.r1 >= 0 && st.r0 > st.fr) atomicMax(p.rfloor + 2 * grow, __float_as_uint(st.r0));
        if (st.r3 >= 0 && st.r2 > st.fp) atomicMax(p.rfloor + 2 * grow + 1, __float_as_uint(st.r2));
      }
      if (EPI == EPI_TOPK && active && (!p.per_cta || tile + (int)gridDim.x >= p.num_tiles)) {
        float2* dst = p.topk + ((size_t)grow * p.n_parts * 2 +
                                (p.per_cta ? (int)blockIdx.x : nt) * 2 + half) * 16;
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[i] = make_float2(tk.v[i], __int_as_float(tk.id[i]));
      }
      if (EPI != EPI_TOPK && active && (!p.per_cta || tile + (int)gridDim.x >= p.num_tiles)) {
        float4 out;
        if (EPI == EPI_ARGMAX)
          out = make_float4(st.r0, __int_as_float(st.r1), st.r2, 0.f);
        else if (EPI == EPI_LSE)
          out = make_float4(st.r0, st.r1f, 0.f, 0.f);
        else                                            // RACE: (key, id) residual, p
          out = make_float4(st.r0, __int_as_float(st.r1), st.r2, __int_as_float(st.r3));
        p.part[(size_t)grow * p.n_parts * 2 + (p.per_cta ? (int)blockIdx.x : nt) * 2 + half] = out;
        if (EPI == EPI_LSE && st.found) p.zchild[grow] = st.zc;
      }
    }
    // the materialised rows' TMA stores complete before the CTA exits
    if (kZTma && lane == 0 && zpend) tma_store_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Vocab-tile widths with a kernel instantiation.  Each is a multiple of 16 (the M=128 MMA's N
// granularity) and fits two accumulators in the 512 TMEM columns.
static const int kWidths[] = {256, 224, 208, 192, 176, 160, 144, 128};

int lmhead_pick_bn(int M, int V, int grid) {
  // With several row tiles the GEMM is tensor-bound and the widest tile is the most efficient.
  // With one row tile it streams W once: time ~ (rounds of tiles per CTA) x (tile width + a
  // fixed per-tile cost of ~48 columns), so pick the width that balances the last round.
  const long m_tiles = (M + 127) / 128;
  if (m_tiles >= 2) return 256;
  int best = 256;
  long best_cost = -1;
  for (int bn : kWidths) {
    const long tiles = m_tiles * ((V + bn - 1) / bn);
    const long rounds = (tiles + grid - 1) / grid;
    const long cost = rounds * (bn + 48);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

template <int EPI, int BM>
static size_t lmhead_smem_bytes(int bn) {
  const size_t base = (size_t)gemm_stages(BM, bn) * (BM + bn) * kBK * 2 + 1024 + (2 * 6 + 5) * 8 + 16;
  // EPI_LSE at BM = 128: 1 KB of alignment and eight 2 KB staging boxes for the TMA stores
  return (EPI == EPI_LSE && BM == 128) ? base + 1024 + kEpiWarps * 32 * 16 * 4 : base;
}

template <int EPI, int BN, int BM>
static cudaError_t launch_bn(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tz,
                             const GemmParams& p, int grid, cudaStream_t stream) {
  const size_t smem = lmhead_smem_bytes<EPI, BM>(BN);
  auto k = lmhead_gemm_kernel<EPI, BN, BM>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), dim3(kGemmThreads), smem, stream, ta, tb, tz, p);
}

template <int EPI, int BM>
static cudaError_t launch_epi(int bn, const CUtensorMap& ta, const CUtensorMap& tb,
                              const CUtensorMap& tz, const GemmParams& p, int grid,
                              cudaStream_t s) {
  switch (bn) {
    case 256: return launch_bn<EPI, 256, BM>(ta, tb, tz, p, grid, s);
    case 224: return launch_bn<EPI, 224, BM>(ta, tb, tz, p, grid, s);
    case 208: return launch_bn<EPI, 208, BM>(ta, tb, tz, p, grid, s);
    case 192: return launch_bn<EPI, 192, BM>(ta, tb, tz, p, grid, s);
    case 176: return launch_bn<EPI, 176, BM>(ta, tb, tz, p, grid, s);
    case 160: return launch_bn<EPI, 160, BM>(ta, tb, tz, p, grid, s);
    case 144: return launch_bn<EPI, 144, BM>(ta, tb, tz, p, grid, s);
    case 128: return launch_bn<EPI, 128, BM>(ta, tb, tz, p, grid, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_lmhead(int epi, int bn, int bm, const CUtensorMap& ta, const CUtensorMap& tb,
                          const CUtensorMap& tz, const GemmParams& p, int grid,
                          cudaStream_t stream) {
  if (epi == EPI_TOPK)
    return bm == 64 ? launch_epi<EPI_TOPK, 64>(bn, ta, tb, tz, p, grid, stream)
                    : launch_epi<EPI_TOPK, 128>(bn, ta, tb, tz, p, grid, stream);
  if (bm == 64) {
    if (epi == EPI_ARGMAX) return launch_epi<EPI_ARGMAX, 64>(bn, ta, tb, tz, p, grid, stream);
    if (epi == EPI_LSE) return launch_epi<EPI_LSE, 64>(bn, ta, tb, tz, p, grid, stream);
    return launch_epi<EPI_RACE, 64>(bn, ta, tb, tz, p, grid, stream);
  }
  if (epi == EPI_ARGMAX) return launch_epi<EPI_ARGMAX, 128>(bn, ta, tb, tz, p, grid, stream);
  if (epi == EPI_LSE) return launch_epi<EPI_LSE, 128>(bn, ta, tb, tz, p, grid, stream);
  return launch_epi<EPI_RACE, 128>(bn, ta, tb, tz, p, grid, stream);
}

}  // namespace etree
