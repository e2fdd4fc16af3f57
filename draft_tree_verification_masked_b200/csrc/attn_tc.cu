// attn_tc.cu -- tree-masked GQA attention on tcgen05 / TMEM (sm_100a).
//
// Every tree node attends to its request's cached keys and to its tree ancestors and itself: the
// target verifies all drafted tokens in one parallel forward, and a draft tree lets one
// verification cover several candidate paths ("Eagle-4 Released: Outpaces DFlash2 and DSpark
// ...", section "Technical Background").  Single-request decoding moves data rather than
// computing ("EAGLE-4 是什麼？...", aiposthub.com, opening section), so each KV byte is read from
// HBM once for all tree nodes and all query heads of a KV-head group.  Both matrix products run
// on the 5th-generation tensor cores:
//
//   S  = Q K^T   tcgen05.mma M=128 (query rows) x N=KEYS x K=128, fp32 into TMEM;
//   O += P V     tcgen05.mma M=128 x N=128 (head dims) x K=KEYS, fp32 accumulated in TMEM.
//
// One CTA = (request, KV head, 128-row block, KV split).  The query rows are the (node, group
// head) pairs of one KV head, row = node * G + g; one TMA box {64 dims, G heads, NB nodes} of the
// [n_total][hq][128] query tensor lands them in exactly that order (NB = floor(128 / G)).
// Warp 0 streams Q once and the KEYS-key K/V tiles through a STAGES-deep ring; warp 1 issues the
// MMAs; four softmax warps own one query row per thread (= one TMEM lane, all of the tile's keys;
// the kernel also supports SW = 8, two warps per row exchanging row maxima): they read S from TMEM, apply
// the key mask (cache length, or the row's ancestor bitmask on the tree tiles), run the online
// softmax in log2 units, and write P (bf16) back into their own TMEM lane, where the PV product
// takes it as its A operand; shared memory holds only Q and the K/V ring.  S and P have three
// buffers each in the 64-key shape (QK^T issued two tiles ahead of PV) and two in the 32-key
// shape (one tile ahead), so the tensor core works on later tiles while the softmax runs.  O is rescaled
// lazily: only when a row's running maximum grows by more than 2^8 does the softmax
// read-modify-write O in TMEM, so P stays below 256 and the usual case has no O traffic.
//
// Two shapes are built.  KEYS = 64 with a 5-deep ring runs one CTA per SM (for few, long
// work items).  KEYS = 32 with a 4-deep ring fits two CTAs per SM, which overlaps one CTA's
// start-up and tail with the other's streaming; its Q rows are rotated into a different TMEM
// lane quarter per CTA so that co-resident CTAs run their softmax on different SM partitions.
#include "kernels.cuh"

namespace etree {

namespace {
constexpr int kQBytes = 2 * 16384;          // Q lo/hi boxes of [128 rows][64 dims]
constexpr float kLazy = 8.0f;               // rescale O only when the max grows by > 2^8

struct TcSmem {
  // barriers and small arrays, placed after the 1024-aligned tile area
  uint64_t kv_full[6], kv_empty[6], q_full, s_full[3], s_free[3], p_full[3], p_free[3];
  uint64_t drain;                           // the MMA issuer's last commit, waited on at exit
  uint64_t anc[64];
  int32_t par[64];
  float xmax[2][4][128];                    // row-max exchange: [tile parity][key part][row]
  float xl[4][128];                         // final row sums of the key parts
  uint64_t xbar[4][2], xlbar[4];            // exchange barriers per lane quarter (bounded waits)
  uint32_t tmem;
};

template <int KEYS>
struct TcShape {
  static constexpr int kBox = KEYS * 128;   // one [KEYS keys][64 dims] bf16 box
  static constexpr int kKV = 4 * kBox;      // K lo/hi + V lo/hi
  // kNS S buffers (fp32, KEYS columns each) at [0, kNS KEYS), O (128 columns) at kOCol, kNP P
  // buffers (bf16 pairs, KEYS / 2 columns each) at kPCol.  QK^T runs kLag tiles ahead of PV.
  // 64 keys: S [0, 192), O [256, 384), P [384, 480) of 512 columns; 32 keys (two CTAs per SM):
  // S [0, 64), P [64, 96), O [128, 256) of 256 columns.  (Measured on the 32-key shape, a third
  // S buffer with a two-tile lead was slower.)
  static constexpr int kNS = KEYS == 64 ? 3 : 2;
  static constexpr int kNP = KEYS == 64 ? 3 : 2;
  static constexpr int kLag = kNS - 1;
  static constexpr int kOCol = KEYS == 64 ? 256 : 128;
  static constexpr int kPCol = KEYS == 64 ? 384 : 64;
  static constexpr int kTmemCols = KEYS == 64 ? 512 : 256;
  static_assert(kNS * KEYS <= kPCol && kNS * KEYS <= kOCol, "S overlaps P or O");
  static_assert(kPCol + kNP * KEYS / 2 <= kOCol || kOCol + 128 <= kPCol, "P overlaps O");
  static_assert(kPCol + kNP * KEYS / 2 <= kTmemCols && kOCol + 128 <= kTmemCols, "TMEM");
};
}  // namespace

template <int KEYS, int STAGES, int SW>
__global__ void __launch_bounds__(32 * (2 + SW), KEYS == 32 ? 2 : 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
               const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kt,
               const __grid_constant__ CUtensorMap tm_vt, AttnParams p, int NB) {
  using Sh = TcShape<KEYS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                                   // 32 KB
  uint8_t* sKV = smem + kQBytes;                        // STAGES x kKV
  TcSmem* sh = reinterpret_cast<TcSmem*>(sKV + STAGES * Sh::kKV);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_req = p.hkv * p.mchunks;
  const int r = p.order ? p.order[blockIdx.x / per_req] : blockIdx.x / per_req;
  const int kvh = (blockIdx.x % per_req) / p.mchunks;
  const int mb = blockIdx.x % p.mchunks;
  const int s = blockIdx.y;
  const int G = p.G;

  const int base = p.cu_nodes[r];
  const int n = p.cu_nodes[r + 1] - base;
  const int L = p.kv_len[r];
  const int64_t sbase = p.slot_base[r];
  const bool paged = p.block_table != nullptr;
  if (n < 1 || n > p.n_max || L < 0 || L > p.kv_len_max ||
      (!paged && (sbase < 0 || sbase + L > p.cache_slots)) ||
      (paged && L > ((int64_t)p.max_pages << p.page_shift))) {
    if (threadIdx.x == 0 && s == 0 && mb == 0 && kvh == 0)
      report(p.ws, ETREE_EDEVICE, (n < 1 || n > p.n_max) ? DET_BAD_NODES : DET_KV_LEN);
    return;
  }
  const int node0 = mb * NB;
  if (node0 >= n) return;
  const int nt_cache = (L + KEYS - 1) / KEYS;
  const int total = nt_cache + (n + KEYS - 1) / KEYS;   // the tree tiles come last
  const int t0 = s * p.tps;
  const int t1 = min(total, t0 + p.tps);
  if (t0 >= t1) return;
  const int T = t1 - t0;
  const bool has_tree = (t1 > nt_cache);
  const int qrows = NB * G;                             // rows the Q box fills
  // lane quarter rotation of the Q rows (see the header)
  int rot = 0;
  if (KEYS == 32) {
    if (qrows <= 32) rot = 32 * (blockIdx.x & 3);
    else if (qrows <= 64) rot = 64 * (blockIdx.x & 1);
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&sh->kv_full[i], 1);
      mbar_init(&sh->kv_empty[i], 1);
    }
    mbar_init(&sh->q_full, 1);
    mbar_init(&sh->drain, 1);
    for (int b = 0; b < 3; ++b) {
      mbar_init(&sh->s_full[b], 1);
      mbar_init(&sh->s_free[b], SW);
      mbar_init(&sh->p_full[b], SW);
      mbar_init(&sh->p_free[b], 1);
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(&sh->xbar[q][0], SW / 4);
      mbar_init(&sh->xbar[q][1], SW / 4);
      mbar_init(&sh->xlbar[q], SW / 4);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem, Sh::kTmemCols);
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
  // rows outside the Q box are zero so that their (unused) products stay finite
  for (int i = threadIdx.x; i < 128 * 16; i += blockDim.x) {
    const int row = i / 16, c = i % 16;
    if (row >= rot && row < rot + qrows) continue;
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
      tma_load_3d(sQ + rot * 128, &tm_q, &sh->q_full, 0, kvh * G, base + node0);
      tma_load_3d(sQ + 16384 + rot * 128, &tm_q, &sh->q_full, 64, kvh * G, base + node0);
      int issued = 0;
      // paged: the page entries of tile j + 1 are fetched while tile j's slot is awaited
      const int nbox = paged ? KEYS / p.cache_box : 0;
      const int32_t* bt = paged ? p.block_table + (size_t)r * p.max_pages : nullptr;
      int32_t pg_cur[4], pg_nxt[4];
      auto fetch_pages = [&](int t, int32_t (&dst)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pi = (t * KEYS + i * p.cache_box) >> p.page_shift;
          dst[i] = (i < nbox && t < nt_cache && pi < p.max_pages) ? __ldg(bt + pi) : -1;
        }
      };
      if (paged) fetch_pages(t0, pg_cur);
      for (int j = 0; j < T; ++j) {
        const int t = t0 + j;
        const int st = j % STAGES;
        const uint32_t ph = (j / STAGES) & 1;
        if (paged) fetch_pages(t + 1, pg_nxt);
        if (j >= STAGES && !mbar_wait(&sh->kv_empty[st], ph ^ 1)) {
          report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
          break;
        }
        uint8_t* dst = sKV + st * Sh::kKV;
        mbar_arrive_expect_tx(&sh->kv_full[st], Sh::kKV);
        if (t < nt_cache && !paged) {
          const int32_t slot = static_cast<int32_t>(sbase + (int64_t)t * KEYS);
          tma_load_3d(dst, &tm_kc, &sh->kv_full[st], 0, kvh, slot);
          tma_load_3d(dst + Sh::kBox, &tm_kc, &sh->kv_full[st], 64, kvh, slot);
          tma_load_3d(dst + 2 * Sh::kBox, &tm_vc, &sh->kv_full[st], 0, kvh, slot);
          tma_load_3d(dst + 3 * Sh::kBox, &tm_vc, &sh->kv_full[st], 64, kvh, slot);
        } else if (t < nt_cache) {
          // paged: KEYS / cache_box boxes per half, each inside one page.  An entry outside
          // the pool is reported; its box then lies past the tensor and TMA fills zeros.
          const int cb = p.cache_box, P = 1 << p.page_shift;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (i >= nbox) break;
            const int pos = t * KEYS + i * cb;
            int32_t page = pg_cur[i];
            if (page < 0 || (int64_t)page * P >= p.cache_slots) {
              if (pos < L) report(p.ws, ETREE_EDEVICE, DET_BAD_PAGE);
              page = (int32_t)(p.cache_slots >> p.page_shift);
            }
            const int32_t slot = page * P + (pos & (P - 1));
            const uint32_t off = (uint32_t)(i * cb * 128);
            tma_load_3d(dst + off, &tm_kc, &sh->kv_full[st], 0, kvh, slot);
            tma_load_3d(dst + Sh::kBox + off, &tm_kc, &sh->kv_full[st], 64, kvh, slot);
            tma_load_3d(dst + 2 * Sh::kBox + off, &tm_vc, &sh->kv_full[st], 0, kvh, slot);
            tma_load_3d(dst + 3 * Sh::kBox + off, &tm_vc, &sh->kv_full[st], 64, kvh, slot);
          }
        } else {
          const int node = base + (t - nt_cache) * KEYS;
          tma_load_3d(dst, &tm_kt, &sh->kv_full[st], 0, kvh, node);
          tma_load_3d(dst + Sh::kBox, &tm_kt, &sh->kv_full[st], 64, kvh, node);
          tma_load_3d(dst + 2 * Sh::kBox, &tm_vt, &sh->kv_full[st], 0, kvh, node);
          tma_load_3d(dst + 3 * Sh::kBox, &tm_vt, &sh->kv_full[st], 64, kvh, node);
        }
        if (paged) {
#pragma unroll
          for (int i = 0; i < 4; ++i) pg_cur[i] = pg_nxt[i];
        }
        issued = j + 1;
      }
      // Before the CTA may exit, every copy into shared memory has landed: the last STAGES
      // loads (earlier ones were consumed, which implies landed) and Q.  Bounded, like all waits.
      bool drained = mbar_wait(&sh->q_full, 0);
      for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j)
        drained = mbar_wait(&sh->kv_full[j % STAGES], (j / STAGES) & 1) && drained;
      if (!drained) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, KEYS);
      const uint32_t idO = idesc_bf16_f32(128, 128) | (1u << 16);   // B (V) is MN-major
      bool ok = mbar_wait(&sh->q_full, 0);
      tc_fence_after();
      const uint64_t dq0 = smem_desc_sw128(sQ), dq1 = smem_desc_sw128(sQ + 16384);
      auto pv = [&](int jj) -> bool {
        const int pb = jj % Sh::kNP;
        if (!mbar_wait(&sh->p_full[pb], (jj / Sh::kNP) & 1)) return false;
        tc_fence_after();
        // A = P from TMEM (16 keys = 8 columns per MMA), B = V from shared memory
        const uint32_t pa = tmem + Sh::kPCol + pb * (KEYS / 2);
        const uint8_t* v0 = sKV + (jj % STAGES) * Sh::kKV + 2 * Sh::kBox;
#pragma unroll
        for (int k = 0; k < KEYS / 16; ++k)
          tc_mma_bf16_ts(tmem + Sh::kOCol, pa + 8 * k, smem_desc_sw128_mn(v0 + k * 2048, Sh::kBox), idO,
                         (jj > 0 || k > 0) ? 1u : 0u);
        tc_commit(&sh->p_free[pb]);
        tc_commit(&sh->kv_empty[jj % STAGES]);
        return true;
      };
      // QK^T of tile j is issued before PV of tile j - kLag, so the softmax finds the next
      // kLag score tiles computed while it works on one
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % STAGES;
        const int sb = j % Sh::kNS;
        if (!mbar_wait(&sh->kv_full[st], (j / STAGES) & 1)) { ok = false; break; }
        if (j >= Sh::kNS && !mbar_wait(&sh->s_free[sb], ((j / Sh::kNS) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* k0 = sKV + st * Sh::kKV;
        const uint64_t dk0 = smem_desc_sw128(k0), dk1 = smem_desc_sw128(k0 + Sh::kBox);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc_mma_bf16(tmem + sb * KEYS, (k < 4 ? dq0 : dq1) + 2 * (k & 3),
                      (k < 4 ? dk0 : dk1) + 2 * (k & 3), idS, k > 0 ? 1u : 0u);
        tc_commit(&sh->s_full[sb]);
        if (j >= Sh::kLag && !pv(j - Sh::kLag)) { ok = false; break; }
      }
      for (int jj = T > Sh::kLag ? T - Sh::kLag : 0; ok && jj < T; ++jj)
        if (!pv(jj)) ok = false;
      // every MMA issued above completes before TMEM is released
      tc_commit(&sh->drain);
      if (!mbar_wait(&sh->drain, 0)) ok = false;
      if (!ok) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
    }
  } else {
    // ------------------------------------------------------------------- softmax warps
    // SW/4 warps per TMEM lane quarter; key part `kh` of a quarter owns keys
    // [kh*CW, kh*CW + CW) of every tile (CW = KEYS / (SW/4)) and O columns [kh*OW, kh*OW + OW).
    constexpr int NH = SW / 4;
    constexpr int CW = KEYS / NH;
    constexpr int OW = 128 / NH;
    const int wq = warp & 3;
    const int kh = (warp - 2) >> 2;
    const int row = wq * 32 + lane;
    const int lrow = row - rot;
    const bool inbox = lrow >= 0 && lrow < qrows;
    const int node_l = inbox ? lrow / G : 0, g = inbox ? lrow - node_l * G : 0;
    const int node = node0 + node_l;
    const bool valid = inbox && node < n;
    const uint64_t anc = (has_tree && valid) ? sh->anc[node] : 0ull;
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int t = t0 + j;
      const int sb = j % Sh::kNS;
      if (!mbar_wait(&sh->s_full[sb], (j / Sh::kNS) & 1)) { ok = false; break; }
      tc_fence_after();
      float sc[CW];
      if constexpr (CW == 64) {
        tmem_ld32(lane_base + sb * KEYS, *reinterpret_cast<float(*)[32]>(sc));
        tmem_ld32(lane_base + sb * KEYS + 32, *reinterpret_cast<float(*)[32]>(sc + 32));
      } else if constexpr (CW == 32) {
        tmem_ld32(lane_base + sb * KEYS + kh * CW, sc);
      } else {
        tmem_ld16(lane_base + sb * KEYS + kh * CW, sc);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->s_free[sb]);

      // Key mask.  Whole cache tiles below kv_len keep every key (the common case, tested once
      // per tile for the CTA); the last cache tile masks by kv_len and tree tiles by the row's
      // ancestor bits.  Scores stay raw here: the scale (> 0) is folded into the exponent.
      const int k0 = kh * CW;                           // first key of this thread in the tile
      const bool full_tile = t < nt_cache && L - t * KEYS >= KEYS;
      if (!full_tile) {
        uint64_t kw;                                    // bit c: key k0 + c is visible
        if (!valid) {
          kw = 0ull;
        } else if (t >= nt_cache) {
          const int sh0 = (t - nt_cache) * KEYS + k0;   // < 64: tree tiles start at node 0
          kw = anc >> sh0;
        } else {
          const int lim = L - t * KEYS - k0;
          kw = lim >= 64 ? ~0ull : (lim > 0 ? ((1ull << lim) - 1ull) : 0ull);
        }
#pragma unroll
        for (int c = 0; c < CW; ++c)
          if (!((kw >> c) & 1ull)) sc[c] = -INFINITY;
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < CW; c += 4) {
        mx0 = fmax3(mx0, sc[c], sc[c + 1]);
        mx1 = fmax3(mx1, sc[c + 2], sc[c + 3]);
      }
      float tmax = fmaxf(mx0, mx1);
      const float sl = p.scale_log2;
      // P = 2^(s * scale_log2 - off) for this thread's keys, packed to bf16, with its row sum.
      float ls0, ls1;
      uint32_t pk[CW / 2];
      auto exps = [&](float off) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int c = 0; c < CW / 2; c += 2) {
          float x0, x1, x2, x3;
          ffma2(x0, x1, sc[2 * c], sc[2 * c + 1], sl, -off);
          ffma2(x2, x3, sc[2 * c + 2], sc[2 * c + 3], sl, -off);
          const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
          const float e2 = ex2_approx(x2), e3 = ex2_approx(x3);
          fadd2(a0, a1, e0, e1);
          fadd2(a0, a1, e2, e3);
          pk[c] = pack_bf16x2(e0, e1);
          pk[c + 1] = pack_bf16x2(e2, e3);
        }
        ls0 = a0;
        ls1 = a1;
      };
      // With NH warps per row the row maximum needs the other warps' key parts.  A row that
      // already has a reference computes P against it while those maxima are in flight, and
      // recomputes only when the combined maximum moves the reference (rare: see kLazy).
      if constexpr (NH > 1) {
        sh->xmax[j & 1][kh][row] = tmax;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->xbar[wq][j & 1]);
      }
      const bool early = NH > 1 && __all_sync(0xffffffffu, m_ref != -INFINITY);
      if (early) exps(m_ref);
      if constexpr (NH > 1) {
        if (!mbar_wait(&sh->xbar[wq][j & 1], (j >> 1) & 1)) { ok = false; break; }
#pragma unroll
        for (int h = 1; h < NH; ++h) tmax = fmaxf(tmax, sh->xmax[j & 1][kh ^ h][row]);
      }
      const float tms = tmax * sl;                      // row maximum in log2 units
      const bool need = tms > m_ref + kLazy;            // also true for the first finite max
      const bool any = __any_sync(0xffffffffu, need);
      const float m_new = need ? tms : m_ref;
      if (!early || need) exps(m_new == -INFINITY ? 0.f : m_new);
      const float corr = need ? ex2_approx(m_ref - m_new) : 1.f;
      l = l * corr + (ls0 + ls1);
      m_ref = m_new;
      // A rescale of O needs every earlier PV product finished (the last one wrote O).
      if (any && j >= 1) {
        if (!mbar_wait(&sh->p_free[(j - 1) % Sh::kNP], ((j - 1) / Sh::kNP) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < OW / 32; ++c) {
          float o[32];
          const uint32_t ta = lane_base + Sh::kOCol + kh * OW + c * 32;
          tmem_ld32(ta, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= corr;
          tmem_st32(ta, o);
        }
      }
      // P buffer j % kNP is free once PV(j - kNP) has completed
      const int pb = j % Sh::kNP;
      if (j >= Sh::kNP) {
        if (!mbar_wait(&sh->p_free[pb], ((j / Sh::kNP) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
      }
      // this thread's CW keys of P into its own TMEM lane (the PV product's A operand)
      static_assert(CW == 64 || CW == 32 || CW == 16, "a 32-, 16- or 8-column P store");
      if constexpr (CW == 64) {
        float pf[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pf[c] = __uint_as_float(pk[c]);
        tmem_st32(lane_base + Sh::kPCol + pb * (KEYS / 2), pf);
      } else if constexpr (CW == 32) {
        tmem_st16(lane_base + Sh::kPCol + pb * (KEYS / 2) + kh * (CW / 2), pk);
      } else {
        tmem_st8(lane_base + Sh::kPCol + pb * (KEYS / 2) + kh * (CW / 2), pk);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->p_full[pb]);
    }
    if (ok && !mbar_wait(&sh->p_free[(T - 1) % Sh::kNP], ((T - 1) / Sh::kNP) & 1)) ok = false;
    if (!ok) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
    if constexpr (NH > 1) {                             // the row sum covers every key part
      sh->xl[kh][row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->xlbar[wq]);
      if (!mbar_wait(&sh->xlbar[wq], 0)) report(p.ws, ETREE_ETIMEOUT, DET_WAIT_ATTN);
      l = 0.f;
#pragma unroll
      for (int h = 0; h < NH; ++h) l += sh->xl[h][row];
    }
    tc_fence_after();
    const size_t gidx = (size_t)(base + (valid ? node : 0)) * p.hq + kvh * G + g;
    if (p.nsplit == 1) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < OW / 32; ++c) {
        const int col = kh * OW + c * 32;
        float o[32];
        tmem_ld32(lane_base + Sh::kOCol + col, o);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + gidx * 128 + col);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                                pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
        }
      }
      if (valid && kh == 0 && p.lse) p.lse[gidx] = (m_ref + log2f(l)) * 0.69314718055994531f;
    } else {
      float* op = p.o_part + (gidx * p.nsplit + s) * 128;
#pragma unroll 1
      for (int c = 0; c < OW / 32; ++c) {
        const int col = kh * OW + c * 32;
        float o[32];
        tmem_ld32(lane_base + Sh::kOCol + col, o);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(op + col);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
      }
      if (valid && kh == 0) p.ml_part[gidx * p.nsplit + s] = make_float2(m_ref, l);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Sh::kTmemCols);
  }
}

template <int KEYS, int STAGES, int SW>
static cudaError_t launch_shape(const CUtensorMap& q, const CUtensorMap& kc, const CUtensorMap& vc,
                                const CUtensorMap& kt, const CUtensorMap& vt, const AttnParams& p,
                                int nb, cudaStream_t stream) {
  using Sh = TcShape<KEYS>;
  const size_t smem = 1024 + kQBytes + (size_t)STAGES * Sh::kKV + sizeof(TcSmem);
  auto k = attn_tc_kernel<KEYS, STAGES, SW>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.B * p.hkv * p.mchunks, p.nsplit);
  k<<<grid, 32 * (2 + SW), smem, stream>>>(q, kc, vc, kt, vt, p, nb);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const CUtensorMap& q, const CUtensorMap& kc, const CUtensorMap& vc,
                           const CUtensorMap& kt, const CUtensorMap& vt, const AttnParams& p,
                           int nb, int n_total, cudaStream_t stream) {
  cudaError_t e = p.keys == 32 ? launch_shape<32, 4, 4>(q, kc, vc, kt, vt, p, nb, stream)
                               : launch_shape<64, 5, 4>(q, kc, vc, kt, vt, p, nb, stream);
  if (e != cudaSuccess || p.nsplit == 1) return e;
  return launch_attn_combine(p, n_total, stream);
}

}  // namespace etree
