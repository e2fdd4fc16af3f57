// api.cu -- the C ABI of libetree: argument validation, workspace layout, TMA descriptors and
// launch planning for the three verification calls.  Every step of the computation runs in the
// kernels of attn_tc.cu, attn_combine.cu, lmhead.cu, accept.cu and compact.cu; this file only plans and
// enqueues them.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include <cstdarg>

#include "kernels.cuh"

namespace etree {

// ------------------------------------------------------------------------------- error text
static thread_local char g_err[512] = "";

static etree_status fail(etree_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

static etree_status cuda_fail(cudaError_t e, const char* where) {
  return fail(ETREE_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

// ------------------------------------------------------------------------------- device info
static int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// ------------------------------------------------------------------------------ attention plan
struct AttnPlan {
  int G, keys, nb, mchunks, nsplit, tps;
};

// Launch plan of the attention call.  The tcgen05 kernel takes 128-row blocks of
// nb = min(floor(128 / G), n_max) whole nodes; with at least one (request, KV head, row block)
// per SM, or 64K or more cached keys, it uses 32-key tiles and two CTAs per SM, otherwise 64-key
// tiles and one CTA per SM.  The KV range is split only to fill one wave of CTAs (a second,
// partial wave costs more than longer splits), keeping >= 4 key tiles per split.
static AttnPlan plan_attn(const etree_batch* b, int hq, int hkv) {
  AttnPlan pl{};
  pl.G = hq / hkv;
  const int sms = sm_count();
  pl.nb = std::min(128 / pl.G, b->n_max);             // nodes per Q box (row block)
  pl.mchunks = (b->n_max + pl.nb - 1) / pl.nb;
  const int pairs = b->B * hkv * pl.mchunks;
  // 32-key tiles (two CTAs per SM) pay off once there is at least one row block per SM, and on
  // very long contexts (>= 64K keys: measured 5-8% faster at 128K, 5% slower at 32K); otherwise
  // few, long work items prefer 64-key tiles split over the SMs
  pl.keys = (pairs >= sms || b->kv_len_max >= 65536) ? 32 : 64;
  const int tiles_max =
      (b->kv_len_max + pl.keys - 1) / pl.keys + (b->n_max + pl.keys - 1) / pl.keys;
  const int per_sm = pl.keys == 32 ? 2 : 1;
  int nsplit = std::max(1, per_sm * sms / pairs);
  nsplit = std::min(nsplit, std::max(1, tiles_max / 4));
  nsplit = std::max(1, std::min(nsplit, tiles_max));
  pl.tps = (tiles_max + nsplit - 1) / nsplit;
  pl.nsplit = (tiles_max + pl.tps - 1) / pl.tps;
  return pl;
}

// ------------------------------------------------------------------------------ workspace map
struct WsLayout {
  size_t order, o_part, ml_part, part, child_tok, zchild, lse2, stop_row, stop_node, cval, hid2,
      part2, rfloor, cnt, ccount, zrow, zc;
  size_t total;
  int n_tiles;
};

static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

static WsLayout layout(const etree_batch* b, int hq, int hkv, int hidden_dim, int vocab) {
  WsLayout w{};
  size_t off = sizeof(WsHeader);
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  const size_t nt = (size_t)std::max(0, b->n_total);
  const size_t B = (size_t)std::max(0, b->B);
  size_t nsplit = 1;
  if (hq > 0 && hkv > 0 && hq % hkv == 0) nsplit = (size_t)plan_attn(b, hq, hkv).nsplit;
  const size_t rows = nt * (size_t)std::max(0, hq);
  w.order = take(hq > 0 ? B * sizeof(int32_t) : 0);
  w.o_part = take(nsplit > 1 ? rows * nsplit * 128 * sizeof(float) : 0);
  w.ml_part = take(nsplit > 1 ? rows * nsplit * sizeof(float2) : 0);
  // two summaries per vocab tile, at the narrowest tile width the LM head may pick (128)
  w.n_tiles = vocab > 0 ? 2 * ((vocab + 127) / 128) : 0;
  w.part = take(nt * (size_t)w.n_tiles * sizeof(float4));
  w.child_tok = take(nt * sizeof(int32_t));
  w.zchild = take(nt * sizeof(float));
  w.lse2 = take(nt * sizeof(float));
  w.stop_row = take(B * sizeof(int32_t));
  w.stop_node = take(B * sizeof(int32_t));
  w.cval = take(B * sizeof(float));
  w.hid2 = take(B * (size_t)std::max(0, hidden_dim) * 2);
  w.part2 = take(B * (size_t)w.n_tiles * sizeof(float4));
  w.rfloor = take(B * 2 * sizeof(uint32_t));
  w.cnt = take(B * sizeof(int32_t));
  w.ccount = take(nt * sizeof(int32_t));
  w.zrow = take(nt * sizeof(int32_t));
  w.zc = take(nt * sizeof(float));
  w.total = off;
  return w;
}

// ----------------------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct MapKey {
  uintptr_t ptr;
  uint64_t d0, d1, d2, rs;
  uint32_t b0, b1, b2, rank;
  int dev;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && rs == o.rs && b0 == o.b0 &&
           b1 == o.b1 && b2 == o.b2 && rank == o.rank && dev == o.dev;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = std::hash<uintptr_t>()(k.ptr);
    h ^= std::hash<uint64_t>()(k.d0 * 1315423911u + k.d1 * 2654435761u + k.d2 + k.rs * 40503u) +
         0x9e3779b9 + (h << 6) + (h >> 2);
    h ^= (size_t)k.b0 * 31 + k.b1 * 17 + k.b2 * 7 + k.rank + (size_t)k.dev * 101;
    return h;
  }
};

static std::mutex g_map_mu;
static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;

// bf16 tensor map with 128-byte swizzle.  rank 2: dims {d0, d1}, row stride d0*2 bytes;
// rank 3: dims {d0, d1, d2}, strides {d0*2, d0*d1*2}.  Cached per (pointer, shape, box, device).
// A bf16 tensor map with 128-byte swizzle, dims {d0 (contiguous), d1, d2}, box {b0, b1, b2}.  Rows
// (dimension 1) are row_bytes apart, or d0 * 2 bytes when row_bytes is 0.  Cached per key.
static etree_status get_map_rows(const void* ptr, int rank, uint64_t d0, uint64_t d1, uint64_t d2,
                                 uint64_t row_bytes, uint32_t b0, uint32_t b1, uint32_t b2,
                                 CUtensorMap* out) {
  int dev = 0;
  cudaGetDevice(&dev);
  MapKey key{reinterpret_cast<uintptr_t>(ptr), d0, d1, d2, row_bytes, b0, b1, b2,
             (uint32_t)rank, dev};
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return ETREE_OK;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(ETREE_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {d0, d1, d2};
  const uint64_t rb = row_bytes ? row_bytes : d0 * 2;
  cuuint64_t strides[2] = {rb, rb * d1};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap m;
  CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(ptr),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ETREE_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    if (g_maps.size() > 4096) g_maps.clear();
    g_maps.emplace(key, m);
  }
  *out = m;
  return ETREE_OK;
}

static etree_status get_map(const void* ptr, int rank, uint64_t d0, uint64_t d1, uint64_t d2,
                            uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMap* out) {
  return get_map_rows(ptr, rank, d0, d1, d2, 0, b0, b1, b2, out);
}

// fp32 2-D tensor map {d0 (contiguous), d1} with row stride d0 * 4 bytes and 64-byte swizzle, for
// the TMA stores of materialised logit rows (box {b0, b1}).  Not cached: encoded per call.
static etree_status get_map_f32_sw64(const void* ptr, uint64_t d0, uint64_t d1, uint32_t b0,
                                     uint32_t b1, CUtensorMap* out) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(ETREE_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {d0, d1};
  cuuint64_t strides[1] = {d0 * 4};
  cuuint32_t box[2] = {b0, b1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ETREE_ECUDA, "cuTensorMapEncodeTiled (fp32) failed (%d)", (int)r);
  return ETREE_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static etree_status check_batch(const etree_batch* b) {
  if (!b) return fail(ETREE_EINVAL, "batch is NULL");
  if (b->B < 1 || b->B > ETREE_MAX_REQUESTS)
    return fail(ETREE_EINVAL, "B=%d outside [1, %d]", b->B, ETREE_MAX_REQUESTS);
  if (b->n_max < 1 || b->n_max > ETREE_MAX_NODES)
    return fail(ETREE_EINVAL, "n_max=%d outside [1, %d]", b->n_max, ETREE_MAX_NODES);
  if (b->n_total < b->B || (int64_t)b->n_total > (int64_t)b->B * b->n_max)
    return fail(ETREE_EINVAL, "n_total=%d inconsistent with B=%d, n_max=%d", b->n_total, b->B,
                b->n_max);
  if (b->kv_len_max < 0) return fail(ETREE_EINVAL, "kv_len_max < 0");
  if (!b->cu_nodes || !b->parent || !b->tokens || !b->kv_len || !b->slot_base || !b->slot_cap)
    return fail(ETREE_EINVAL, "a batch array is NULL");
  return ETREE_OK;
}

static etree_status check_ws(const etree_batch* b, int hq, int hkv, int hidden_dim, int vocab,
                             void* ws, size_t bytes) {
  if (!ws) return fail(ETREE_EINVAL, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return fail(ETREE_EINVAL, "workspace is not 256-byte aligned");
  const size_t need = layout(b, hq, hkv, hidden_dim, vocab).total;
  if (bytes < need) return fail(ETREE_EINVAL, "workspace has %zu bytes, needs %zu", bytes, need);
  return ETREE_OK;
}

template <class T>
static T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}


// ------------------------------------------------------------------ statically backed scratch
// Scratch for etree_verify_attn_noalloc: a fixed array in device global memory, created when the
// library's module is loaded in a context and held until that context ends.  Host code must not
// use the symbol as a pointer; it asks the runtime for the device address in the current
// context.  The address is cached per context, keyed by the driver's context id, which is unique
// for the life of the process: a device reset or a caller-made context gets a fresh lookup.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_attn_scratch[kStaticScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static std::mutex g_scratch_mu;
static std::unordered_map<unsigned long long, void*> g_scratch_ptr;

// Device address of g_attn_scratch in the calling thread's current context.
static etree_status static_scratch(void** out) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id)
    return fail(ETREE_ECUDA, "etree_verify_attn_noalloc: cuCtxGetCurrent / cuCtxGetId unavailable");
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS)
    return fail(ETREE_ECUDA, "etree_verify_attn_noalloc: cuCtxGetCurrent failed");
  void* fresh = nullptr;
  if (!ctx) {
    // no context yet on this thread: the lookup itself makes the device's primary context
    // current (the runtime's usual lazy initialisation)
    const cudaError_t e = cudaGetSymbolAddress(&fresh, g_attn_scratch);
    if (e != cudaSuccess || !fresh)
      return cuda_fail(e, "etree_verify_attn_noalloc: cudaGetSymbolAddress");
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx)
      return fail(ETREE_ECUDA, "etree_verify_attn_noalloc: no current context");
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS)
    return fail(ETREE_ECUDA, "etree_verify_attn_noalloc: cuCtxGetId failed");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  auto it = g_scratch_ptr.find(id);
  if (it == g_scratch_ptr.end()) {
    if (!fresh) {
      const cudaError_t e = cudaGetSymbolAddress(&fresh, g_attn_scratch);
      if (e != cudaSuccess || !fresh)
        return cuda_fail(e, "etree_verify_attn_noalloc: cudaGetSymbolAddress");
    }
    if (g_scratch_ptr.size() > 1024) g_scratch_ptr.clear();
    it = g_scratch_ptr.emplace(id, fresh).first;
  }
  *out = it->second;
  return ETREE_OK;
}

}  // namespace etree

using namespace etree;

// =================================================================================== C ABI
extern "C" {

int etree_version(void) { return 100; }

const char* etree_strerror(etree_status s) {
  switch (s) {
    case ETREE_OK: return "ok";
    case ETREE_EINVAL: return "invalid argument";
    case ETREE_EUNSUPPORTED: return "unsupported configuration";
    case ETREE_ECUDA: return "CUDA error";
    case ETREE_EDEVICE: return "device-detected input error";
    case ETREE_ETIMEOUT: return "on-device wait timed out";
    case ETREE_ENOSPACE: return "request cache slots exhausted";
  }
  return "unknown status";
}

const char* etree_last_error(void) { return g_err; }

etree_status etree_attn_plan(const etree_batch* batch, int hq, int hkv, int32_t* kernel,
                             int32_t* rows_per_cta, int32_t* row_blocks, int32_t* splits,
                             int32_t* tiles_per_split, int32_t* launches) {
  etree_status st = check_batch(batch);
  if (st) return st;
  if (hq < 1 || hkv < 1 || hq % hkv != 0 || hq / hkv > 64)
    return fail(ETREE_EINVAL, "hq=%d, hkv=%d", hq, hkv);
  const AttnPlan pl = plan_attn(batch, hq, hkv);
  if (kernel) *kernel = 1;
  if (rows_per_cta) *rows_per_cta = pl.nb * pl.G;
  if (row_blocks) *row_blocks = pl.mchunks;
  if (splits) *splits = pl.nsplit;
  if (tiles_per_split) *tiles_per_split = pl.tps;
  if (launches) *launches = (pl.nsplit > 1 ? 2 : 1) + (batch->B >= 8 ? 1 : 0);
  return ETREE_OK;
}

size_t etree_workspace_size(const etree_batch* batch, int hq, int hkv, int head_dim,
                            int hidden_dim, int vocab) {
  (void)head_dim;
  if (check_batch(batch) != ETREE_OK) return 0;
  return layout(batch, hq, hkv, hidden_dim, vocab).total;
}

etree_status etree_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < sizeof(WsHeader))
    return fail(ETREE_EINVAL, "workspace too small");
  cudaError_t e =
      cudaMemsetAsync(workspace, 0, sizeof(WsHeader), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ETREE_OK : cuda_fail(e, "etree_workspace_init");
}

// ------------------------------------------------------------------ low-rank candidate head
struct LowrankLayout {
  size_t part, g, lists, cand, tkth, fmax, fcnt, total;
  int nk, nlists;
};

static LowrankLayout lowrank_layout(int M, int H, int r, int V) {
  LowrankLayout w{};
  size_t off = sizeof(WsHeader);
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  w.nk = lowrank_down_chunks(H);
  w.nlists = 2 * ((V + 127) / 128);                 // per vocab tile at the narrowest width
  // the sample's split-K partials (or the down projection's, in its split-K form)
  const size_t sample = (size_t)((r + 127) / 128) * M * lowrank_sample_cols(V);
  w.part = take(std::max((size_t)w.nk * M * r, sample) * sizeof(float));
  w.g = take((size_t)M * r * 2);
  w.lists = take((size_t)M * w.nlists * 16 * sizeof(float2));
  w.cand = take((size_t)M * 16 * sizeof(int32_t));
  w.tkth = take((size_t)M * sizeof(uint32_t));
  w.fmax = take((size_t)lowrank_floor_maxima(M) * sizeof(float));
  w.fcnt = take((size_t)M * sizeof(int32_t));
  w.total = off;
  return w;
}

size_t etree_lowrank_workspace_size(int M, int hidden_dim, int rank, int vocab) {
  if (M < 1 || hidden_dim < 1 || rank < 1 || vocab < 1) return 0;
  return lowrank_layout(M, hidden_dim, rank, vocab).total;
}

etree_status etree_lowrank_candidates(const uint16_t* hidden, int M, int hidden_dim,
                                      const uint16_t* D, const uint16_t* U, int rank,
                                      const uint16_t* W, int vocab, int k, int32_t* out_ids,
                                      float* out_logit, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  if (!hidden || !D || !U || !W || !out_ids || !out_logit || !workspace)
    return fail(ETREE_EINVAL, "a pointer is NULL");
  if (M < 1 || M > (1 << 20)) return fail(ETREE_EINVAL, "M=%d", M);
  if (hidden_dim < 64 || hidden_dim % 64 || hidden_dim > 8192)
    return fail(ETREE_EUNSUPPORTED, "hidden_dim=%d must be a multiple of 64 in [64, 8192]",
                hidden_dim);
  if (rank < 64 || rank % 64 || rank > 8192)
    return fail(ETREE_EUNSUPPORTED, "rank=%d must be a multiple of 64 in [64, 8192]", rank);
  if (k < 1 || k > 16 || vocab < k) return fail(ETREE_EINVAL, "k=%d (1..16, <= vocab)", k);
  if (!aligned16(hidden) || !aligned16(D) || !aligned16(U) || !aligned16(W) || !aligned16(workspace))
    return fail(ETREE_EINVAL, "hidden, D, U, W and the workspace must be 16-byte aligned");
  const LowrankLayout w = lowrank_layout(M, hidden_dim, rank, vocab);
  if (workspace_bytes < w.total)
    return fail(ETREE_EINVAL, "workspace has %zu bytes, needs %zu", workspace_bytes, w.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* hb = reinterpret_cast<const __nv_bfloat16*>(hidden);
  __nv_bfloat16* g = at<__nv_bfloat16>(workspace, w.g);
  uint32_t* tkth = at<uint32_t>(workspace, w.tkth);
  CUtensorMap th, td, tg, tus;
  etree_status st;
  if ((st = get_map(hidden, 2, hidden_dim, M, 1, 64, 64, 1, &th))) return st;
  if ((st = get_map(D, 2, hidden_dim, rank, 1, 64, 64, 1, &td))) return st;
  if ((st = get_map(g, 2, rank, M, 1, 64, 64, 1, &tg))) return st;
  // the sample: every stride-th row of U
  const int S = lowrank_sample_cols(vocab), stride = vocab / S;
  if ((st = get_map_rows(U, 2, rank, S, 1, (uint64_t)stride * rank * 2, 64, 64, 1, &tus)))
    return st;
  int32_t* fcnt = at<int32_t>(workspace, w.fcnt);
  float* part = at<float>(workspace, w.part);
  WsHeader* ws = at<WsHeader>(workspace, 0);
  cudaError_t e = launch_lowrank_down(th, td, M, hidden_dim, rank, part, g, tkth, fcnt, ws, s);
  if (e == cudaSuccess)
    e = launch_lowrank_sample(tg, tus, M, rank, vocab, part, at<float>(workspace, w.fmax), fcnt,
                              tkth, ws, s);
  if (e != cudaSuccess) return cuda_fail(e, "etree_lowrank_candidates (down, sample)");

  const int sms = sm_count();
  const int bn = lmhead_pick_bn(M, vocab, sms);
  const int bm = M <= 64 ? 64 : 128;
  CUtensorMap ta, tb;
  if ((st = get_map(g, 2, rank, M, 1, 64, bm, 1, &ta))) return st;
  if ((st = get_map(U, 2, rank, vocab, 1, 64, bn, 1, &tb))) return st;
  GemmParams gp{};
  gp.M = M;
  gp.V = vocab;
  gp.K = rank;
  gp.m_tiles = (M + bm - 1) / bm;
  gp.n_tiles = (vocab + bn - 1) / bn;
  gp.num_tiles = gp.m_tiles * gp.n_tiles;
  gp.k_blocks = rank / 64;
  gp.ws = at<WsHeader>(workspace, 0);
  const int grid = std::min(gp.num_tiles, sms);
  gp.per_cta = gp.m_tiles == 1;
  gp.n_parts = gp.per_cta ? grid : gp.n_tiles;
  gp.topk = at<float2>(workspace, w.lists);
  gp.tkth = tkth;
  e = launch_lmhead(3, bn, bm, ta, tb, tb, gp, grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "etree_lowrank_candidates (screen)");
  e = launch_lowrank_finish(gp.topk, 2 * gp.n_parts, M, k, at<int32_t>(workspace, w.cand), hb,
                            reinterpret_cast<const __nv_bfloat16*>(W), hidden_dim, vocab,
                            out_ids, out_logit, s);
  return e == cudaSuccess ? ETREE_OK : cuda_fail(e, "etree_lowrank_candidates (rescore)");
}

etree_status etree_device_status(void* workspace, void* stream, int32_t* detail) {
  if (!workspace) return fail(ETREE_EINVAL, "workspace is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "etree_device_status sync");
  int32_t h[2] = {0, 0};
  e = cudaMemcpy(h, workspace, sizeof h, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "etree_device_status read");
  e = cudaMemsetAsync(workspace, 0, sizeof h, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "etree_device_status clear");
  if (detail) *detail = h[1];
  return static_cast<etree_status>(h[0]);
}

// The bounded-wait path every pipeline relies on, exercised on purpose: one thread waits on an
// mbarrier that no thread ever arrives at; the wait gives up after its iteration cap and the
// kernel records ETREE_ETIMEOUT (detail DET_SELFTEST) in the workspace status word.  Nothing
// traps, and the context stays usable.  The self-test runs the same wait loop with a cap of 256
// tries (about a millisecond) instead of the pipelines' (about 8 s), so the test is brief.
constexpr uint32_t kSelftestWaitCap = 256;

__global__ void selftest_wait_kernel(WsHeader* ws) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    if (!mbar_wait(&bar, 0, kSelftestWaitCap)) report(ws, ETREE_ETIMEOUT, DET_SELFTEST);
  }
}

etree_status etree_selftest_timeout(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < sizeof(WsHeader) || ((uintptr_t)workspace & 255))
    return fail(ETREE_EINVAL, "workspace is NULL, smaller than its header or misaligned");
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      at<WsHeader>(workspace, 0));
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ETREE_OK : cuda_fail(e, "etree_selftest_timeout launch");
}

// A paged cache: the block table [B][max_pages] and the page size (a power of two >= 16).
struct PagedArgs {
  const int32_t* block_table;
  int32_t max_pages;
  int32_t page_size;
};

static etree_status check_paged(const PagedArgs* pg, int64_t num_pages) {
  if (!pg) return ETREE_OK;
  if (!pg->block_table || ((uintptr_t)pg->block_table & 3))
    return fail(ETREE_EINVAL, "block_table is NULL or misaligned");
  if (pg->max_pages < 1) return fail(ETREE_EINVAL, "max_pages=%d", pg->max_pages);
  const int P = pg->page_size;
  if (P < 16 || P > (1 << 20) || (P & (P - 1)))
    return fail(ETREE_EINVAL, "page_size=%d: need a power of two in [16, 2^20]", P);
  if (num_pages < 1 || num_pages * P > INT32_MAX)
    return fail(ETREE_EINVAL, "num_pages=%lld: need 1 <= num_pages * page_size < 2^31",
                (long long)num_pages);
  return ETREE_OK;
}

static int log2i(int x) {
  int k = 0;
  while ((1 << k) < x) ++k;
  return k;
}

// Host-visible checks of the attention arguments other than the workspace.
static etree_status check_attn_args(const etree_batch* b, const uint16_t* q,
                                    const uint16_t* k_tree, const uint16_t* v_tree,
                                    const uint16_t* k_cache, const uint16_t* v_cache,
                                    int64_t cache_slots, int hq, int hkv, int head_dim,
                                    float scale, const uint16_t* out, const float* lse) {
  etree_status st = check_batch(b);
  if (st) return st;
  if (head_dim != ETREE_HEAD_DIM)
    return fail(ETREE_EUNSUPPORTED, "head_dim=%d (only 128 is built)", head_dim);
  if (hq < 1 || hkv < 1 || hq % hkv != 0 || hq / hkv > 64)
    return fail(ETREE_EINVAL, "hq=%d, hkv=%d: need hq %% hkv == 0 and hq/hkv <= 64", hq, hkv);
  if (!q || !k_tree || !v_tree || !k_cache || !v_cache || !out)
    return fail(ETREE_EINVAL, "a tensor pointer is NULL");
  if (!aligned16(q) || !aligned16(k_tree) || !aligned16(v_tree) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(out) || (lse && ((uintptr_t)lse & 3)))
    return fail(ETREE_EINVAL, "tensors must be 16-byte aligned");
  if (cache_slots < 1 || cache_slots > INT32_MAX)
    return fail(ETREE_EINVAL, "cache_slots=%lld outside [1, 2^31)", (long long)cache_slots);
  if (!std::isfinite(scale)) return fail(ETREE_EINVAL, "scale is not finite");
  return ETREE_OK;
}

static etree_status verify_attn_impl(const etree_batch* b, const uint16_t* q,
                                     const uint16_t* k_tree, const uint16_t* v_tree,
                                     const uint16_t* k_cache, const uint16_t* v_cache,
                                     int64_t cache_slots, int hq, int hkv, int head_dim,
                                     float scale, uint16_t* out, float* lse,
                                     const PagedArgs* pg, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  etree_status st = check_attn_args(b, q, k_tree, v_tree, k_cache, v_cache, cache_slots, hq, hkv,
                                    head_dim, scale, out, lse);
  if (st) return st;
  if ((st = check_ws(b, hq, hkv, 0, 0, workspace, workspace_bytes))) return st;

  const AttnPlan pl = plan_attn(b, hq, hkv);
  CUtensorMap kc, vc, kt, vt;
  const uint32_t kb = (uint32_t)pl.keys;
  const uint32_t cbox = pg ? (uint32_t)std::min(pl.keys, pg->page_size) : kb;
  if ((st = get_map(k_cache, 3, 128, hkv, cache_slots, 64, 1, cbox, &kc))) return st;
  if ((st = get_map(v_cache, 3, 128, hkv, cache_slots, 64, 1, cbox, &vc))) return st;
  if ((st = get_map(k_tree, 3, 128, hkv, b->n_total, 64, 1, kb, &kt))) return st;
  if ((st = get_map(v_tree, 3, 128, hkv, b->n_total, 64, 1, kb, &vt))) return st;

  const WsLayout w = layout(b, hq, hkv, 0, 0);
  AttnParams p{};
  p.order = nullptr;
  p.cu_nodes = b->cu_nodes;
  p.parent = b->parent;
  p.kv_len = b->kv_len;
  p.slot_base = b->slot_base;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.o_part = at<float>(workspace, w.o_part);
  p.ml_part = at<float2>(workspace, w.ml_part);
  p.ws = at<WsHeader>(workspace, 0);
  p.B = b->B;
  p.hq = hq;
  p.hkv = hkv;
  p.G = pl.G;
  p.n_max = b->n_max;
  p.kv_len_max = b->kv_len_max;
  p.cache_slots = cache_slots;
  p.mchunks = pl.mchunks;
  p.nsplit = pl.nsplit;
  p.tps = pl.tps;
  p.keys = pl.keys;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.block_table = pg ? pg->block_table : nullptr;
  p.max_pages = pg ? pg->max_pages : 0;
  p.page_shift = pg ? log2i(pg->page_size) : 0;
  p.cache_box = (int)cbox;
  cudaError_t e;
  // with many requests of mixed lengths, dispatch the longest first
  p.order = nullptr;
  if (b->B >= 8) {
    p.order = at<int32_t>(workspace, w.order);
    e = launch_attn_order(b->kv_len, b->B, at<int32_t>(workspace, w.order),
                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "etree_verify_attn order");
  }
  CUtensorMap tq;
  if ((st = get_map(q, 3, 128, hq, b->n_total, 64, pl.G, pl.nb, &tq))) return st;
  e = launch_attn_tc(tq, kc, vc, kt, vt, p, pl.nb, b->n_total, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ETREE_OK : cuda_fail(e, "etree_verify_attn launch");
}

etree_status etree_verify_attn(const etree_batch* b, const uint16_t* q, const uint16_t* k_tree,
                               const uint16_t* v_tree, const uint16_t* k_cache,
                               const uint16_t* v_cache, int64_t cache_slots, int hq, int hkv,
                               int head_dim, float scale, uint16_t* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream) {
  return verify_attn_impl(b, q, k_tree, v_tree, k_cache, v_cache, cache_slots, hq, hkv, head_dim,
                          scale, out, lse, nullptr, workspace, workspace_bytes, stream);
}

etree_status etree_verify_attn_paged(const etree_batch* b, const int32_t* block_table,
                                     int32_t max_pages, int32_t page_size, const uint16_t* q,
                                     const uint16_t* k_tree, const uint16_t* v_tree,
                                     const uint16_t* k_pool, const uint16_t* v_pool,
                                     int64_t num_pages, int hq, int hkv, int head_dim,
                                     float scale, uint16_t* out, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  const PagedArgs pg{block_table, max_pages, page_size};
  etree_status st = check_paged(&pg, num_pages);
  if (st) return st;
  return verify_attn_impl(b, q, k_tree, v_tree, k_pool, v_pool, num_pages * page_size, hq, hkv,
                          head_dim, scale, out, lse, &pg, workspace, workspace_bytes, stream);
}

// The caller's logit buffer of the branching-tree sampler (etree_lmhead_accept_tree).
struct TreeRows {
  float* zbuf;
  int32_t rows;
};

static etree_status lmhead_accept_impl(const etree_batch* b, const uint16_t* hidden,
                                       const uint16_t* w_lm, int hidden_dim, int vocab,
                                       float temperature, const float* q_draft, uint64_t seed,
                                       uint64_t step, int32_t* accept_len, int32_t* path,
                                       int32_t* out_tokens, int32_t* node_argmax,
                                       float* node_gap, const TreeRows* tree, void* workspace,
                                       size_t workspace_bytes, void* stream,
                                       void* const* marks = nullptr) {
  etree_status st = check_batch(b);
  if (st) return st;
  if (hidden_dim < 64 || hidden_dim % 64 != 0)
    return fail(ETREE_EUNSUPPORTED, "hidden_dim=%d must be a positive multiple of 64",
                hidden_dim);
  if (vocab < 1) return fail(ETREE_EINVAL, "vocab=%d", vocab);
  if (!(temperature >= 0.f) || !std::isfinite(temperature))
    return fail(ETREE_EINVAL, "temperature must be finite and >= 0");
  if (temperature > 0.f && !q_draft) return fail(ETREE_EINVAL, "T > 0 needs q_draft");
  if (!hidden || !w_lm || !accept_len || !path || !out_tokens)
    return fail(ETREE_EINVAL, "a tensor pointer is NULL");
  if (!aligned16(hidden) || !aligned16(w_lm))
    return fail(ETREE_EINVAL, "hidden and w_lm must be 16-byte aligned");
  if ((st = check_ws(b, 0, 0, hidden_dim, vocab, workspace, workspace_bytes))) return st;
  // the workspace regions used here do not depend on the attention shape
  const WsLayout w = layout(b, 0, 0, hidden_dim, vocab);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const int sms = sm_count();
  const int bn = lmhead_pick_bn(b->n_total, vocab, sms);
  // up to 64 rows: M=64 MMAs with half-height hidden tiles (the W stream is the cost)
  const int bm = b->n_total <= 64 ? 64 : 128;
  CUtensorMap ta, tb;
  if ((st = get_map(hidden, 2, hidden_dim, b->n_total, 1, 64, bm, 1, &ta))) return st;
  if ((st = get_map(w_lm, 2, hidden_dim, vocab, 1, 64, bn, 1, &tb))) return st;

  GemmParams g{};
  g.M = b->n_total;
  g.V = vocab;
  g.K = hidden_dim;
  g.m_tiles = (b->n_total + bm - 1) / bm;
  g.n_tiles = (vocab + bn - 1) / bn;
  g.num_tiles = g.m_tiles * g.n_tiles;
  g.k_blocks = hidden_dim / 64;
  g.ws = at<WsHeader>(workspace, 0);
  g.part = at<float4>(workspace, w.part);
  g.child_tok = at<int32_t>(workspace, w.child_tok);
  g.zchild = at<float>(workspace, w.zchild);
  g.k_log2 = temperature > 0.f ? 1.4426950408889634f / temperature : 0.f;
  g.stop_row = at<int32_t>(workspace, w.stop_row);
  g.stop_node = at<int32_t>(workspace, w.stop_node);
  g.cval = at<float>(workspace, w.cval);
  g.lse2 = at<float>(workspace, w.lse2);
  g.q_draft = q_draft;
  g.seed = seed;
  g.step = step;
  const int grid = std::min(g.num_tiles, sms);
  g.per_cta = g.m_tiles == 1;
  g.n_parts = g.per_cta ? grid : g.n_tiles;
  int32_t* cnt = at<int32_t>(workspace, w.cnt);
  g.cnt = cnt;
  g.cnt_n = b->B;

  AcceptParams a{};
  a.B = b->B;
  a.n_total = b->n_total;
  a.n_max = b->n_max;
  a.V = vocab;
  a.n_tiles = 2 * g.n_parts;
  a.cu_nodes = b->cu_nodes;
  a.parent = b->parent;
  a.tokens = b->tokens;
  a.part = g.part;
  a.accept_len = accept_len;
  a.path = path;
  a.out_tokens = out_tokens;
  a.node_argmax = node_argmax;
  a.node_gap = node_gap;
  a.ws = g.ws;
  a.k_log2 = g.k_log2;
  a.zchild = g.zchild;
  a.lse2 = at<float>(workspace, w.lse2);
  a.q_draft = q_draft;
  a.seed = seed;
  a.step = step;
  a.stop_row = at<int32_t>(workspace, w.stop_row);
  a.stop_node = at<int32_t>(workspace, w.stop_node);
  a.cval = at<float>(workspace, w.cval);
  a.hidden = reinterpret_cast<const __nv_bfloat16*>(hidden);
  a.hid2 = at<__nv_bfloat16>(workspace, w.hid2);
  a.H = hidden_dim;
  a.part2 = at<float4>(workspace, w.part2);
  a.rfloor = at<uint32_t>(workspace, w.rfloor);

  // phase marks (measurement only): events recorded after the set-up kernels, the first GEMM,
  // the acceptance kernels and the draw GEMM
  auto mark = [&](int k) {
    if (marks && marks[k]) cudaEventRecord(static_cast<cudaEvent_t>(marks[k]), s);
  };
  cudaError_t e;
  if (temperature == 0.f) {
    mark(0);
    e = launch_lmhead(0, bn, bm, ta, tb, tb, g, grid, s);
    mark(1);
    if (e == cudaSuccess) e = launch_accept_greedy(a, at<int32_t>(workspace, w.child_tok), cnt, s);
    mark(2);
    mark(3);
    return e == cudaSuccess ? ETREE_OK : cuda_fail(e, "etree_lmhead_accept (T=0)");
  }
  if (!tree) {                               // chains: accept tests fused with the row merge
    e = launch_chain_prep(a, at<int32_t>(workspace, w.child_tok), s);
    mark(0);
    if (e == cudaSuccess) e = launch_lmhead(1, bn, bm, ta, tb, tb, g, grid, s);
    mark(1);
    if (e == cudaSuccess) e = launch_accept_chain(a, cnt, s);
  } else {                                   // trees: materialised rows of branching nodes
    int32_t* zrow = at<int32_t>(workspace, w.zrow);
    float* zc = at<float>(workspace, w.zc);
    e = launch_tree_prep(a, reinterpret_cast<const __nv_bfloat16*>(w_lm),
                         at<int32_t>(workspace, w.ccount), zrow, tree->rows, zc, s);
    mark(0);
    g.child_tok = nullptr;
    g.zrow = zrow;
    g.zbuf = tree->zbuf;
    // every row kept at M >= 128 rows: the rows leave through TMA stores of 32 x 16 boxes
    CUtensorMap tz = tb;
    if (tree->rows >= b->n_total && bm == 128 && (vocab & 3) == 0 && aligned16(tree->zbuf)) {
      if ((st = get_map_f32_sw64(tree->zbuf, (uint64_t)vocab, (uint64_t)b->n_total, 16, 32, &tz)))
        return st;
      g.z_tma = 1;
    }
    if (e == cudaSuccess) e = launch_lmhead(1, bn, bm, ta, tb, tz, g, grid, s);
    g.z_tma = 0;
    mark(1);
    g.zrow = nullptr;
    g.zbuf = nullptr;
    if (e == cudaSuccess)
      e = launch_tree_walk(a, tree->rows >= b->n_total ? nullptr : zc, zrow, tree->zbuf, sms, s);
    if (e == cudaSuccess && tree->rows >= b->n_total) {
      // every row's logits are in zbuf: the draw reads the stop rows there (no second W pass)
      mark(2);
      mark(3);
      const int parts = draw_parts(b->B, vocab, sms, w.n_tiles);
      e = launch_draw_rows(a, zrow, tree->zbuf, parts, at<float4>(workspace, w.part2), cnt, s);
      return e == cudaSuccess ? ETREE_OK : cuda_fail(e, "etree_lmhead_accept (T>0, draw)");
    }
  }
  mark(2);
  if (e != cudaSuccess) return cuda_fail(e, "etree_lmhead_accept (T>0, pass 1)");
  // the draw pass: the stop row of every request, M = B rows
  const int bn2 = lmhead_pick_bn(b->B, vocab, sms);
  const int bm2 = b->B <= 64 ? 64 : 128;
  CUtensorMap th, tb2;
  if ((st = get_map(a.hid2, 2, hidden_dim, b->B, 1, 64, bm2, 1, &th))) return st;
  if ((st = get_map(w_lm, 2, hidden_dim, vocab, 1, 64, bn2, 1, &tb2))) return st;
  GemmParams g2 = g;
  g2.M = b->B;
  g2.m_tiles = (b->B + bm2 - 1) / bm2;
  g2.n_tiles = (vocab + bn2 - 1) / bn2;
  g2.num_tiles = g2.m_tiles * g2.n_tiles;
  g2.part = at<float4>(workspace, w.part2);
  const int grid2 = std::min(g2.num_tiles, sms);
  g2.per_cta = g2.m_tiles == 1;
  g2.n_parts = g2.per_cta ? grid2 : g2.n_tiles;
  g2.cnt = nullptr;
  g2.rfloor = a.rfloor;
  a.n_tiles2 = 2 * g2.n_parts;
  e = launch_lmhead(2, bn2, bm2, th, tb2, tb2, g2, grid2, s);
  mark(3);
  if (e == cudaSuccess) e = launch_bonus(a, s);
  return e == cudaSuccess ? ETREE_OK : cuda_fail(e, "etree_lmhead_accept (T>0, pass 2)");
}

etree_status etree_lmhead_accept(const etree_batch* b, const uint16_t* hidden,
                                 const uint16_t* w_lm, int hidden_dim, int vocab,
                                 float temperature, const float* q_draft, uint64_t seed,
                                 uint64_t step, int32_t* accept_len, int32_t* path,
                                 int32_t* out_tokens, int32_t* node_argmax, float* node_gap,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return lmhead_accept_impl(b, hidden, w_lm, hidden_dim, vocab, temperature, q_draft, seed, step,
                            accept_len, path, out_tokens, node_argmax, node_gap, nullptr,
                            workspace, workspace_bytes, stream);
}

etree_status etree_lmhead_accept_tree(const etree_batch* b, const uint16_t* hidden,
                                      const uint16_t* w_lm, int hidden_dim, int vocab,
                                      float temperature, const float* q_draft, uint64_t seed,
                                      uint64_t step, int32_t* accept_len, int32_t* path,
                                      int32_t* out_tokens, float* zbuf, int32_t zbuf_rows,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (zbuf_rows < 0 || (zbuf_rows > 0 && !zbuf))
    return fail(ETREE_EINVAL, "zbuf_rows=%d with zbuf=%p", zbuf_rows, (void*)zbuf);
  if (zbuf && !aligned16(zbuf)) return fail(ETREE_EINVAL, "zbuf must be 16-byte aligned");
  const TreeRows tr{zbuf, zbuf_rows};
  return lmhead_accept_impl(b, hidden, w_lm, hidden_dim, vocab, temperature, q_draft, seed, step,
                            accept_len, path, out_tokens, nullptr, nullptr,
                            temperature > 0.f ? &tr : nullptr, workspace, workspace_bytes,
                            stream);
}

etree_status etree_lmhead_accept_timed(const etree_batch* b, const uint16_t* hidden,
                                       const uint16_t* w_lm, int hidden_dim, int vocab,
                                       float temperature, const float* q_draft, uint64_t seed,
                                       uint64_t step, int32_t* accept_len, int32_t* path,
                                       int32_t* out_tokens, int32_t* node_argmax,
                                       float* node_gap, float* zbuf, int32_t zbuf_rows,
                                       int32_t branching, void* const* marks, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (branching && (zbuf_rows < 0 || (zbuf_rows > 0 && !zbuf)))
    return fail(ETREE_EINVAL, "zbuf_rows=%d with zbuf=%p", zbuf_rows, (void*)zbuf);
  if (branching && zbuf && !aligned16(zbuf))
    return fail(ETREE_EINVAL, "zbuf must be 16-byte aligned");
  const TreeRows tr{zbuf, zbuf_rows};
  return lmhead_accept_impl(b, hidden, w_lm, hidden_dim, vocab, temperature, q_draft, seed, step,
                            accept_len, path, out_tokens, branching ? nullptr : node_argmax,
                            branching ? nullptr : node_gap,
                            (branching && temperature > 0.f) ? &tr : nullptr, workspace,
                            workspace_bytes, stream, marks);
}

static etree_status kv_compact_impl(const etree_batch* b, const int32_t* accept_len,
                                    const int32_t* path, const uint16_t* k_tree,
                                    const uint16_t* v_tree, uint16_t* k_cache,
                                    uint16_t* v_cache, int n_layers, int64_t tree_layer_stride,
                                    int64_t cache_layer_stride, int hkv, int head_dim,
                                    int32_t* kv_len_out, const PagedArgs* pg, int64_t pool_slots,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  etree_status st = check_batch(b);
  if (st) return st;
  if (head_dim != ETREE_HEAD_DIM)
    return fail(ETREE_EUNSUPPORTED, "head_dim=%d (only 128 is built)", head_dim);
  if (hkv < 1 || n_layers < 1 || n_layers > 65535 || (int64_t)hkv * head_dim * 2 % 16)
    return fail(ETREE_EINVAL, "hkv=%d, n_layers=%d", hkv, n_layers);
  if (!accept_len || !path || !k_tree || !v_tree || !k_cache || !v_cache || !kv_len_out)
    return fail(ETREE_EINVAL, "a pointer is NULL");
  if (kv_len_out == b->kv_len) return fail(ETREE_EINVAL, "kv_len_out aliases batch->kv_len");
  if (!aligned16(k_tree) || !aligned16(v_tree) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(ETREE_EINVAL, "K/V tensors must be 16-byte aligned");
  const int64_t row = (int64_t)hkv * head_dim;
  if (n_layers > 1 && (tree_layer_stride < row * b->n_total || cache_layer_stride < row ||
                       tree_layer_stride % 8 || cache_layer_stride % 8))
    return fail(ETREE_EINVAL, "layer strides must cover a layer and be multiples of 8");
  if (pg && n_layers > 1 && cache_layer_stride < row * pool_slots)
    return fail(ETREE_EINVAL, "cache_layer_stride must cover a layer's page pool");
  if ((st = check_ws(b, 0, 0, 0, 0, workspace, workspace_bytes))) return st;
  CompactParams p{};
  p.cu_nodes = b->cu_nodes;
  p.kv_len = b->kv_len;
  p.slot_base = b->slot_base;
  p.slot_cap = b->slot_cap;
  p.accept_len = accept_len;
  p.path = path;
  p.k_tree = reinterpret_cast<const uint4*>(k_tree);
  p.v_tree = reinterpret_cast<const uint4*>(v_tree);
  p.k_cache = reinterpret_cast<uint4*>(k_cache);
  p.v_cache = reinterpret_cast<uint4*>(v_cache);
  p.kv_len_out = kv_len_out;
  p.ws = at<WsHeader>(workspace, 0);
  p.B = b->B;
  p.n_max = b->n_max;
  p.n_layers = n_layers;
  p.tree_layer_stride16 = tree_layer_stride / 8;
  p.cache_layer_stride16 = cache_layer_stride / 8;
  p.row16 = (int)(row / 8);
  p.block_table = pg ? pg->block_table : nullptr;
  p.max_pages = pg ? pg->max_pages : 0;
  p.page_shift = pg ? log2i(pg->page_size) : 0;
  p.cache_slots = pool_slots;
  // the layers are spread over about 16 CTAs per SM
  cudaError_t e = launch_compact(p, 32 * sm_count(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ETREE_OK : cuda_fail(e, "etree_kv_compact launch");
}

etree_status etree_kv_compact(const etree_batch* b, const int32_t* accept_len,
                              const int32_t* path, const uint16_t* k_tree,
                              const uint16_t* v_tree, uint16_t* k_cache, uint16_t* v_cache,
                              int n_layers, int64_t tree_layer_stride,
                              int64_t cache_layer_stride, int hkv, int head_dim,
                              int32_t* kv_len_out, void* workspace, size_t workspace_bytes,
                              void* stream) {
  return kv_compact_impl(b, accept_len, path, k_tree, v_tree, k_cache, v_cache, n_layers,
                         tree_layer_stride, cache_layer_stride, hkv, head_dim, kv_len_out,
                         nullptr, 0, workspace, workspace_bytes, stream);
}

etree_status etree_kv_compact_paged(const etree_batch* b, const int32_t* block_table,
                                    int32_t max_pages, int32_t page_size,
                                    const int32_t* accept_len, const int32_t* path,
                                    const uint16_t* k_tree, const uint16_t* v_tree,
                                    uint16_t* k_pool, uint16_t* v_pool, int64_t num_pages,
                                    int n_layers, int64_t tree_layer_stride,
                                    int64_t cache_layer_stride, int hkv, int head_dim,
                                    int32_t* kv_len_out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  const PagedArgs pg{block_table, max_pages, page_size};
  etree_status st = check_paged(&pg, num_pages);
  if (st) return st;
  return kv_compact_impl(b, accept_len, path, k_tree, v_tree, k_pool, v_pool, n_layers,
                         tree_layer_stride, cache_layer_stride, hkv, head_dim, kv_len_out, &pg,
                         num_pages * page_size, workspace, workspace_bytes, stream);
}

// Tree attention without a caller workspace: the split partials and the status words live in
// the library's static scratch array (see etree.h for the contract).
etree_status etree_verify_attn_noalloc(const etree_batch* b, const uint16_t* q,
                                       const uint16_t* k_tree, const uint16_t* v_tree,
                                       const uint16_t* k_cache, const uint16_t* v_cache,
                                       int64_t cache_slots, int hq, int hkv, int head_dim,
                                       float scale, uint16_t* out, float* lse,
                                       int32_t* status_out, void* stream) {
  // every host check runs before the shared array is touched: a rejected call changes nothing
  etree_status st = check_attn_args(b, q, k_tree, v_tree, k_cache, v_cache, cache_slots, hq, hkv,
                                    head_dim, scale, out, lse);
  if (st) return st;
  if (status_out && ((uintptr_t)status_out & 3))
    return fail(ETREE_EINVAL, "status_out must be 4-byte aligned");
  const size_t need = layout(b, hq, hkv, 0, 0).total;
  if (need > kStaticScratchBytes)
    return fail(ETREE_EINVAL,
                "etree_verify_attn_noalloc: this batch needs %zu bytes of scratch, more than the "
                "%zu-byte static array; use etree_verify_attn with a workspace",
                need, kStaticScratchBytes);
  void* ws = nullptr;
  if ((st = static_scratch(&ws))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status words must start at zero for every call; the partials are written before read
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(WsHeader), s);
  if (e != cudaSuccess) return cuda_fail(e, "etree_verify_attn_noalloc: clear status");
  st = etree_verify_attn(b, q, k_tree, v_tree, k_cache, v_cache, cache_slots, hq, hkv, head_dim,
                         scale, out, lse, ws, kStaticScratchBytes, stream);
  if (st) return st;
  if (status_out) {
    e = cudaMemcpyAsync(status_out, ws, 2 * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "etree_verify_attn_noalloc: copy status");
  }
  return ETREE_OK;
}

}  // extern "C"
