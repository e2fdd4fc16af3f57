// kernels.cuh -- parameter blocks and launchers of the etree kernels, shared by the kernel
// translation units and the C-ABI layer.
#pragma once
#include "common.cuh"

namespace etree {

// Order-preserving map of fp32 to uint32 (monotone: a < b iff enc(a) < enc(b)), so that atomicMax
// on the code keeps a running maximum of floats of either sign.
__host__ __device__ __forceinline__ uint32_t enc_order(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__host__ __device__ __forceinline__ float dec_order(uint32_t c) {
  const uint32_t u = (c & 0x80000000u) ? (c & 0x7fffffffu) : ~c;
  float x;
  memcpy(&x, &u, 4);
  return x;
}

struct AttnParams {
  const int32_t* cu_nodes;
  const int32_t* parent;
  const int32_t* kv_len;
  const int64_t* slot_base;
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  float* lse;
  float* o_part;
  float2* ml_part;
  WsHeader* ws;
  int B, hq, hkv, G, n_max, kv_len_max;
  int64_t cache_slots;
  int mchunks, nsplit, tps;
  int keys;                 // keys per KV tile (the tree takes ceil(n / keys) tiles at the end)
  const int32_t* order;     // [B] requests by decreasing KV length (dispatch order), or null
  float scale_log2;
  // Paged cache (block_table != null): position t of request r is pool slot
  // block_table[r * max_pages + t / 2^page_shift] * 2^page_shift + t % 2^page_shift; cache
  // tiles are loaded in boxes of cache_box rows (KEYS, or the page size when pages are smaller).
  const int32_t* block_table;
  int max_pages, page_shift, cache_box;
};
cudaError_t launch_attn_combine(const AttnParams& p, int n_total, cudaStream_t stream);
cudaError_t launch_attn_order(const int32_t* kv_len, int B, int32_t* order, cudaStream_t stream);
cudaError_t launch_attn_tc(const CUtensorMap& q, const CUtensorMap& kc, const CUtensorMap& vc,
                           const CUtensorMap& kt, const CUtensorMap& vt, const AttnParams& p,
                           int nb, int n_total, cudaStream_t stream);

struct GemmParams {
  int M, V, K, m_tiles, n_tiles, num_tiles, k_blocks;
  // per_cta = 1 (one row tile only): each CTA folds all its vocab tiles into one summary per
  // row and half, at slot blockIdx.x; else one summary per vocab tile, at slot nt.  n_parts is
  // the number of slots per row.
  int per_cta, n_parts;
  int32_t* cnt;                     // if set, CTA 0 zeroes cnt[0 .. cnt_n) (acceptance counters)
  int cnt_n;
  const int32_t* zrow;              // EPI_LSE, if set: row g's logits go to zbuf[zrow[g]][V]
  float* zbuf;                      // when zrow[g] >= 0 (rows of branching tree nodes)
  int z_tma;                        // EPI_LSE, BM = 128: every row is stored (zrow[g] = g) through
                                    // the tm_z tensor map (32-row x 16-column boxes)
  float2* topk;                     // EPI_TOPK: per (row, slot, half) 16 (value, id bits)
  uint32_t* tkth;                   // EPI_TOPK: per row, order-encoded lower bound of the k-th
  WsHeader* ws;
  float4* part;
  const int32_t* child_tok;
  float* zchild;
  float k_log2;
  const int32_t* stop_row;
  const int32_t* stop_node;
  // Draw weights of the race pass per request: w = max(0, p - cval q); cval = 0 draws from p,
  // cval < 0 marks a residual without positive weight (the bonus is drawn from p).
  const float* cval;
  uint32_t* rfloor;                 // RACE: per request, the best (residual, p) keys published
                                    // so far (fp32 bits; zeroed by the acceptance kernels)
  const float* lse2;
  const float* q_draft;
  uint64_t seed, step;
};
int lmhead_pick_bn(int M, int V, int grid);
cudaError_t launch_lmhead(int epi, int bn, int bm, const CUtensorMap& ta, const CUtensorMap& tb,
                          const CUtensorMap& tz, const GemmParams& p, int grid,
                          cudaStream_t stream);

struct AcceptParams {
  int B, n_total, n_max, V, n_tiles, n_tiles2;
  const int32_t* cu_nodes;
  const int32_t* parent;
  const int32_t* tokens;
  const float4* part;
  int32_t* accept_len;
  int32_t* path;
  int32_t* out_tokens;
  int32_t* node_argmax;
  float* node_gap;
  WsHeader* ws;
  float k_log2;
  const float* zchild;
  float* lse2;
  const float* q_draft;
  uint64_t seed, step;
  int32_t* stop_row;
  int32_t* stop_node;
  float* cval;
  const __nv_bfloat16* hidden;
  __nv_bfloat16* hid2;
  int H;
  const float4* part2;
  uint32_t* rfloor;                 // [B][2] race floors of the draw pass, zeroed per request
};
cudaError_t launch_accept_greedy(const AcceptParams& p, int32_t* arg_ws, int32_t* cnt,
                                 cudaStream_t s);
cudaError_t launch_chain_prep(const AcceptParams& p, int32_t* child_tok, cudaStream_t s);
cudaError_t launch_accept_chain(const AcceptParams& p, int32_t* cnt, cudaStream_t s);
cudaError_t launch_bonus(const AcceptParams& p, cudaStream_t s);
int draw_parts(int B, int V, int sms, int max_parts);
cudaError_t launch_draw_rows(const AcceptParams& p, const int32_t* zrow, const float* zbuf,
                             int parts, float4* dpart, int32_t* dcnt, cudaStream_t s);
cudaError_t launch_tree_prep(const AcceptParams& p, const __nv_bfloat16* w_lm, int32_t* ccount,
                             int32_t* zrow, int zbuf_rows, float* zc, cudaStream_t s);
cudaError_t launch_tree_walk(const AcceptParams& p, const float* zc, const int32_t* zrow,
                             const float* zbuf, int sms, cudaStream_t s);

int lowrank_down_chunks(int H);
int lowrank_sample_cols(int V);
int lowrank_floor_maxima(int M);
cudaError_t launch_lowrank_down(const CUtensorMap& tm_h, const CUtensorMap& tm_d, int M, int H,
                                int r, float* part, __nv_bfloat16* g, uint32_t* tkth,
                                int32_t* fcnt, WsHeader* ws, cudaStream_t s);
cudaError_t launch_lowrank_sample(const CUtensorMap& tm_g, const CUtensorMap& tm_us, int M, int r,
                                  int V, float* part, float* fmax, int32_t* fcnt, uint32_t* tkth,
                                  WsHeader* ws, cudaStream_t s);
cudaError_t launch_lowrank_finish(const float2* lists, int nlists, int M, int k, int32_t* cand,
                                  const __nv_bfloat16* hid, const __nv_bfloat16* W, int H, int V,
                                  int32_t* out_ids, float* out_logit, cudaStream_t s);

struct CompactParams {
  const int32_t* cu_nodes;
  const int32_t* kv_len;
  const int64_t* slot_base;
  const int32_t* slot_cap;
  const int32_t* accept_len;
  const int32_t* path;
  const uint4* k_tree;
  const uint4* v_tree;
  uint4* k_cache;
  uint4* v_cache;
  int32_t* kv_len_out;
  WsHeader* ws;
  int B, n_max, n_layers;
  int64_t tree_layer_stride16, cache_layer_stride16;
  int row16;
  // Paged cache (block_table != null): destination position t of request r is pool slot
  // block_table[r * max_pages + t / 2^page_shift] * 2^page_shift + t % 2^page_shift, and
  // slot_base is unused; pool slots per layer: cache_slots.
  const int32_t* block_table;
  int max_pages, page_shift;
  int64_t cache_slots;
};
cudaError_t launch_compact(const CompactParams& p, int ctas, cudaStream_t s);

}  // namespace etree
