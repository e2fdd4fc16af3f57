/*
 * etree.h -- C ABI of libetree: the target model's one-pass verification of a draft token tree
 * (EAGLE-style speculative decoding) on NVIDIA B200 (sm_100a).
 *
 * What the three calls compute.  Speculative decoding lets a small draft model propose tokens
 * that the target model then checks all at once, in one parallel forward pass: the target keeps
 * the longest drafted prefix consistent with its own distribution and adds one token of its own
 * after the first rejected position ("Eagle-4 Released: Outpaces DFlash2 and DSpark ...",
 * kongchang.com/en, section "Technical Background", speculative-decoding paragraph).  EAGLE-2's
 * dynamic draft tree lets one verification cover several candidate paths (same section).  Tree
 * verification needs an unquantized KV cache, and engines admit trees and chains for up to 512
 * running requests ("EAGLE-4 官方推理代码发布：eagle-harness v0.1.0 ...", arex-research.com,
 * paragraph on hardware coverage and limits).  Per-sequence acceptance lengths under continuous
 * batching are the main engineering difficulty ("Eagle-4 Released ...", section "Current
 * Limitation").
 *
 *   etree_verify_attn    tree-masked GQA attention of every tree node against its request's
 *                        bf16 KV cache plus the tree nodes that are its ancestors (or itself);
 *   etree_lmhead_accept  LM-head projection of every node's hidden state fused with a per-row
 *                        argmax (T = 0) or max / log-sum-exp (T > 0) reduction -- logits are
 *                        never written to memory -- followed by the acceptance walk that returns
 *                        the longest accepted path and the bonus token;
 *   etree_kv_compact     copies the root's and the accepted nodes' K/V into the request's next
 *                        cache slots.
 *
 * Conventions shared by every call:
 *  - Pointers are DEVICE pointers unless stated; the caller owns all memory.  bf16 tensors are
 *    passed as uint16_t bit patterns.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *  - Calls are asynchronous: they validate host-visible arguments, enqueue kernels and return.
 *    Stream order holds as usual: every input a call reads may be produced by the work enqueued
 *    just before it on the same stream.  Some kernels are launched with programmatic dependent
 *    launch and start their set-up (barriers, tensor memory, descriptor and weight prefetch)
 *    while the previous kernel finishes, but read their inputs and write their outputs only
 *    after it has completed.  The LM-head GEMM requests its first weight tiles (W, or U for the
 *    low-rank screen) before that wait, so the one case to avoid is a kernel that signals its
 *    dependents early (griddepcontrol.launch_dependents) and writes those weights, enqueued right
 *    before the call; no kernel of this library writes them.
 *  - Problems visible on the host return at once (ETREE_EINVAL / ETREE_EUNSUPPORTED) and enqueue
 *    nothing.  Problems visible only on the device (a malformed parent array, a KV length past
 *    its bound, a full cache) are recorded in the workspace status word; the affected request is
 *    skipped with safe outputs and etree_device_status() returns the code.  No kernel traps.
 *  - The library allocates no device memory.  The caller passes a workspace of at least
 *    etree_workspace_size() bytes (256-byte aligned), zeroed once by etree_workspace_init().
 *    One workspace serves one stream at a time.
 *  - The only global state is a per-process cache of TMA descriptors keyed by pointer and shape.
 */
#ifndef ETREE_H
#define ETREE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ETREE_OK = 0,
  ETREE_EINVAL = -1,        /* bad argument: null pointer, size out of range, misalignment   */
  ETREE_EUNSUPPORTED = -2,  /* valid but not supported: head_dim != 128, T > 0 on a tree ...  */
  ETREE_ECUDA = -3,         /* a CUDA runtime/driver call failed                              */
  ETREE_EDEVICE = -4,       /* device-detected input error (malformed tree, bad length, ...)  */
  ETREE_ETIMEOUT = -5,      /* a bounded on-device wait gave up                               */
  ETREE_ENOSPACE = -6       /* a request's cache slots cannot hold the accepted tokens        */
} etree_status;

/* Compile-time limits of the library. */
#define ETREE_MAX_NODES 64      /* nodes per tree, root included (ancestor masks are uint64)  */
#define ETREE_MAX_REQUESTS 4096
#define ETREE_HEAD_DIM 128
#define ETREE_PATH_STRIDE 64    /* path is [B][64]                                            */
#define ETREE_OUT_STRIDE 65     /* out_tokens is [B][65]: up to 63 accepted + 1 bonus, padded */

/*
 * One verification step's batch of requests.  Request r owns nodes cu_nodes[r] ..
 * cu_nodes[r+1]-1 (its "local" node j is global node cu_nodes[r] + j).  Local node 0 is the
 * root, the last committed token: its K/V are produced by this step and are NOT yet in the
 * cache.  Every other node is a draft token whose parent has a smaller local index.
 */
typedef struct etree_batch {
  int32_t B;                  /* requests, 1 .. ETREE_MAX_REQUESTS                          */
  int32_t n_total;            /* total nodes = cu_nodes[B]                                   */
  int32_t n_max;              /* max nodes of one request, 1 .. ETREE_MAX_NODES              */
  int32_t kv_len_max;         /* host-side upper bound on every kv_len[r] (sizes the grid)  */
  const int32_t *cu_nodes;    /* device [B+1], cu_nodes[0] = 0, non-decreasing               */
  const int32_t *parent;      /* device [n_total], LOCAL parent; -1 for the root            */
  const int32_t *tokens;      /* device [n_total], token id of each node                     */
  const int32_t *kv_len;      /* device [B], tokens already in request r's cache             */
  const int64_t *slot_base;   /* device [B], first pooled-cache slot of request r            */
  const int32_t *slot_cap;    /* device [B], slots reserved for request r                    */
} etree_batch;

/* Bytes of workspace that the three calls need for this batch and these shapes. */
size_t etree_workspace_size(const etree_batch *batch, int hq, int hkv, int head_dim,
                            int hidden_dim, int vocab);

/* Zeroes the status words of a fresh workspace (asynchronous, on `stream`). */
etree_status etree_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Tree-masked GQA attention.  The target scores every drafted token in one parallel forward, and
 * a draft tree lets that pass cover several candidate paths ("Eagle-4 Released: Outpaces DFlash2
 * and DSpark ...", section "Technical Background"); each node therefore sees its request's cache
 * and exactly its own ancestors.  The KV cache stays unquantized bf16 ("EAGLE-4 官方推理代码发布
 * ...", paragraph on hardware coverage and limits).
 * For node i of request r and query head h (KV head h / (hq/hkv)):
 * keys = the kv_len[r] cached positions (pooled rows slot_base[r] + t) followed by the tree nodes
 * j with j == i or j an ancestor of i;  out = softmax(scale * q k^T) v;  lse = log sum exp.
 *   q        [n_total][hq][head_dim]  bf16
 *   k_tree   [n_total][hkv][head_dim] bf16, v_tree likewise (this step's K/V of every node)
 *   k_cache  [cache_slots][hkv][head_dim] bf16 pooled cache, v_cache likewise
 *   out      [n_total][hq][head_dim]  bf16
 *   lse      [n_total][hq] fp32 natural-log log-sum-exp of the scaled scores; may be NULL
 * head_dim must be 128; hq % hkv == 0; hq/hkv <= 64; all tensors 16-byte aligned.
 * The library reads `cache_slots` rows at most; cached rows at positions >= kv_len[r] are ignored.
 */
etree_status etree_verify_attn(const etree_batch *batch, const uint16_t *q,
                               const uint16_t *k_tree, const uint16_t *v_tree,
                               const uint16_t *k_cache, const uint16_t *v_cache,
                               int64_t cache_slots, int hq, int hkv, int head_dim, float scale,
                               uint16_t *out, float *lse, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * Tree attention for callers that cannot allocate device memory.  Serving engines commonly
 * reserve nearly all of HBM for their own KV-cache pool at start-up, so a later cudaMalloc can
 * fail; cudaMalloc can also synchronise the device and stall a latency-critical decode loop; and
 * some plugin hosts hand their plugins no allocator at all.  Such callers cannot size and pass a
 * workspace.  The paper has no counterpart: this is a deployment convenience.
 * Same arguments, computation and output as etree_verify_attn, without a workspace: the split
 * partials and the status words live in one static 16 MiB device array inside the library, which
 * every context that loads the library holds until the context ends.  16 MiB covers the largest
 * KV split the planner makes at the shapes this library is measured on (about 12 MiB at a
 * 128K-token cache, 40/8 heads, 16 nodes).  The call allocates nothing (no cudaMalloc / cudaFree,
 * no allocating library routine).
 *  - Every host-side check of etree_verify_attn runs first; a rejected call touches nothing.
 *  - A batch that needs more than 16 MiB of scratch (etree_workspace_size with hidden_dim = 0 and
 *    vocab = 0) is rejected with ETREE_EINVAL before any device work; use etree_verify_attn.
 *  - The first call in a CUDA context looks up the array's device address there
 *    (cudaGetSymbolAddress) and caches it under the context's unique id, so a device reset or a
 *    context of the caller's own gets its own lookup; make that first call before any stream
 *    capture.
 *  - Every call clears the status words, then reuses the array, which keeps the last call's
 *    contents.  Calls whose kernels overlap on the GPU (other streams, other threads) race on
 *    the array: serialise them.
 *  - status_out (device, 2 int32, may be NULL) receives the call's device status and detail code
 *    (the values etree_device_status would return), written asynchronously on `stream`.
 */
etree_status etree_verify_attn_noalloc(const etree_batch *batch, const uint16_t *q,
                                       const uint16_t *k_tree, const uint16_t *v_tree,
                                       const uint16_t *k_cache, const uint16_t *v_cache,
                                       int64_t cache_slots, int hq, int hkv, int head_dim,
                                       float scale, uint16_t *out, float *lse,
                                       int32_t *status_out, void *stream);

/*
 * Tree attention over a paged KV cache (block tables, as serving engines hold KV).  Same result
 * as etree_verify_attn on the logical caches: position t (0 <= t < kv_len[r]) of request r lives
 * at pool slot  block_table[r * max_pages + t / page_size] * page_size + t % page_size  of
 * k_pool / v_pool, each [num_pages * page_size][hkv][head_dim] bf16 (16-byte aligned).
 * batch->slot_base is not used.  page_size is a power of two in [16, 2^20]; pages smaller than
 * the kernel's key tile are loaded page by page.  block_table is a device int32 array
 * [B][max_pages]; only entries covering positions below kv_len[r] are read for keys.  An entry
 * outside [0, num_pages) records ETREE_EDEVICE (detail 11) and its keys read as zeros;
 * kv_len[r] > max_pages * page_size records ETREE_EDEVICE (detail 3).  Other arguments,
 * workspace and errors as etree_verify_attn, with num_pages * page_size in place of cache_slots.
 * (Paged caches are how the engines the pages plug into hold KV: "EAGLE-4 官方推理代码发布 ...",
 * section on the harness being a plug-in for SGLang and vLLM.)
 */
etree_status etree_verify_attn_paged(const etree_batch *batch, const int32_t *block_table,
                                     int32_t max_pages, int32_t page_size, const uint16_t *q,
                                     const uint16_t *k_tree, const uint16_t *v_tree,
                                     const uint16_t *k_pool, const uint16_t *v_pool,
                                     int64_t num_pages, int hq, int hkv, int head_dim,
                                     float scale, uint16_t *out, float *lse, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * LM head + acceptance.  The target keeps the longest drafted prefix consistent with its own
 * distribution and adds one token of its own after the first rejection ("Eagle-4 Released ...",
 * section "Technical Background"); at T > 0 the rule must keep the target's output distribution
 * ("EAGLE-4 官方推理代码发布 ...", section on sizing the tree by measured cost).  The vocab head
 * is the costly part of an LM head (65.4% of a draft forward: "EAGLE-4 是什麼？...",
 * aiposthub.com, Fig. 2), so its logits are reduced where they are computed and never stored.
 * z = hidden W^T (fp32 accumulate over bf16 inputs) for every node row.
 *  T == 0 (greedy): t*(u) = argmax z_u (lowest id on ties).  From the root, repeatedly move to
 *    the lowest-index child whose token equals t*(current); the node where no child matches
 *    stops the walk and t* there is the bonus token.
 *  T > 0 (chains only, every node has <= 1 child): p_u = softmax(z_u / T); node k's token x was
 *    drafted from q_draft row k-1; it is accepted iff U * q(x) < p(x), U a seeded uniform.  At
 *    the first rejection (node u) the bonus is drawn from norm(max(0, p_u - q_u)); when all are
 *    accepted it is drawn from p of the last node; a residual with no positive weight (p <= q
 *    everywhere: p = q up to rounding) is answered by a draw from p_u.  Draws are exponential
 *    races over every vocab id (the id with the largest w_v / E_v, E_v = -log U_v) with
 *    Philox4x64-10 uniforms keyed by (seed, step) and countered by (vocab id / 8, node, request,
 *    stream), so results are reproducible bit for bit.  A branching tree records
 *    ETREE_EUNSUPPORTED (detail 5, "not a chain") and that request accepts nothing; sample
 *    branching trees with etree_lmhead_accept_tree.
 *   hidden      [n_total][hidden_dim] bf16;   w_lm [vocab][hidden_dim] bf16 (K contiguous)
 *   q_draft     [n_total][vocab] fp32 draft probabilities (T > 0 only, else may be NULL)
 *   accept_len  [B] accepted draft nodes a_r (0 .. n_r - 1)
 *   path        [B][64] local node ids: path[r][0] = 0 (root), path[r][1..a_r]; rest -1
 *   out_tokens  [B][65] tokens of the accepted nodes, then the bonus token; rest -1
 *   node_argmax [n_total] per-node argmax (T == 0 only; may be NULL)
 *   node_gap    [n_total] per-node top1 - top2 logit gap, fp32 (T == 0 only; may be NULL)
 * hidden_dim must be a multiple of 64; vocab >= 256.
 */
etree_status etree_lmhead_accept(const etree_batch *batch, const uint16_t *hidden,
                                 const uint16_t *w_lm, int hidden_dim, int vocab,
                                 float temperature, const float *q_draft, uint64_t seed,
                                 uint64_t step, int32_t *accept_len, int32_t *path,
                                 int32_t *out_tokens, int32_t *node_argmax, float *node_gap,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * LM head + stochastic acceptance over general draft trees (T > 0; T == 0 behaves exactly like
 * etree_lmhead_accept).  The pages verify whole trees in one pass ("Eagle-4 Released: Outpaces
 * DFlash2 and DSpark ...", section "Technical Background") but give no sampling rule for
 * siblings; this call takes multi-candidate speculative sampling (SpecInfer, Miao et al. 2023):
 * the children of node u, whose tokens were drafted independently from q_draft row u, are tested
 * in node-index order against a running target r that starts at p_u = softmax(z_u / T): child c
 * with token x is accepted iff U_c * q_u(x) < r(x), and each rejection replaces r by
 * norm(max(0, r - q_u)), which equals max(0, p_u - c q_u) / N(c) for an offset c that grows by
 * N(c) = sum_v max(0, p_u(v) - c q_u(v)) per rejection.  An accepted child becomes the node
 * whose children are tested next.  The walk stops at a leaf or when all children of a node are
 * rejected; the bonus is drawn there from max(0, p_u - c q_u) (from p_u when nothing was
 * rejected there) with the exponential race of etree_lmhead_accept; a residual without positive
 * weight is answered by a draw from p_u.  On chains the results equal etree_lmhead_accept's.
 *   zbuf       caller-owned device buffer [zbuf_rows][vocab] fp32, 16-byte aligned: the logits
 *              of every node with two or more children are written there (in node order),
 *              because each sibling rejection needs a pass over the whole row.  At most
 *              floor((n_total - B) / 2) rows are ever needed.  A batch with more branching nodes
 *              than zbuf_rows records ETREE_ENOSPACE (detail 10) and the requests left without a
 *              row accept nothing: their bonus is drawn from the root's p (a one-token
 *              decode).  zbuf may be NULL when zbuf_rows == 0 (chains need no rows).
 *              A malformed request (a parent not below its child: ETREE_EDEVICE detail 1; a
 *              token outside [0, vocab): detail 9) accepts nothing and gets no bonus token:
 *              path[r][0] = 0, out_tokens[r] all -1.
 *              With zbuf_rows >= n_total, every node's logits are stored (row g for node g) and
 *              the bonus draw reads the stop row there instead of making a second pass over
 *              w_lm for the B stop rows: the tokens are the same, the second W pass (a GEMM of B
 *              rows) is replaced by reading B logit rows, at the cost of n_total x vocab x 4
 *              bytes of buffer.  This works for chains as well as trees.
 *   Other arguments as in etree_lmhead_accept (no node_argmax / node_gap outputs).
 * Errors: host-side as etree_lmhead_accept, plus ETREE_EINVAL for zbuf_rows < 0, a NULL zbuf
 * with zbuf_rows > 0, or a misaligned zbuf.
 */
etree_status etree_lmhead_accept_tree(const etree_batch *batch, const uint16_t *hidden,
                                      const uint16_t *w_lm, int hidden_dim, int vocab,
                                      float temperature, const float *q_draft, uint64_t seed,
                                      uint64_t step, int32_t *accept_len, int32_t *path,
                                      int32_t *out_tokens, float *zbuf, int32_t zbuf_rows,
                                      void *workspace, size_t workspace_bytes, void *stream);

/*
 * etree_lmhead_accept (branching = 0) or etree_lmhead_accept_tree (branching = 1, with zbuf and
 * zbuf_rows; node_argmax / node_gap are then unused), with phase marks for measuring where the
 * call's device time goes.  marks (host array of 4 cudaEvent_t, each may be NULL; the whole
 * array may be NULL) are recorded on `stream` after: [0] the set-up kernels before the first
 * GEMM, [1] the first GEMM (every node row), [2] the acceptance kernels, [3] the draw GEMM over
 * the stop rows (T > 0; at T = 0 marks 2 and 3 coincide).  Results are identical to the
 * unmarked calls; the event records keep kernels from overlapping their neighbours' set-up, so
 * time whole steps with the unmarked calls.  The pages report end-to-end figures only; this
 * call exists to report the second (draw) pass separately from the algorithmic first pass.
 */
etree_status etree_lmhead_accept_timed(const etree_batch *batch, const uint16_t *hidden,
                                       const uint16_t *w_lm, int hidden_dim, int vocab,
                                       float temperature, const float *q_draft, uint64_t seed,
                                       uint64_t step, int32_t *accept_len, int32_t *path,
                                       int32_t *out_tokens, int32_t *node_argmax,
                                       float *node_gap, float *zbuf, int32_t zbuf_rows,
                                       int32_t branching, void *const *marks, void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * KV compaction.  Requests accept different numbers of drafted tokens each step, and keeping
 * their caches aligned under continuous batching is the engineering difficulty the pages name
 * ("Eagle-4 Released ...", section "Community Reaction and Future Outlook"): the accepted nodes'
 * K/V move into the request's next contiguous slots.
 * For each of n_layers layers and each request r with a = accept_len[r]:
 *   cache[slot_base[r] + kv_len[r] + k] <- tree[cu_nodes[r] + path[r][k]],  k = 0 .. a,
 * for K and V, then kv_len_out[r] = kv_len[r] + a + 1 (the bonus token's K/V come next step).
 * path is the [B][64] array etree_lmhead_accept writes; all 64 entries of a row are read.
 * Rows are [hkv][head_dim] bf16.  Layer l of the tree K/V starts tree_layer_stride ELEMENTS after
 * layer l-1, likewise for the caches.  kv_len_out must not alias batch->kv_len.  A request whose
 * new rows would pass slot_cap[r] is left untouched (kv_len_out = kv_len) with ETREE_ENOSPACE.
 */
etree_status etree_kv_compact(const etree_batch *batch, const int32_t *accept_len,
                              const int32_t *path, const uint16_t *k_tree,
                              const uint16_t *v_tree, uint16_t *k_cache, uint16_t *v_cache,
                              int n_layers, int64_t tree_layer_stride,
                              int64_t cache_layer_stride, int hkv, int head_dim,
                              int32_t *kv_len_out, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * KV compaction into a paged cache: as etree_kv_compact, with destination position
 * t = kv_len[r] + k going to pool slot block_table[r * max_pages + t / page_size] * page_size +
 * t % page_size (layout and page rules of etree_verify_attn_paged).  slot_cap[r] is the
 * request's mapped capacity in tokens; a request whose new rows would pass it is left untouched
 * with ETREE_ENOSPACE, and one whose destination page entry lies outside [0, num_pages) is left
 * untouched with ETREE_EDEVICE (detail 11).  For n_layers > 1, cache_layer_stride must cover
 * num_pages * page_size rows.
 */
etree_status etree_kv_compact_paged(const etree_batch *batch, const int32_t *block_table,
                                    int32_t max_pages, int32_t page_size,
                                    const int32_t *accept_len, const int32_t *path,
                                    const uint16_t *k_tree, const uint16_t *v_tree,
                                    uint16_t *k_pool, uint16_t *v_pool, int64_t num_pages,
                                    int n_layers, int64_t tree_layer_stride,
                                    int64_t cache_layer_stride, int hkv, int head_dim,
                                    int32_t *kv_len_out, void *workspace,
                                    size_t workspace_bytes, void *stream);

/*
 * Low-rank candidate head: screen the vocabulary with a factorised projection, then score only
 * the survivors exactly.  EAGLE-4's draft uses such a head in place of its full vocabulary
 * projection ("EAGLE-4 是什麼？...", aiposthub.com, section "EAGLE-4 是什麼？先看推測解碼為什麼能變快",
 * Fig. 2: the vocab head is 65.4% of a 574 us draft forward; rank 512 brings the forward to
 * 326 us, rank 128 to 255 us).  For each of M rows h (hidden [M][hidden_dim] bf16):
 *   g  = h D^T   (D [rank][hidden_dim] bf16), fp32 accumulation, rounded to bf16;
 *   z~ = g U^T   (U [vocab][rank] bf16), fp32 accumulation: the approximate logits;
 *   C  = the k ids of largest z~ (lower id first on equal values), 1 <= k <= 16;
 *   z_c = h . W_c (W [vocab][hidden_dim] bf16, the exact head), fp32 accumulation;
 * out_ids [M][k] holds C ordered by z_c descending (lower id first on equal values) and
 * out_logit [M][k] the z_c.  hidden_dim and rank are multiples of 64, at most 8192.  The
 * workspace (etree_lowrank_workspace_size bytes, 16-byte aligned, status words cleared by
 * etree_workspace_init) is independent of the verification workspace; etree_device_status reads
 * its status.  All pointers are device pointers, 16-byte aligned.  Asynchronous on `stream`.
 */
size_t etree_lowrank_workspace_size(int M, int hidden_dim, int rank, int vocab);
etree_status etree_lowrank_candidates(const uint16_t *hidden, int M, int hidden_dim,
                                      const uint16_t *D, const uint16_t *U, int rank,
                                      const uint16_t *W, int vocab, int k, int32_t *out_ids,
                                      float *out_logit, void *workspace, size_t workspace_bytes,
                                      void *stream);

/*
 * Hardware-aware tree sizing (host-only; no device work).  The pages size the draft tree from the
 * measured cost of drafting and verifying at the running batch size and hardware
 * ("EAGLE-4 官方推理代码发布 ...", arex-research.com, section "投机树多大，由实测成本决定").
 *
 * etree_cost_table: measured µs of one verification step (attention, LM head with acceptance,
 * compaction; draft_tree_verification_masked_b200/calibrate.py writes one) on the grid
 * B[0..nB) x N[0..nN) x L[0..nL) (each strictly ascending; N = tree nodes per request, root
 * included; L = cached tokens per request), us[(i * nN + j) * nL + k] for (B[i], N[j], L[k]).
 * All pointers are host pointers owned by the caller.
 */
typedef struct {
  int32_t nB, nN, nL;
  const int32_t *B, *N, *L;
  const float *us;
} etree_cost_table;

/*
 * Step time at (B, N, L): trilinear interpolation on the grid, each axis extended linearly past
 * its first and last points; negative results clamp to 0.  ETREE_EINVAL for a malformed table.
 */
etree_status etree_verify_cost(const etree_cost_table *table, double B, double N, double L,
                               double *us_out);

typedef struct {
  int32_t depth, width, nodes;      /* chosen static tree; depth 0 = no speculation (1 node) */
  double expected_accept;           /* expected accepted draft tokens per request and step */
  double step_us;                   /* draft time + interpolated verification time */
  double tokens_per_s;              /* B (expected_accept + 1) / step_us, whole batch */
} etree_tree_plan;

/*
 * The static draft tree that maximises expected tokens per second for B requests of L cached
 * tokens.  Shape: `depth` levels; at each level the top draft candidate continues the spine and
 * width - 1 lower-ranked candidates sit beside it as leaves, so nodes = 1 + depth * width
 * (<= max_nodes <= 64, depth <= max_depth <= 63, width <= max_width).  Acceptance model: at
 * every level the target's token is the rank-k draft candidate with probability acc_rank[k]
 * (k = 0 .. n_rank-1, sum <= 1, independent across levels); the walk continues only through the
 * spine, so E[accepted] = sum_{j=1..depth} acc_rank[0]^(j-1) (acc_rank[0] + ... + acc_rank[width-1]).
 * Step time = draft_us_fixed + depth * draft_us_per_level (both 0 when depth = 0) plus
 * etree_verify_cost(B, nodes, L); a step time of 0 (a table extrapolated below zero) counts as
 * 0 tokens/s.  Ties (within 1e-12 relative) go to the fewer nodes, then the shallower tree.
 * ETREE_EINVAL for out-of-range arguments or a malformed table.
 */
etree_status etree_plan_tree(const etree_cost_table *table, int32_t B, int32_t L,
                             const float *acc_rank, int32_t n_rank, float draft_us_per_level,
                             float draft_us_fixed, int32_t max_depth, int32_t max_width,
                             int32_t max_nodes, etree_tree_plan *out);

/*
 * Synchronizes `stream`, reads the workspace status word (the first device-detected error since
 * the last read, ETREE_OK if none), stores its detail code in *detail (if not NULL) and clears
 * both words.  Detail codes:
 *    0  none
 *    1  bad parent: parent[0] != -1 or parent[i] outside [0, i)
 *    2  bad node count: a request with 0 or more than n_max nodes
 *    3  bad kv_len: negative, above kv_len_max, or past the cache pool
 *    4  capacity: kv_len + accepted + 1 > slot_cap
 *    5  not a chain: T > 0 on a node with more than one child (etree_lmhead_accept)
 *    6  bad path: path or accept_len out of range in compaction
 *    7  attention wait: a bounded wait gave up in attention
 *    8  gemm wait: a bounded wait gave up in the LM-head GEMM
 *    9  bad token: a token id outside [0, vocab)
 *   10  logit rows: more branching nodes than zbuf rows (etree_lmhead_accept_tree)
 *   11  bad page: a block-table entry outside [0, num_pages) for a used position
 *   12  self-test wait: etree_selftest_timeout's deliberately unfinished wait gave up
 *   13  walk wait: the tree walk gave up waiting for another CTA's part of a residual sum
 */
etree_status etree_device_status(void *workspace, void *stream, int32_t *detail);

/*
 * Diagnostic: launches one thread that waits on a barrier nothing ever completes, through the same
 * bounded wait every kernel of the library uses.  The wait gives up after its iteration cap
 * (about 8 s on a B200) and records ETREE_ETIMEOUT with detail 12 in the workspace status word,
 * which etree_device_status then returns; nothing traps and the context stays usable.  The
 * workspace needs only its 256-byte status header (256-byte aligned).
 */
etree_status etree_selftest_timeout(void *workspace, size_t workspace_bytes, void *stream);

/* Static description of a status code. */
const char *etree_strerror(etree_status status);

/* Message describing the last host-side failure of a call on this thread ("" if none). */
const char *etree_last_error(void);

/*
 * The launch plan etree_verify_attn uses for this batch and head shape (host-only, no device
 * work): the kernel (always 1, the tcgen05/TMEM kernel), query rows per CTA, row blocks per
 * (request, KV head), KV splits, key tiles per split, and the number of kernels the call
 * launches.  Any output pointer may be NULL.
 */
etree_status etree_attn_plan(const etree_batch *batch, int hq, int hkv, int32_t *kernel,
                             int32_t *rows_per_cta, int32_t *row_blocks, int32_t *splits,
                             int32_t *tiles_per_split, int32_t *launches);

/* Library version: major * 10000 + minor * 100 + patch. */
int etree_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ETREE_H */
