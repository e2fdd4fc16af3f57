/*
 * oracle.c -- plain, slow, fp64 CPU reference for draft-tree verification.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load this library.  The CUDA library never includes, links or calls it, and it shares
 * no code with the CUDA path.
 *
 * What it computes is the plain definition of each step of the target's one-pass verification of
 * a draft token tree (speculative decoding as described on the pages "Eagle-4 Released: Outpaces
 * DFlash2 and DSpark ..." (kongchang.com/en), section "Technical Background": the target checks
 * all drafted tokens in one parallel forward, keeps the prefix consistent with its own
 * distribution and adds one token of its own after the first rejection; EAGLE-2's dynamic draft
 * tree lets one verification cover several candidate paths).  All floating point is fp64 on the
 * exact bf16/fp32 input values; the only library routines are exp and log from libm.
 *
 * Readings taken where the pages are silent:
 *  - node 0 of a request is the root (the last committed token); its K/V are produced by this pass
 *    and are not yet in the cache;
 *  - attention has no positional term, soft-cap or window: q and k arrive ready to dot;
 *  - greedy: argmax ties go to the lowest vocab id; among children carrying the argmax token the
 *    lowest node index is taken;
 *  - T>0 on chains: node k's token was drafted from q of node k-1; accept iff U*q < p (strict);
 *    the bonus/residual token is drawn by an exponential race over all vocab ids with
 *    Philox4x64-10 uniforms (oracle_race), an exact sampler of the normalised weights;
 *  - a residual with no positive weight (p <= q everywhere, which in exact arithmetic means
 *    p = q, where the rejected draft would have been accepted with probability 1) draws the
 *    bonus from p itself, so the emitted token still follows the target's distribution;
 *  - T>0 on branching trees (the pages give no rule): siblings are candidates drafted
 *    independently from their parent's q and are tested in index order by multi-candidate
 *    speculative sampling, each rejection replacing the target by its normalised residual
 *    (oracle_accept_tree).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_OK = 0, OR_EINVAL = -1, OR_EUNSUPPORTED = -2, OR_ENOSPACE = -6 };

static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------------------------------
 * Tree ancestry.  anc[i] has bit j set iff node j is i itself or an ancestor of i; depth(root)=0.
 * The tree arrives as a parent array with parent[0] = -1 and parent[i] < i for i > 0.
 * Returns OR_OK, or OR_EINVAL for a malformed parent array.  n <= 64.
 * ------------------------------------------------------------------------------------------- */
int oracle_ancestry(int n, const int32_t *parent, uint64_t *anc, int32_t *depth) {
    if (n < 1 || n > 64) return OR_EINVAL;
    if (parent[0] != -1) return OR_EINVAL;
    anc[0] = 1ull;
    depth[0] = 0;
    for (int i = 1; i < n; ++i) {
        int p = parent[i];
        if (p < 0 || p >= i) return OR_EINVAL;
        anc[i] = anc[p] | (1ull << i);
        depth[i] = depth[p] + 1;
    }
    return OR_OK;
}

static int request_of(int B, const int32_t *cu_nodes, int g) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (cu_nodes[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* ---------------------------------------------------------------------------------------------
 * Tree-masked GQA attention, one output row per (node, query head).
 *
 * For node i of request r and query head h (KV head h / (hq/hkv)): the keys are the r's cached
 * positions 0 .. kv_len[r]-1 (pooled cache rows slot_base[r] + t) followed by the tree nodes j
 * that are i or an ancestor of i (rows cu_nodes[r] + j of the tree K/V).
 *   s_j = scale * <q, k_j>;  p_j = exp(s_j - max s) / sum;  o = sum_j p_j v_j;
 *   lse = max s + log(sum exp(s_j - max s)).
 * Layouts: q [n_total][hq][d]; k_tree, v_tree [n_total][hkv][d]; caches [slots][hkv][d]; all bf16
 * bits.  rows == NULL computes every (node, head), written at [node*hq + h]; otherwise rows holds
 * nrows pairs (node, head) and the outputs are [k].  Returns OR_OK or OR_EINVAL (bad tree).
 * ------------------------------------------------------------------------------------------- */
int oracle_attention(int B, const int32_t *cu_nodes, const int32_t *parent, const int32_t *kv_len,
                     const int64_t *slot_base, const uint16_t *q, const uint16_t *k_tree,
                     const uint16_t *v_tree, const uint16_t *k_cache, const uint16_t *v_cache,
                     int hq, int hkv, int d, double scale, int nrows, const int32_t *rows,
                     double *out, double *lse, int nthreads) {
    const int ntot = cu_nodes[B];
    const int group = hq / hkv;
    const long total = rows ? (long)nrows : (long)ntot * hq;
    int status = OR_OK;
    set_threads(nthreads);
#pragma omp parallel
    {
        double *s = NULL;
        long s_cap = 0;
#pragma omp for schedule(dynamic, 1)
        for (long k = 0; k < total; ++k) {
            int g = rows ? rows[2 * k] : (int)(k / hq);
            int h = rows ? rows[2 * k + 1] : (int)(k % hq);
            int r = request_of(B, cu_nodes, g);
            int base = cu_nodes[r], n = cu_nodes[r + 1] - cu_nodes[r];
            int i = g - base;
            uint64_t anc[64];
            int32_t dep[64];
            if (oracle_ancestry(n, parent + base, anc, dep) != OR_OK) {
#pragma omp atomic write
                status = OR_EINVAL;
                continue;
            }
            int kvh = h / group;
            long L = kv_len[r];
            long nkeys = L + n;
            if (nkeys > s_cap) {
                free(s);
                s_cap = nkeys;
                s = (double *)malloc(sizeof(double) * (size_t)s_cap);
            }
            const uint16_t *qrow = q + ((size_t)g * hq + h) * d;
            double qv[256];
            for (int c = 0; c < d; ++c) qv[c] = bf16_value(qrow[c]);
            /* scores over cache keys, then the ancestor tree keys (others are left out) */
            double mx = -INFINITY;
            for (long t = 0; t < L; ++t) {
                const uint16_t *kr = k_cache + ((size_t)(slot_base[r] + t) * hkv + kvh) * d;
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += qv[c] * bf16_value(kr[c]);
                s[t] = scale * acc;
                if (s[t] > mx) mx = s[t];
            }
            for (int j = 0; j < n; ++j) {
                if (!((anc[i] >> j) & 1ull)) { s[L + j] = -INFINITY; continue; }
                const uint16_t *kr = k_tree + ((size_t)(base + j) * hkv + kvh) * d;
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += qv[c] * bf16_value(kr[c]);
                s[L + j] = scale * acc;
                if (s[L + j] > mx) mx = s[L + j];
            }
            double den = 0.0;
            double o[256];
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (long t = 0; t < nkeys; ++t) {
                if (s[t] == -INFINITY) continue;
                double p = exp(s[t] - mx);
                den += p;
                const uint16_t *vr = (t < L)
                    ? v_cache + ((size_t)(slot_base[r] + t) * hkv + kvh) * d
                    : v_tree + ((size_t)(base + (t - L)) * hkv + kvh) * d;
                for (int c = 0; c < d; ++c) o[c] += p * bf16_value(vr[c]);
            }
            double *orow = out + (size_t)k * d;
            for (int c = 0; c < d; ++c) orow[c] = o[c] / den;
            if (lse) lse[k] = mx + log(den);
        }
        free(s);
    }
    return status;
}

/* ---------------------------------------------------------------------------------------------
 * LM-head logits z[k][v] = sum_h hidden[rows[k]][h] * W[v][h], summed over h in increasing order
 * in fp64.  hidden [*][H], W [V][H] (bf16 bits, row-major).  z is [nrows][V].
 * ------------------------------------------------------------------------------------------- */
void oracle_logits(int nrows, const int32_t *rows, int H, int V, const uint16_t *hidden,
                   const uint16_t *w, double *z, int nthreads) {
    /* x transposed to [H][nrows] so that the row accumulators sit side by side */
    double *xt = (double *)malloc(sizeof(double) * (size_t)H * (size_t)nrows);
    for (int k = 0; k < nrows; ++k)
        for (int h = 0; h < H; ++h)
            xt[(size_t)h * nrows + k] = bf16_value(hidden[(size_t)rows[k] * H + h]);
    set_threads(nthreads);
#pragma omp parallel
    {
        double *wrow = (double *)malloc(sizeof(double) * (size_t)H);
        double *acc = (double *)malloc(sizeof(double) * (size_t)nrows);
#pragma omp for schedule(static)
        for (int v = 0; v < V; ++v) {
            for (int h = 0; h < H; ++h) wrow[h] = bf16_value(w[(size_t)v * H + h]);
            for (int k = 0; k < nrows; ++k) acc[k] = 0.0;
            for (int h = 0; h < H; ++h) {
                const double wv = wrow[h];
                const double *xr = xt + (size_t)h * nrows;
                for (int k = 0; k < nrows; ++k) acc[k] += xr[k] * wv;
            }
            for (int k = 0; k < nrows; ++k) z[(size_t)k * V + v] = acc[k];
        }
        free(wrow);
        free(acc);
    }
    free(xt);
}

/* Per row: argmax (lowest vocab id among equal maxima), the maximum and the second largest value
 * of the row taken as a multiset (equal to the maximum when it occurs twice). */
void oracle_row_top2(int nrows, int V, const double *z, int32_t *arg, double *top1,
                     double *top2) {
    for (int k = 0; k < nrows; ++k) {
        const double *row = z + (size_t)k * V;
        int best = 0;
        for (int v = 1; v < V; ++v)
            if (row[v] > row[best]) best = v;
        double second = -INFINITY;
        for (int v = 0; v < V; ++v)
            if (v != best && row[v] > second) second = row[v];
        arg[k] = best;
        top1[k] = row[best];
        top2[k] = second;
    }
}

/* ---------------------------------------------------------------------------------------------
 * Greedy (T=0) acceptance walk over one request's tree.
 * Start at the root.  While some child c of the current node u carries the token argmax(z_u),
 * accept the lowest-index such child and move to it.  The first node with no matching child
 * stops the walk and argmax there is the bonus token.
 * path[0] = 0 and path[1..a] are the accepted nodes; out_tokens[0..a-1] their tokens and
 * out_tokens[a] the bonus; entries past that are -1 (path has 64 slots, out_tokens 65).
 * Returns a (accepted draft nodes) or OR_EINVAL for a malformed tree.
 * ------------------------------------------------------------------------------------------- */
int oracle_walk_greedy(int n, const int32_t *parent, const int32_t *tokens, const int32_t *arg,
                       int32_t *path, int32_t *out_tokens) {
    uint64_t anc[64];
    int32_t dep[64];
    for (int k = 0; k < 64; ++k) path[k] = -1;
    for (int k = 0; k < 65; ++k) out_tokens[k] = -1;
    if (oracle_ancestry(n, parent, anc, dep) != OR_OK) return OR_EINVAL;
    int u = 0, a = 0;
    path[0] = 0;
    for (;;) {
        int want = arg[u], next = -1;
        for (int c = 1; c < n; ++c)
            if (parent[c] == u && tokens[c] == want) { next = c; break; }
        if (next < 0) break;
        out_tokens[a] = tokens[next];
        ++a;
        path[a] = next;
        u = next;
    }
    out_tokens[a] = arg[u];
    return a;
}

/* ---------------------------------------------------------------------------------------------
 * Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
 * SC'11): ten rounds of two 64x64->128 multiplies on a 4-word counter under a 2-word key, the
 * key bumped by the Weyl constants between rounds.
 * ------------------------------------------------------------------------------------------- */
static void mul128(uint64_t a, uint64_t b, uint64_t *hi, uint64_t *lo) {
    unsigned __int128 p = (unsigned __int128)a * (unsigned __int128)b;
    *hi = (uint64_t)(p >> 64);
    *lo = (uint64_t)p;
}

void oracle_philox4x64(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
    const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
    uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t hi0, lo0, hi1, lo1;
        mul128(M0, c0, &hi0, &lo0);
        mul128(M1, c2, &hi1, &lo1);
        uint64_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += W0;
        k1 += W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The method's seeded uniform in (0,1).  One Philox block (counter (v/8, node, request, stream)
 * under key (seed, step)) gives 4 words of 64 bits; each word holds two 23-bit fields, bits
 * 63..41 and bits 31..9.  Vocab id v takes word (v/2) % 4, the high field for even v and the
 * low field for odd v, centred: U = (field + 0.5) * 2^-23, a value that single precision holds
 * exactly and that lies in [2^-24, 1 - 2^-24].  Streams: 0 the bonus draw's race over vocab ids
 * (node = the stop node), 1 the accept tests (v = 0, node = the child). */
double oracle_uniform(uint64_t seed, uint64_t step, uint32_t r, uint32_t node, uint32_t v,
                      uint32_t stream) {
    uint64_t ctr[4] = {v >> 3, node, r, stream};
    uint64_t key[2] = {seed, step};
    uint64_t out[4];
    oracle_philox4x64(ctr, key, out);
    uint64_t x = out[(v >> 1) & 3u];
    uint64_t field = (v & 1u) ? ((x & 0xFFFFFFFFull) >> 9) : (x >> 41);
    return ((double)field + 0.5) * (1.0 / 8388608.0);
}

/* The bonus draw: an exponential race over weights w (>= 0).  Every id with w_v > 0 gets the
 * key log w_v - log(-log U_v), U_v = oracle_uniform(seed, step, r, node, v, 0); the winner is the
 * largest key, ties to the lowest v.  -log U_v is a standard exponential E_v, and the id with
 * the smallest E_v / w_v is id v with probability w_v / sum w exactly (the minimum of
 * independent exponentials of rates w_v), so the race samples the normalised weights without
 * forming them.  Returns the token, or -1 when no weight is positive; *best_key (nullable)
 * receives the winning key. */
int oracle_race(int V, const double *w, uint64_t seed, uint64_t step, int r, int node,
                double *best_key) {
    int best = -1;
    double bk = -INFINITY;
    for (int v = 0; v < V; ++v) {
        if (!(w[v] > 0.0)) continue;
        double U = oracle_uniform(seed, step, (uint32_t)r, (uint32_t)node, (uint32_t)v, 0);
        double key = log(w[v]) - log(-log(U));
        if (best < 0 || key > bk) { bk = key; best = v; }
    }
    if (best_key) *best_key = bk;
    return best;
}

/* p = softmax(z / T) of one row, in fp64. */
static void softmax_t(int V, const double *z, double T, double *p) {
    double m = -INFINITY;
    for (int v = 0; v < V; ++v) if (z[v] / T > m) m = z[v] / T;
    double s = 0.0;
    for (int v = 0; v < V; ++v) s += exp(z[v] / T - m);
    double lse = m + log(s);
    for (int v = 0; v < V; ++v) p[v] = exp(z[v] / T - lse);
}

/* ---------------------------------------------------------------------------------------------
 * Stochastic (T>0) acceptance over one request that is a chain (parent[k] = k-1).
 * Node k (k >= 1) holds token x_k drafted from q_{k-1}; the target's distribution at node u is
 * p_u = softmax(z_u / T).  Walk k = 1, 2, ...: accept x_k iff U_k * q_{k-1}(x_k) < p_{k-1}(x_k)
 * (U_k = oracle_uniform(seed, step, r, k, 0, 1)).  At the first rejection (stop node u = k-1) the
 * bonus is drawn from norm(max(0, p_u - q_u)); when every node is accepted (u = n-1) it is drawn
 * from p_u.  Both draws are oracle_race at node u.  If the residual has no positive weight
 * (p <= q everywhere, i.e. p = q up to rounding, where exact arithmetic would have accepted the
 * draft) the bonus is drawn from p_u by the same race.
 * z and q are the request's rows [n][V] (q fp32 as given).  info (nullable) receives
 * {stop node, 1 if a rejection happened else 0, 1 if the residual fell back to p}.
 * Returns a, OR_EINVAL for a malformed tree or OR_EUNSUPPORTED for a tree that is not a chain.
 * ------------------------------------------------------------------------------------------- */
int oracle_accept_chain(int n, const int32_t *parent, const int32_t *tokens, const double *z,
                        const float *q, int V, double T, uint64_t seed, uint64_t step, int r,
                        int32_t *path, int32_t *out_tokens, int32_t *info) {
    uint64_t anc[64];
    int32_t dep[64];
    for (int k = 0; k < 64; ++k) path[k] = -1;
    for (int k = 0; k < 65; ++k) out_tokens[k] = -1;
    if (oracle_ancestry(n, parent, anc, dep) != OR_OK) return OR_EINVAL;
    for (int k = 1; k < n; ++k)
        if (parent[k] != k - 1) return OR_EUNSUPPORTED;
    double *p = (double *)malloc(sizeof(double) * (size_t)V);
    double *w = (double *)malloc(sizeof(double) * (size_t)V);
    int a = 0, rejected = 0;
    path[0] = 0;
    for (int k = 1; k < n; ++k) {
        int u = k - 1, x = tokens[k];
        softmax_t(V, z + (size_t)u * V, T, p);
        double qx = (double)q[(size_t)u * V + x];
        double U = oracle_uniform(seed, step, (uint32_t)r, (uint32_t)k, 0, 1);
        if (U * qx < p[x]) {
            out_tokens[a] = x;
            ++a;
            path[a] = k;
        } else {
            rejected = 1;
            break;
        }
    }
    int u = a;  /* stop node: the last accepted node (the root when nothing was accepted) */
    softmax_t(V, z + (size_t)u * V, T, p);
    int fell_back = 0, bonus;
    if (rejected) {
        for (int v = 0; v < V; ++v) {
            double d = p[v] - (double)q[(size_t)u * V + v];
            w[v] = d > 0.0 ? d : 0.0;
        }
        bonus = oracle_race(V, w, seed, step, r, u, NULL);
        if (bonus < 0) {
            /* no positive residual weight: p <= q everywhere, i.e. p = q up to rounding; the
             * bonus is drawn from p, the distribution exact arithmetic would have emitted */
            fell_back = 1;
            bonus = oracle_race(V, p, seed, step, r, u, NULL);
        }
    } else {
        bonus = oracle_race(V, p, seed, step, r, u, NULL);
    }
    out_tokens[a] = bonus;
    if (info) { info[0] = u; info[1] = rejected; info[2] = fell_back; }
    free(p);
    free(w);
    return a;
}

/* ---------------------------------------------------------------------------------------------
 * Round-to-nearest-even of x to bf16 (8 significant bits, fp32's exponent range), returned as
 * bits.  Written from the definition: among the two bf16 values around x, the nearer; on a tie,
 * the one whose last significand bit is 0.  Finite inputs within bf16 range only.
 * ------------------------------------------------------------------------------------------- */
uint16_t oracle_bf16_round(double x) {
    if (x == 0.0) return signbit(x) ? 0x8000u : 0u;
    const double ax = fabs(x);
    int e;
    frexp(ax, &e);                                /* ax = m 2^e, m in [0.5, 1) */
    if (e < -125) e = -125;                        /* subnormal range: fixed spacing 2^-133 */
    const double ulp = ldexp(1.0, e - 8);          /* spacing of bf16 values in [2^(e-1), 2^e) */
    double lo = floor(ax / ulp) * ulp;
    double hi = lo + ulp;
    double r;
    const double dl = ax - lo, dh = hi - ax;
    if (dl < dh) r = lo;
    else if (dh < dl) r = hi;
    else r = fmod(lo / ulp, 2.0) == 0.0 ? lo : hi;
    float f = (float)(x < 0 ? -r : r);             /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------------------------------------
 * Low-rank candidate head (the draft's output layer in the pages: "EAGLE-4 是什麼？...",
 * aiposthub.com, section "EAGLE-4 是什麼？先看推測解碼為什麼能變快": a small matrix screens
 * candidate tokens, then only the few candidates are scored exactly).  For each of M rows h
 * (bf16, [M][H]):
 *   g = h D^T                  D [r][H] bf16: the down projection;
 *   z~ = g U^T                 U [V][r] bf16: approximate logits;
 *   C = the k ids of largest z~ (ties to the lowest id);
 *   z_c = h . W_c for c in C   W [V][H] bf16: exact logits of the candidates;
 * out_ids [M][k]: C ordered by z_c descending (ties to the lowest id), out_logit [M][k] the z_c;
 * kth [M] (nullable): the k-th largest z~; z_approx [M][V] (nullable): z~; g_out [M][r]
 * (nullable): g.  fp64 throughout, on the exact bf16 input values.
 * ------------------------------------------------------------------------------------------- */
void oracle_lowrank_candidates(int M, int H, int V, int r, int k, const uint16_t *hid,
                               const uint16_t *D, const uint16_t *U, const uint16_t *W,
                               int32_t *out_ids, double *out_logit, double *kth,
                               double *z_approx, double *g_out, int nthreads) {
    set_threads(nthreads);
    double *g = (double *)malloc(sizeof(double) * (size_t)M * r);
#pragma omp parallel for schedule(static)
    for (int t = 0; t < M * r; ++t) {
        const int m = t / r, j = t % r;
        double acc = 0.0;
        for (int h = 0; h < H; ++h)
            acc += bf16_value(hid[(size_t)m * H + h]) * bf16_value(D[(size_t)j * H + h]);
        g[t] = acc;
    }
    if (g_out) memcpy(g_out, g, sizeof(double) * (size_t)M * r);
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M; ++m) {
        double *z = (double *)malloc(sizeof(double) * (size_t)V);
        for (int v = 0; v < V; ++v) {
            double acc = 0.0;
            for (int j = 0; j < r; ++j) acc += g[(size_t)m * r + j] * bf16_value(U[(size_t)v * r + j]);
            z[v] = acc;
        }
        if (z_approx) memcpy(z_approx + (size_t)m * V, z, sizeof(double) * (size_t)V);
        /* top-k by z~: repeated selection of the largest remaining (lowest id on ties) */
        int32_t cand[64];
        char *taken = (char *)calloc((size_t)V, 1);
        for (int i = 0; i < k; ++i) {
            int best = -1;
            for (int v = 0; v < V; ++v)
                if (!taken[v] && (best < 0 || z[v] > z[best])) best = v;
            taken[best] = 1;
            cand[i] = best;
        }
        if (kth) kth[m] = z[cand[k - 1]];
        free(taken);
        double ex[64];
        for (int i = 0; i < k; ++i) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += bf16_value(hid[(size_t)m * H + h]) * bf16_value(W[(size_t)cand[i] * H + h]);
            ex[i] = acc;
        }
        /* order by exact logit, descending, lowest id on ties (insertion sort of <= 64) */
        for (int i = 1; i < k; ++i) {
            const int ci = cand[i];
            const double xi = ex[i];
            int j = i - 1;
            while (j >= 0 && (ex[j] < xi || (ex[j] == xi && cand[j] > ci))) {
                ex[j + 1] = ex[j];
                cand[j + 1] = cand[j];
                --j;
            }
            ex[j + 1] = xi;
            cand[j + 1] = ci;
        }
        for (int i = 0; i < k; ++i) {
            out_ids[(size_t)m * k + i] = cand[i];
            out_logit[(size_t)m * k + i] = ex[i];
        }
        free(z);
    }
    free(g);
}

/* ---------------------------------------------------------------------------------------------
 * Stochastic (T>0) acceptance over a general tree: multi-candidate speculative sampling (the
 * multi-step rule of SpecInfer, Miao et al., "SpecInfer: Accelerating Large Language Model Serving
 * with Tree-based Speculative Inference and Verification", 2023, restated here).
 *
 * The children c_1 < c_2 < ... of node u carry tokens x_i drafted independently from q_u.  The
 * running target starts at r = p_u = softmax(z_u / T).  Child c_i is accepted iff
 * U_i * q_u(x_i) < r(x_i), with U_i = oracle_uniform(seed, step, r, c_i, 0, 1) (the chain rule's
 * stream, keyed by the child); acceptance moves the walk to c_i, whose own target restarts at its
 * p.  A rejection replaces r by norm(max(0, r - q_u)).  Every such residual has the closed form
 *     r_i = max(0, p_u - c_i q_u) / N(c_i),   N(c) = sum_v max(0, p_u(v) - c q_u(v)),
 *     c_0 = 0, N(c_0) = 1,  c_{i+1} = c_i + N(c_i),
 * since max(0, r_i - q_u) = max(0, p_u - (c_i + N(c_i)) q_u) / N(c_i) wherever it is positive.
 * With candidates drawn independently from q_u, each step is an exact speculative-sampling step
 * from the current residual, so the emitted token follows p_u.
 *
 * The walk stops at a node with no children or whose children are all rejected; the bonus is
 * then drawn with oracle_race at that node from the weights max(0, p_u - c q_u) (c = 0 when no
 * child was rejected: the weights are p_u).  If a rejection leaves N(c) = 0 (the running target
 * equalled q up to rounding; probability zero in exact arithmetic) the walk stops there and the
 * bonus is drawn from p_u by the same race, as in the chain rule.  On a chain this is exactly
 * oracle_accept_chain (c = 1 after the single rejection).
 *
 * z and q are the request's rows [n][V].  info (nullable): {stop node, rejections at the stop
 * node, 1 if the fallback was taken}; c_out (nullable): the c of the bonus draw.
 * Returns a, or OR_EINVAL for a malformed tree or a token outside [0, V).
 * ------------------------------------------------------------------------------------------- */
int oracle_accept_tree(int n, const int32_t *parent, const int32_t *tokens, const double *z,
                       const float *q, int V, double T, uint64_t seed, uint64_t step, int r,
                       int32_t *path, int32_t *out_tokens, int32_t *info, double *c_out) {
    uint64_t anc[64];
    int32_t dep[64];
    for (int k = 0; k < 64; ++k) path[k] = -1;
    for (int k = 0; k < 65; ++k) out_tokens[k] = -1;
    if (oracle_ancestry(n, parent, anc, dep) != OR_OK) return OR_EINVAL;
    for (int k = 1; k < n; ++k)
        if (tokens[k] < 0 || tokens[k] >= V) return OR_EINVAL;
    double *p = (double *)malloc(sizeof(double) * (size_t)V);
    double *w = (double *)malloc(sizeof(double) * (size_t)V);
    int u = 0, a = 0, nrej = 0, fell_back = 0;
    double c = 0.0;
    path[0] = 0;
    for (;;) {
        softmax_t(V, z + (size_t)u * V, T, p);
        const float *qu = q + (size_t)u * V;
        double Nc = 1.0;
        int next = -1;
        c = 0.0;
        nrej = 0;
        for (int j = u + 1; j < n && !fell_back; ++j) {
            if (parent[j] != u) continue;
            const int x = tokens[j];
            const double qx = (double)qu[x];
            double rx = p[x] - c * qx;
            rx = rx > 0.0 ? rx / Nc : 0.0;
            const double U = oracle_uniform(seed, step, (uint32_t)r, (uint32_t)j, 0, 1);
            if (U * qx < rx) {
                next = j;
                break;
            }
            ++nrej;
            c += Nc;
            Nc = 0.0;
            for (int v = 0; v < V; ++v) {
                const double d = p[v] - c * (double)qu[v];
                if (d > 0.0) Nc += d;
            }
            if (!(Nc > 0.0)) fell_back = 1;
        }
        if (next < 0) break;
        out_tokens[a] = tokens[next];
        ++a;
        path[a] = next;
        u = next;
    }
    int bonus = -1;
    if (!fell_back) {
        const float *qu = q + (size_t)u * V;
        for (int v = 0; v < V; ++v) {
            const double d = p[v] - c * (double)qu[v];
            w[v] = d > 0.0 ? d : 0.0;
        }
        bonus = oracle_race(V, w, seed, step, r, u, NULL);
        if (bonus < 0) fell_back = 1;
    }
    if (fell_back) bonus = oracle_race(V, p, seed, step, r, u, NULL);
    out_tokens[a] = bonus;
    if (info) { info[0] = u; info[1] = nrej; info[2] = fell_back; }
    if (c_out) *c_out = c;
    free(p);
    free(w);
    return a;
}

/* ---------------------------------------------------------------------------------------------
 * KV compaction.  For every layer l and request r with a = accept_len[r]:
 *   cache[l][slot_base[r] + kv_len[r] + k] <- tree[l][cu_nodes[r] + path[r][k]],  k = 0..a,
 * for K and V (path[r][0] is the root), and kv_len_out[r] = kv_len[r] + a + 1.  A request whose
 * rows would pass slot_cap[r] is left untouched (kv_len_out = kv_len) and the call returns
 * OR_ENOSPACE; a path entry outside the request's nodes gives OR_EINVAL the same way.
 * Rows are [hkv][d] bf16; strides are in elements.
 * ------------------------------------------------------------------------------------------- */
int oracle_kv_compact(int B, const int32_t *cu_nodes, const int32_t *kv_len,
                      const int64_t *slot_base, const int32_t *slot_cap,
                      const int32_t *accept_len, const int32_t *path, const uint16_t *k_tree,
                      const uint16_t *v_tree, uint16_t *k_cache, uint16_t *v_cache, int n_layers,
                      int64_t tree_layer_stride, int64_t cache_layer_stride, int hkv, int d,
                      int32_t *kv_len_out) {
    int status = OR_OK;
    const size_t row = (size_t)hkv * d;
    for (int r = 0; r < B; ++r) {
        int a = accept_len[r];
        int n = cu_nodes[r + 1] - cu_nodes[r];
        kv_len_out[r] = kv_len[r];
        if (a < 0 || a >= n || a > 63) { status = OR_EINVAL; continue; }
        if ((int64_t)kv_len[r] + a + 1 > (int64_t)slot_cap[r]) { status = OR_ENOSPACE; continue; }
        int bad = 0;
        for (int k = 0; k <= a; ++k) {
            int j = path[(size_t)r * 64 + k];
            if (j < 0 || j >= n) bad = 1;
        }
        if (bad) { status = OR_EINVAL; continue; }
        for (int l = 0; l < n_layers; ++l)
            for (int k = 0; k <= a; ++k) {
                int j = path[(size_t)r * 64 + k];
                size_t src = (size_t)l * tree_layer_stride + (size_t)(cu_nodes[r] + j) * row;
                size_t dst = (size_t)l * cache_layer_stride
                           + (size_t)(slot_base[r] + kv_len[r] + k) * row;
                memcpy(k_cache + dst, k_tree + src, row * sizeof(uint16_t));
                memcpy(v_cache + dst, v_tree + src, row * sizeof(uint16_t));
            }
        kv_len_out[r] = kv_len[r] + a + 1;
    }
    return status;
}

/* ---------------------------------------------------------------------------------------------
 * Batched forms of the two definitions above, for statistical checks over many requests:
 * request r (0-based) uses rows cu_nodes[r] .. cu_nodes[r+1]-1 of z and q, and its own index r in
 * the uniforms' counter.  Per-request results as in oracle_accept_chain (path [B][64],
 * out_tokens [B][65], info [B][3]); accept_len[r] holds a or the error code.
 * ------------------------------------------------------------------------------------------- */
void oracle_accept_chain_batch(int B, const int32_t *cu_nodes, const int32_t *parent,
                               const int32_t *tokens, const double *z, const float *q, int V,
                               double T, uint64_t seed, uint64_t step, int32_t *accept_len,
                               int32_t *path, int32_t *out_tokens, int32_t *info, int nthreads) {
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 64)
    for (int r = 0; r < B; ++r) {
        int a0 = cu_nodes[r], n = cu_nodes[r + 1] - cu_nodes[r];
        accept_len[r] = oracle_accept_chain(n, parent + a0, tokens + a0, z + (size_t)a0 * V,
                                            q + (size_t)a0 * V, V, T, seed, step, r,
                                            path + (size_t)r * 64, out_tokens + (size_t)r * 65,
                                            info + (size_t)r * 3);
    }
}

/* Batched oracle_accept_tree, laid out like oracle_accept_chain_batch; c_out [B]. */
void oracle_accept_tree_batch(int B, const int32_t *cu_nodes, const int32_t *parent,
                              const int32_t *tokens, const double *z, const float *q, int V,
                              double T, uint64_t seed, uint64_t step, int32_t *accept_len,
                              int32_t *path, int32_t *out_tokens, int32_t *info, double *c_out,
                              int nthreads) {
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 64)
    for (int r = 0; r < B; ++r) {
        int a0 = cu_nodes[r], n = cu_nodes[r + 1] - cu_nodes[r];
        accept_len[r] = oracle_accept_tree(n, parent + a0, tokens + a0, z + (size_t)a0 * V,
                                           q + (size_t)a0 * V, V, T, seed, step, r,
                                           path + (size_t)r * 64, out_tokens + (size_t)r * 65,
                                           info + (size_t)r * 3, c_out + r);
    }
}

/* n races over the same weights, race k using request index r0 + k and the given node. */
void oracle_race_many(int n, int V, const double *w, uint64_t seed, uint64_t step, int r0,
                      int node, int32_t *out, int nthreads) {
    set_threads(nthreads);
#pragma omp parallel for schedule(static)
    for (int k = 0; k < n; ++k) out[k] = oracle_race(V, w, seed, step, r0 + k, node, NULL);
}
