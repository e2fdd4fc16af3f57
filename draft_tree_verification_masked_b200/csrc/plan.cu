// plan.cu -- hardware-aware draft-tree sizing from measured verification costs (host code).
//
// The size of the draft tree follows the measured cost of drafting and verifying at the running
// batch size, hardware and workload: a calibration measures the costs, and the serving rounds
// narrow the verification width as the batch grows ("EAGLE-4 官方推理代码发布 ...",
// arex-research.com, section "投机树多大，由实测成本决定"; "EAGLE-4 是什麼？...", aiposthub.com,
// section "EAGLE-4 是什麼？先看推測解碼為什麼能變快": the harness times draft and verification at
// warm-up and then picks how many tokens and branches to guess).  This file holds the
// verification side of that decision:
//
//  * etree_verify_cost: the step time at (B, N, L) by piecewise-linear interpolation of a
//    calibrated cost table (calibrate.py), extended linearly past the grid's ends;
//  * etree_plan_tree: the static tree shape (depth, width) that maximises expected tokens per
//    second under a stated acceptance model (include/etree.h).
#include <cmath>
#include <cstring>

#include "etree.h"

namespace {

// Index i and weight f of x on the ascending grid g[0..n): x ~ g[i] + f (g[i+1] - g[i]); f may
// leave [0, 1] past the ends (linear extension of the first / last segment).
void locate(const int32_t* g, int n, double x, int* i, double* f) {
  if (n == 1) {
    *i = 0;
    *f = 0.0;
    return;
  }
  int k = 0;
  while (k + 2 < n && x > g[k + 1]) ++k;
  *i = k;
  *f = (x - g[k]) / (double)(g[k + 1] - g[k]);
}

bool ascending(const int32_t* g, int n) {
  for (int k = 0; k + 1 < n; ++k)
    if (!(g[k] < g[k + 1])) return false;
  return n >= 1;
}

double at(const etree_cost_table* t, int i, int j, int k) {
  return (double)t->us[((size_t)i * t->nN + j) * t->nL + k];
}

}  // namespace

extern "C" etree_status etree_verify_cost(const etree_cost_table* t, double B, double N,
                                          double L, double* us_out) {
  if (!t || !us_out || !t->B || !t->N || !t->L || !t->us || t->nB < 1 || t->nN < 1 ||
      t->nL < 1)
    return ETREE_EINVAL;
  if (!ascending(t->B, t->nB) || !ascending(t->N, t->nN) || !ascending(t->L, t->nL))
    return ETREE_EINVAL;
  int ib, in, il;
  double fb, fn, fl;
  locate(t->B, t->nB, B, &ib, &fb);
  locate(t->N, t->nN, N, &in, &fn);
  locate(t->L, t->nL, L, &il, &fl);
  // trilinear over the cell's corners (a single-point axis has weight 1 on its point)
  double acc = 0.0;
  for (int db = 0; db < (t->nB > 1 ? 2 : 1); ++db)
    for (int dn = 0; dn < (t->nN > 1 ? 2 : 1); ++dn)
      for (int dl = 0; dl < (t->nL > 1 ? 2 : 1); ++dl) {
        const double w = (t->nB > 1 ? (db ? fb : 1.0 - fb) : 1.0) *
                         (t->nN > 1 ? (dn ? fn : 1.0 - fn) : 1.0) *
                         (t->nL > 1 ? (dl ? fl : 1.0 - fl) : 1.0);
        acc += w * at(t, ib + db, in + dn, il + dl);
      }
  *us_out = acc > 0.0 ? acc : 0.0;
  return ETREE_OK;
}

extern "C" etree_status etree_plan_tree(const etree_cost_table* t, int32_t B, int32_t L,
                                        const float* acc_rank, int32_t n_rank,
                                        float draft_us_per_level, float draft_us_fixed,
                                        int32_t max_depth, int32_t max_width,
                                        int32_t max_nodes, etree_tree_plan* out) {
  if (!out || !acc_rank || B < 1 || L < 0 || n_rank < 1 || max_depth < 0 || max_depth > 63 ||
      max_width < 1 || max_width > 64 || max_nodes < 1 || max_nodes > ETREE_MAX_NODES ||
      !(draft_us_per_level >= 0.f) || !(draft_us_fixed >= 0.f))
    return ETREE_EINVAL;
  double mass = 0.0;
  for (int k = 0; k < n_rank; ++k) {
    if (!(acc_rank[k] >= 0.f)) return ETREE_EINVAL;
    mass += acc_rank[k];
  }
  if (mass > 1.0 + 1e-6) return ETREE_EINVAL;
  bool have = false;
  etree_tree_plan best{};
  for (int d = 0; d <= max_depth; ++d) {
    for (int w = 1; w <= (d == 0 ? 1 : max_width); ++w) {
      const int nodes = 1 + d * w;
      if (nodes > max_nodes) break;
      // spine candidate (rank 1) continues the walk; ranks 2..w are leaves beside it
      const double s = acc_rank[0];
      double side = 0.0;
      for (int k = 1; k < w && k < n_rank; ++k) side += acc_rank[k];
      double e = 0.0, reach = 1.0;                    // reach = P(level j is tested)
      for (int j = 1; j <= d; ++j) {
        e += reach * (s + side);
        reach *= s;
      }
      double vus;
      const etree_status st = etree_verify_cost(t, (double)B, (double)nodes, (double)L, &vus);
      if (st) return st;
      const double step = (d > 0 ? (double)draft_us_fixed + d * (double)draft_us_per_level : 0.0)
                          + vus;
      const double tps = step > 0.0 ? (double)B * (e + 1.0) / step * 1e6 : 0.0;
      // more tokens/s wins; within 1e-12 relative, fewer nodes, then fewer levels
      const bool better = have && tps > best.tokens_per_s * (1.0 + 1e-12);
      const bool tie = have && !better && tps >= best.tokens_per_s * (1.0 - 1e-12) &&
                       (nodes < best.nodes || (nodes == best.nodes && d < best.depth));
      if (!have || better || tie) {
        have = true;
        best.depth = d;
        best.width = w;
        best.nodes = nodes;
        best.expected_accept = e;
        best.step_us = step;
        best.tokens_per_s = tps;
      }
    }
  }
  *out = best;
  return ETREE_OK;
}
