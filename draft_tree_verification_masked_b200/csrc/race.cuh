// race.cuh -- the bonus draw's exponential race over vocab ids, shared by the draw-pass GEMM
// epilogue (lmhead.cu) and the draw over materialised logit rows (accept.cu).
//
// After the target rejects a draft (or accepts all of them) it emits one token of its own, drawn
// so that the emitted token follows the target's distribution ("Eagle-4 Released: Outpaces
// DFlash2 and DSpark ...", section "Technical Background").  The draw is an exponential race:
// every id with weight w_v > 0 gets the key w_v / E_v, E_v = -log U_v a standard exponential
// (U_v the stream-0 uniform of (id, stop node, request)), and the largest key wins, the lower id
// on equal keys; the winner is id v with probability w_v / sum w.  Two races run side by side:
// over the residual w = max(0, p - c q) (c > 0) and over p itself (the draw when nothing was
// rejected, and the answer when the residual has no positive weight).
#pragma once
#include "common.cuh"
#include "philox.cuh"

namespace etree {

// Screening margin: an id is skipped only when its key is certainly below the threshold,
// allowing for the rounding of -log U (a few ulp) and of the quotient.
constexpr float kRaceShrink = 1.0f - 1.0f / 1048576.0f;

// The race over the 8 ids c0 .. c0+7 (c0 a multiple of 8) with logits z[0..7] and draft
// probabilities q[0..7] (read only when c > 0).  p_v = 2^(z_v k_log2 - L2).  (kr, ir) and (kp, ip)
// are the residual's and p's leaders so far (key -inf and id -1 when none); thr_r and thr_p the
// screening thresholds: since E_v >= 1 - U_v, an id whose weight is below thr * (1 - U_v) cannot
// beat thr and skips the logarithm.  A threshold is at most the row's final maximum key (the
// caller builds it from keys of real ids, shrunk by kRaceShrink).
__device__ __forceinline__ void race8(const float* z, const float* q, int c0, int V, float k_log2,
                                      float L2, float c, uint64_t seed, uint64_t step,
                                      uint32_t node, uint32_t req, float& thr_r, float& thr_p,
                                      float& kr, int& ir, float& kp, int& ip) {
  const bool resid = c > 0.f;
  float u[8];
  uniforms8(seed, step, (uint32_t)(c0 >> 3), node, req, 0u, u);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int v = c0 + e;
    if (v >= V) break;
    const float pv = exp2f(z[e] * k_log2 - L2);
    const float wr = resid ? fmaxf(pv - c * q[e], 0.f) : 0.f;
    const float d = 1.f - u[e];                        // exact: U has 24 significant bits
    const bool cp = pv > 0.f && pv >= thr_p * d;
    const bool cr = wr > 0.f && wr >= thr_r * d;
    if (cp || cr) {
      const float E = -logf(u[e]);
      if (cp) {
        const float key = __fdiv_rn(pv, E);
        if (key > kp) {
          kp = key;
          ip = v;
          thr_p = fmaxf(thr_p, key * kRaceShrink);
        }
      }
      if (cr) {
        const float key = __fdiv_rn(wr, E);
        if (key > kr) {
          kr = key;
          ir = v;
          thr_r = fmaxf(thr_r, key * kRaceShrink);
        }
      }
    }
  }
}

}  // namespace etree
