// philox.cuh -- Philox4x64-10 counter-based generator (Salmon, Moraes, Dror, Shaw, "Parallel
// Random Numbers: As Easy as 1, 2, 3", SC'11), and the seeded uniforms of the acceptance rule.
#pragma once
#include <stdint.h>

namespace etree {

__device__ __forceinline__ void philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3,
                                              uint64_t k0, uint64_t k1, uint64_t (&out)[4]) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint64_t lo0 = 0xD2E7470EE14C6C93ull * c0;
    const uint64_t hi0 = __umul64hi(0xD2E7470EE14C6C93ull, c0);
    const uint64_t lo1 = 0xCA5A826395121157ull * c2;
    const uint64_t hi1 = __umul64hi(0xCA5A826395121157ull, c2);
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += 0x9E3779B97F4A7C15ull;
    k1 += 0xBB67AE8584CAA73Bull;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

// The eight uniforms of vocab ids 8*vb .. 8*vb+7 at (node, request, stream) under (seed, step):
// each 64-bit output word holds two 23-bit fields, bits 63..41 (even id) and bits 31..9 (odd
// id), centred: U = (field + 0.5) * 2^-23.  Single precision holds every such value exactly,
// and all lie in [2^-24, 1 - 2^-24], so -log U is finite and positive.
__device__ __forceinline__ void uniforms8(uint64_t seed, uint64_t step, uint32_t vb, uint32_t node,
                                          uint32_t req, uint32_t stream, float (&u)[8]) {
  uint64_t w[4];
  philox4x64_10(vb, node, req, stream, seed, step, w);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    u[2 * i] = (static_cast<float>(static_cast<uint32_t>(w[i] >> 41)) + 0.5f) * (1.0f / 8388608.0f);
    u[2 * i + 1] =
        (static_cast<float>(static_cast<uint32_t>(w[i]) >> 9) + 0.5f) * (1.0f / 8388608.0f);
  }
}

}  // namespace etree
