// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
// SC'11) and the uniforms of the acceptance rule, device side.
//
// One round maps counter (c0, c1, c2, c3) and key (k0, k1) to
//   (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0))
// and then adds the Weyl constants to the key; ten rounds.
//
// Counter layout of the verify step: (c0, r, step_lo, purpose), r = logit row.
//   acceptance uniform of row r: c0 = 0, purpose 0, u = (word0 >> 8) * 2^-24 in [0, 1)
//   token uniform of token v:   c0 = v >> 1, the 64-bit word (word[2(v&1)+1] : word[2(v&1)]),
//                               V = its 24 leading significant bits scaled into (0, 1)
#pragma once

#include <stdint.h>

namespace sdv {

struct Philox4 {
  uint32_t x, y, z, w;
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    // one 32 x 32 -> 64-bit product gives both halves
    const uint64_t p0 = (uint64_t)kM0 * c0, p1 = (uint64_t)kM1 * c2;
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += kW0;
    k1 += kW1;
  }
  return Philox4{c0, c1, c2, c3};
}

__device__ __forceinline__ float accept_uniform(uint64_t seed, uint32_t step, uint32_t row) {
  const Philox4 o = philox4x32_10(0u, row, step, 0u, (uint32_t)seed, (uint32_t)(seed >> 32));
  return (float)(o.x >> 8) * 0x1.0p-24f;
}

// 24 leading significant bits of a 64-bit word, scaled so the result lies in (0, 1); 0 -> 0.
// Converting the word to float32 rounding toward zero keeps exactly its 24 leading significant
// bits, m * 2^(40-n) (n leading zeros); the power-of-two scale 2^-64 is exact (the result,
// at least 2^-88, stays normal).
__device__ __forceinline__ float float_uniform64(uint64_t w) {
  return __ull2float_rz(w) * 0x1.0p-64f;
}

// Token uniforms of tokens 2*c and 2*c+1 of a row (one Philox call).
__device__ __forceinline__ void token_uniform_pair(uint64_t seed, uint32_t step, uint32_t row,
                                                   uint32_t purpose, uint32_t c, float &v_even,
                                                   float &v_odd) {
  const Philox4 o = philox4x32_10(c, row, step, purpose, (uint32_t)seed, (uint32_t)(seed >> 32));
  v_even = float_uniform64(((uint64_t)o.y << 32) | o.x);
  v_odd = float_uniform64(((uint64_t)o.w << 32) | o.z);
}

}  // namespace sdv
