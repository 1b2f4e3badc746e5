// Seeded Gumbel-max sampling over a support (xorl issue #71, section 3: the
// sampling program ends in a "seeded gumbel" step).  The pages fix neither
// the generator nor the noise recipe; the one implemented here:
//
//   score_ij = fl32(l_ij / T_i) + G_ij,   G_ij = -log(-log U_ij)      (fp32)
//   y_i      = argmax over j in S_i of score_ij, the smallest j on ties
//   U_ij     = (bits 63..40 of r + 1/2) 2^-24,  r = word (j mod 4) of
//              Philox4x64-10(counter = (floor(j / 4), 0, 0, 0), key = (seed, i))
//
// Every floating-point step is a single IEEE round-to-nearest operation
// (explicit _rn intrinsics, nothing contracted into a fused multiply-add),
// so the decision does not depend on the compiler.
#pragma once

#include <stdint.h>

namespace vs {

// Philox4x64 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011): per round the two Philox-4x64
// multipliers take words 0 and 2 to 128-bit products, whose high halves are
// xored with words 1 and 3 and the round key; the key advances by the two
// Weyl constants between rounds.
__device__ __forceinline__ void philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3,
                                              uint64_t k0, uint64_t k1, uint64_t (&w)[4]) {
  constexpr uint64_t kM0 = 0xD2E7470EE14C6C93ull, kM1 = 0xCA5A826395121157ull;
  constexpr uint64_t kW0 = 0x9E3779B97F4A7C15ull, kW1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint64_t hi0 = __umul64hi(kM0, c0), lo0 = kM0 * c0;
    const uint64_t hi1 = __umul64hi(kM1, c2), lo1 = kM1 * c2;
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  w[0] = c0;
  w[1] = c1;
  w[2] = c2;
  w[3] = c3;
}

// Natural logarithm of a positive normal fp32 value, one fixed sequence of
// rounded operations: x = m 2^e with m in [sqrt(1/2), sqrt(2)); log m =
// 2 atanh(s), s = (m - 1) / (m + 1), from the series 2 (s + s^3/3 + s^5/5 +
// s^7/7 + s^9/9); e ln 2 with ln 2 split into a head whose products are
// exact and a tail (Cody and Waite's argument reduction).
__device__ __forceinline__ float gumbel_log(float x) {
  const uint32_t b = __float_as_uint(x);
  int e = static_cast<int>(b >> 23) - 127;
  float m = __uint_as_float((b & 0x007FFFFFu) | 0x3F800000u);
  if (m > 1.41421356f) {
    m = __fmul_rn(m, 0.5f);
    e += 1;
  }
  const float f = __fsub_rn(m, 1.0f);
  const float s = __fdiv_rn(f, __fadd_rn(f, 2.0f));
  const float z = __fmul_rn(s, s);
  float t = 1.0f / 9.0f;
  t = __fmul_rn(t, z);
  t = __fadd_rn(t, 1.0f / 7.0f);
  t = __fmul_rn(t, z);
  t = __fadd_rn(t, 1.0f / 5.0f);
  t = __fmul_rn(t, z);
  t = __fadd_rn(t, 1.0f / 3.0f);
  const float s2 = __fmul_rn(s, 2.0f);
  const float lm = __fadd_rn(s2, __fmul_rn(s2, __fmul_rn(z, t)));
  const float ef = static_cast<float>(e);
  const float tail = __fadd_rn(__fmul_rn(ef, 1.42860677e-06f), lm);  // ln 2 - head
  return __fadd_rn(__fmul_rn(ef, 0.693145751953125f), tail);         // head 0x3F317200
}

// G for one Philox word.
__device__ __forceinline__ float gumbel_of(uint64_t r) {
  const float u = __fmul_rn(__fadd_rn(static_cast<float>(r >> 40), 0.5f), 5.9604644775390625e-08f);
  return -gumbel_log(-gumbel_log(u));
}

// The four G of tokens 4q .. 4q + 3 of row `row`.
__device__ __forceinline__ void gumbel4(uint64_t seed, uint32_t row, uint64_t q, float (&g)[4]) {
  uint64_t w[4];
  philox4x64_10(q, 0, 0, 0, seed, row, w);
#pragma unroll
  for (int i = 0; i < 4; ++i) g[i] = gumbel_of(w[i]);
}

// Candidate key: larger score first, then the smaller token id (a larger
// key wins an unsigned max); 0 means no candidate.
__device__ __forceinline__ unsigned long long gumbel_key(float score, int32_t j) {
  const uint32_t b = __float_as_uint(score);
  const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<unsigned long long>(ord) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(j));
}
__device__ __forceinline__ int32_t gumbel_key_id(unsigned long long k) {
  return k == 0ull ? -1 : static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k));
}

// Score of token j with logit value x (fp32) at temperature T.
__device__ __forceinline__ float gumbel_score(float x, float T, float g) {
  return __fadd_rn(__fdiv_rn(x, T), g);
}

// Block-wide max of candidate keys (every thread gets it); scratch holds
// one entry per warp.
__device__ __forceinline__ unsigned long long block_max_key(unsigned long long k,
                                                            unsigned long long* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long t = __shfl_xor_sync(0xffffffffu, k, o);
    k = t > k ? t : k;
  }
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = k;
  cta_sync();
  unsigned long long m = 0ull;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) m = scratch[w] > m ? scratch[w] : m;
  cta_sync();
  return m;
}

}  // namespace vs
