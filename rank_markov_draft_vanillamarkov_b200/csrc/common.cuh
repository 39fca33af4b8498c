// Shared device helpers of the Markov-head kernels: element conversion, the
// packed argmax key, the device status word and Philox4x32-10.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dspark_markov.h"

namespace dspark {

// ---------------------------------------------------------------------------
// Element conversion. Corrected logits are rounded once, round-to-nearest-even.
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---------------------------------------------------------------------------
// Argmax key: the score's bits mapped to an unsigned order in the high word and
// the complement of the vocabulary id in the low word, so that the largest key
// is the largest score and, among equal scores, the lowest id. NaN is made a
// single positive quiet NaN, which orders above +inf; -0 is made +0 so that
// the two zeros tie, as they compare equal.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t orderable_bits(float s) {
  uint32_t b = __float_as_uint(s);
  if (s != s) b = 0x7fc00000u;
  if (s == 0.0f) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ unsigned long long pack_key(float score, uint32_t v) {
  return ((unsigned long long)orderable_bits(score) << 32) | (unsigned long long)(0xffffffffu - v);
}

__device__ __forceinline__ uint32_t key_token(unsigned long long key) {
  return 0xffffffffu - (uint32_t)(key & 0xffffffffull);
}

__device__ __forceinline__ void report_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
// as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplies per round, the
// key advanced by two Weyl constants between rounds.
// ---------------------------------------------------------------------------
struct Philox4 {
  uint32_t x, y, z, w;
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    // Each multiply is one 32 x 32 -> 64-bit product (high and low words together).
    const uint64_t p0 = (uint64_t)c0 * 0xD2511F53u;
    const uint64_t p1 = (uint64_t)c2 * 0xCD9E8D57u;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0, n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    c0 = n0;
    c1 = (uint32_t)p1;
    c2 = n2;
    c3 = (uint32_t)p0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return Philox4{c0, c1, c2, c3};
}

// The same generator with its ten round keys given: round_keys[2i] and
// round_keys[2i+1] are (k0, k1) after i Weyl steps. Kernels whose key is fixed
// for the launch receive them precomputed (round_keys_for below), as kernel
// parameters, so the rounds need no key arithmetic.
struct PhiloxRoundKeys {
  uint32_t k[20];
};

__host__ __device__ inline PhiloxRoundKeys round_keys_for(uint64_t seed) {
  PhiloxRoundKeys r;
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  for (int i = 0; i < 10; ++i) {
    r.k[2 * i] = k0;
    r.k[2 * i + 1] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return r;
}

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 const PhiloxRoundKeys& rk) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const uint64_t p0 = (uint64_t)c0 * 0xD2511F53u;
    const uint64_t p1 = (uint64_t)c2 * 0xCD9E8D57u;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ rk.k[2 * i], n2 = (uint32_t)(p0 >> 32) ^ c3 ^ rk.k[2 * i + 1];
    c0 = n0;
    c1 = (uint32_t)p1;
    c2 = n2;
    c3 = (uint32_t)p0;
  }
  return Philox4{c0, c1, c2, c3};
}

__device__ __forceinline__ uint32_t philox_word(const Philox4& p, uint32_t i) {
  return i == 0 ? p.x : i == 1 ? p.y : i == 2 ? p.z : p.w;
}

// u = (2 * (w >> 9) + 1) * 2^-24 lies strictly inside (0, 1) and is exact in
// binary32. It is formed without an integer-to-float conversion: the top 23
// bits of w as the mantissa of a number in [1, 2) give 1 + m 2^-23, and
// subtracting 1 - 2^-24 leaves (2m + 1) 2^-24, which is representable, so the
// subtraction is exact.
__device__ __forceinline__ float uniform_from_word(uint32_t w) {
  return __uint_as_float(0x3F800000u | (w >> 9)) - 0.999999940395355224609375f;
}

// e = -ln u for such a u, accurate relative to e itself (e is as small as
// 6e-8 for u near 1, and those draws are the likely winners). With d = 1 - u,
// which is exact (u is a multiple of 2^-24 in (0, 1)):
//   d < 1/16:  the Taylor series -ln(1 - d) = d + d^2/2 + d^3/3 + d^4/4 + d^5/5
//              + ..., whose remainder is below d^6 / (6 (1 - d)), i.e. under
//              2e-7 of e;
//   otherwise: -ln 2 * log2(u) with the hardware log2 approximation, whose
//              absolute error (about 2^-22 in log2) is under 3e-6 of e >= 0.0645.
__device__ __forceinline__ float neg_log_uniform(float u) {
  const float d = 1.0f - u;
  const float series = d * fmaf(d, fmaf(d, fmaf(d, fmaf(d, 0.2f, 0.25f), 0.333333343f), 0.5f), 1.0f);
  const float via_log2 = __log2f(u) * -0.693147182f;
  return d < 0.0625f ? series : via_log2;
}

// The Gumbel variate g = -ln(e), e = -ln u. The outer log needs only a small
// absolute error (e lies in [6e-8, 16.7]), which the hardware log2 gives:
// |g - exact| stays below about 5e-6 over all 2^23 possible u.
__device__ __forceinline__ float gumbel_from_word(uint32_t w) {
  return __log2f(neg_log_uniform(uniform_from_word(w))) * -0.693147182f;
}

__device__ __forceinline__ float noise_for(uint64_t seed, uint32_t b, uint32_t k, uint32_t v) {
  const Philox4 p = philox4x32_10(v >> 2, k, b, 0u, (uint32_t)seed, (uint32_t)(seed >> 32));
  return gumbel_from_word(philox_word(p, v & 3u));
}

}  // namespace dspark
