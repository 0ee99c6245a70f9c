// kvq_quant.cuh -- per-group quantisation of rotated, lambda-scaled channels to
// signed int4 or int8 ("When Quantization Is Free", gist.science/de/paper/2605.05699,
// "Methodik" 2: per-group abs-max scale, rounding to signed int4/int8, nibble packing).
//
// int4: scale = fp16_rn(min(absmax / 7, 65504)); code = clamp(rint(y / scale), -7, 7)
// (0 where the scale is 0), two's-complement nibbles, even channel in the low
// nibble. The rounding is the fp32 "magic number" FMA: y * (1/scale) + (1.5 * 2^23
// + 8) leaves code + 8 in the low four mantissa bits (round to nearest even), so
// packing is integer shifts and a byte permute.
// int8: the same with 127 in place of 7 and 1.5 * 2^23 + 128 (code + 128 in the low
// byte), one two's-complement byte per channel.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_ptx.cuh"

namespace kvq {

constexpr float kMagic = 12582920.0f;    // 1.5 * 2^23 + 8: bits = 0x4B400008 + code
constexpr float kMagicLo = 12582913.0f;  // code -7
constexpr float kMagicHi = 12582927.0f;  // code +7

// max |y_i| (max is exact, so the order of the reduction does not matter): a tree
// of three-input maxima, the first level on absolute values.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
  float d;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
template <int G>
__device__ __forceinline__ float absmax(const float (&y)[G]) {
  static_assert(G == 16 || G == 32, "group size");
  constexpr int L1 = (G + 2) / 3;  // 11 (G = 32) or 6 (G = 16)
  float m[L1];
#pragma unroll
  for (int i = 0; i < G / 3; ++i) m[i] = max3_abs(y[3 * i], y[3 * i + 1], y[3 * i + 2]);
  if constexpr (G % 3 == 2) m[L1 - 1] = fmaxf(fabsf(y[G - 2]), fabsf(y[G - 1]));
  if constexpr (G % 3 == 1) m[L1 - 1] = fabsf(y[G - 1]);
  // 11 -> 4 -> 2 -> 1, or 6 -> 2 -> 1
  if constexpr (L1 == 11) {
    const float a0 = max3(m[0], m[1], m[2]), a1 = max3(m[3], m[4], m[5]), a2 = max3(m[6], m[7], m[8]);
    const float a3 = fmaxf(m[9], m[10]);
    return fmaxf(max3(a0, a1, a2), a3);
  } else {
    return fmaxf(max3(m[0], m[1], m[2]), max3(m[3], m[4], m[5]));
  }
}

// a / Q for a >= 0 and a constant Q, correctly rounded without a branch: Markstein's
// correction of the quotient through the correctly rounded reciprocal y = RN(1/Q),
// q0 = RN(a y), r = a - Q q0 (exact by the fma), q = RN(q0 + r y). (Checked exhaustively
// against exact rational division on 124 K fp32 values, including neighbours of multiples
// of Q, for Q = 7 and 127.)
template <int Q>
__device__ __forceinline__ float div_by_const(float a) {
  constexpr float y = 1.0f / Q;
  const float q0 = a * y;
  const float r = fmaf(-static_cast<float>(Q), q0, a);
  return fmaf(r, y, q0);
}

// 1 / s for a positive finite fp16 scale s (so s is a normal fp32 value): the hardware
// approximation refined by one Newton-Raphson step (x1 = x0 + x0 (1 - s x0)). The result
// is within an ulp of 1 / s; a code depends on it only through y * (1 / s) at a rounding
// boundary, where the acceptance rule allows either neighbour.
__device__ __forceinline__ float recip_pos(float s) {
  float x0;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(x0) : "f"(s));
  return fmaf(x0, fmaf(-s, x0, 1.0f), x0);
}

constexpr float kMagic8 = 12583040.0f;    // 1.5 * 2^23 + 128: bits = 0x4B400080 + code
constexpr float kMagic8Lo = 12582913.0f;  // code -127
constexpr float kMagic8Hi = 12583167.0f;  // code +127

// One group of G values (already lambda-scaled): G * BITS / 32 code words (nibble
// pairs for BITS = 4, bytes for BITS = 8) and the fp16 scale bits.
template <int G, int BITS = 4>
__device__ __forceinline__ void quantize_group(const float (&y)[G], uint32_t (&words)[G * BITS / 32],
                                               uint32_t& sbits) {
  static_assert(BITS == 4 || BITS == 8, "code width");
  const float a = absmax<G>(y);
  if constexpr (BITS == 8) {
    const float sf = fminf(div_by_const<127>(a), 65504.0f);
    const __half hs = __float2half_rn(sf);
    const float sq = __half2float(hs);
    const float inv = sq > 0.0f ? recip_pos(sq) : 0.0f;
    sbits = __half_as_ushort(hs);
    uint32_t bits[G];
    if (a * inv < 127.5f) {
#pragma unroll
      for (int i = 0; i < G; ++i) bits[i] = __float_as_uint(fmaf(y[i], inv, kMagic8));
    } else {
#pragma unroll
      for (int i = 0; i < G; ++i)
        bits[i] = __float_as_uint(fminf(fmaxf(fmaf(y[i], inv, kMagic8), kMagic8Lo), kMagic8Hi));
    }
    // low byte of each word = code + 128 (1..255): four bytes per word, then the sign flip
#pragma unroll
    for (int w = 0; w < G / 4; ++w) {
      const uint32_t lo = prmt(bits[4 * w], bits[4 * w + 1], 0x3340u);
      const uint32_t hi = prmt(bits[4 * w + 2], bits[4 * w + 3], 0x3340u);
      words[w] = prmt(lo, hi, 0x5410u) ^ 0x80808080u;
    }
    return;
  }
  const float sf = fminf(div_by_const<7>(a), 65504.0f);
  const __half hs = __float2half_rn(sf);
  const float sq = __half2float(hs);
  const float inv = sq > 0.0f ? recip_pos(sq) : 0.0f;
  sbits = __half_as_ushort(hs);
  // |y| * inv can reach 7.5 only when the scale lost precision (fp16 subnormal or the
  // 65504 cap): then clamp to the +-7 codes before packing
  uint32_t bits[G];
  if (a * inv < 7.5f) {
#pragma unroll
    for (int i = 0; i < G; ++i) bits[i] = __float_as_uint(fmaf(y[i], inv, kMagic));
  } else {
#pragma unroll
    for (int i = 0; i < G; ++i) bits[i] = __float_as_uint(fminf(fmaxf(fmaf(y[i], inv, kMagic), kMagicLo), kMagicHi));
  }
  // low byte of each word = code + 8 (0..15): two nibbles per byte, four bytes per word
#pragma unroll
  for (int w = 0; w < G / 8; ++w) {
    const uint32_t* bb = bits + 8 * w;
    const uint32_t lo = bb[0] + (bb[1] << 4) + ((bb[2] + (bb[3] << 4)) << 8);
    const uint32_t hi = bb[4] + (bb[5] << 4) + ((bb[6] + (bb[7] << 4)) << 8);
    words[w] = prmt(lo, hi, 0x5410u) ^ 0x88888888u;
  }
}

}  // namespace kvq
