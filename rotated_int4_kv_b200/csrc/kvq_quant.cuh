// kvq_quant.cuh -- per-group quantisation of rotated, lambda-scaled channels to
// signed int4 ("When Quantization Is Free", gist.science/de/paper/2605.05699,
// "Methodik" 2: per-group abs-max scale, symmetric int4 codes, nibble packing).
//
// scale = fp16_rn(min(absmax / 7, 65504)); code = clamp(rint(y / scale), -7, 7)
// (0 where the scale is 0), two's-complement nibbles, even channel in the low
// nibble. The rounding is the fp32 "magic number" FMA: y * (1/scale) + (1.5 * 2^23
// + 8) leaves code + 8 in the low four mantissa bits (round to nearest even), so
// packing is integer shifts and a byte permute.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_ptx.cuh"

namespace kvq {

constexpr float kMagic = 12582920.0f;    // 1.5 * 2^23 + 8: bits = 0x4B400008 + code
constexpr float kMagicLo = 12582913.0f;  // code -7
constexpr float kMagicHi = 12582927.0f;  // code +7

// One group of G values (already lambda-scaled): G/8 packed code words and the
// fp16 scale bits.
template <int G>
__device__ __forceinline__ void quantize_group(const float (&y)[G], uint32_t (&words)[G / 8], uint32_t& sbits) {
  // abs-max as a pairwise tree (max is exact, so the order does not matter)
  float m[G / 2];
#pragma unroll
  for (int i = 0; i < G / 2; ++i) m[i] = fmaxf(fabsf(y[2 * i]), fabsf(y[2 * i + 1]));
#pragma unroll
  for (int w = G / 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  const float a = m[0];
  const float sf = fminf(__fdiv_rn(a, 7.0f), 65504.0f);
  const __half hs = __float2half_rn(sf);
  const float sq = __half2float(hs);
  const float inv = sq > 0.0f ? __frcp_rn(sq) : 0.0f;
  sbits = __half_as_ushort(hs);
  const bool clampit = a * inv >= 7.5f;
  uint32_t b[G];
#pragma unroll
  for (int i = 0; i < G; i += 2) {
    float2 q = __ffma2_rn(make_float2(y[i], y[i + 1]), make_float2(inv, inv), make_float2(kMagic, kMagic));
    if (clampit) {
      q.x = fminf(fmaxf(q.x, kMagicLo), kMagicHi);
      q.y = fminf(fmaxf(q.y, kMagicLo), kMagicHi);
    }
    b[i] = __float_as_uint(q.x);
    b[i + 1] = __float_as_uint(q.y);
  }
#pragma unroll
  for (int w = 0; w < G / 8; ++w) {
    const uint32_t* bb = b + 8 * w;
    const uint32_t x01 = bb[0] + (bb[1] << 4);
    const uint32_t x23 = bb[2] + (bb[3] << 4);
    const uint32_t x45 = bb[4] + (bb[5] << 4);
    const uint32_t x67 = bb[6] + (bb[7] << 4);
    words[w] = prmt(x01 + (x23 << 8), x45 + (x67 << 8), 0x5410u) ^ 0x88888888u;
  }
}

}  // namespace kvq
