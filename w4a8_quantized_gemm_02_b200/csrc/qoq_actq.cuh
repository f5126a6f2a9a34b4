// Per-token INT8 activation quantization of FP16 values, shared by the
// stand-alone quantizer and the GEMM that quantizes its own activations:
// both must produce the same codes and scales bit for bit.
//
// Method: "QServe: W4A8KV4 Quantization and System Co-design for Efficient
// LLM Serving" -- the 8-bit activations of W4A8 (Insight), per token.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace qoq {

// fp16(amax / qmax) with the two guards of the format: 1.0 for an all-zero
// row, the smallest positive FP16 value when the quotient rounds to zero.
__device__ __forceinline__ __half scale_from_absmax(float amax, float qmax) {
  if (amax == 0.0f) return __ushort_as_half(0x3c00);
  __half s = __float2half_rn(__fdiv_rn(amax, qmax));
  if ((__half_as_ushort(s) & 0x7fff) == 0) s = __ushort_as_half(0x0001);
  return s;
}

// ---------------------------------------------------------------------------
// Per-token activation quantization.
//
// The code of a value is rne(x / sx) clamped to [-127, 127], computed without
// a division:
//  1. t = fma(x, rcp(sx), 1.5 * 2^23) rounds x * rcp to an integer q0 in one
//     step: t holds 1.5 * 2^23 + q0, so its low byte is q0 as a two's
//     complement INT8 and t - 1.5 * 2^23 is q0 exactly.
//  2. e = x - q0 * sx is exact (one fused multiply-add: q0 * sx and x are short
//     FP16-derived numbers).  q0 is within 0.5 + 2^-17 of x / sx, so it is the
//     nearest integer unless |e| >= sx / 2.  That is rare (a quotient within
//     2^-17 of a half-integer), and only then does a lane take the fix-up:
//     |e| > sx / 2 moves q0 one step towards e, |e| == sx / 2 is a tie that
//     goes to the even neighbour.
// The result is the round-half-even of the exact quotient x / sx.  For FP16 x
// and sx that equals rounding the binary32 quotient (the binary32 result can
// only sit on a half-integer if the exact quotient does), so the codes match
// an IEEE binary32 division bit for bit.
// When sx is a normal FP16 number, |x| / sx <= 127 / (1 - 2^-11) < 127.5 and
// no code can leave [-127, 127]; only rows whose scale is subnormal clamp.
// ---------------------------------------------------------------------------
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

template <bool kClamp>
__device__ __forceinline__ uint2 quantize8(uint4 v, float sf, float rcp, float half_sf) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  float x[8], t[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __half22float2(h[j]);
    x[2 * j] = f.x;
    x[2 * j + 1] = f.y;
  }
  bool near_half = false;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    t[j] = __fmaf_rn(x[j], rcp, kRoundMagic);
    const float e = __fmaf_rn(-(t[j] - kRoundMagic), sf, x[j]);
    near_half |= fabsf(e) >= half_sf;
  }
  if (near_half) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float e = __fmaf_rn(-(t[j] - kRoundMagic), sf, x[j]);
      const float ae = fabsf(e);
      const bool odd = __float_as_uint(t[j]) & 1u;   // the offset 1.5 * 2^23 is even
      if (ae > half_sf || (ae == half_sf && odd)) t[j] += e > 0.0f ? 1.0f : -1.0f;
    }
  }
  if (kClamp) {
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = fminf(fmaxf(t[j], kRoundMagic - 127.0f), kRoundMagic + 127.0f);
  }
  uint32_t b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) b[j] = __float_as_uint(t[j]);
  const uint32_t w0 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040),
                                  0x5410);
  const uint32_t w1 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040),
                                  0x5410);
  return make_uint2(w0, w1);
}

__device__ __forceinline__ __half2 absmax8(uint4 v, __half2 amax) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int j = 0; j < 4; ++j) amax = __hmax2(amax, __habs2(h[j]));
  return amax;
}

}  // namespace qoq
