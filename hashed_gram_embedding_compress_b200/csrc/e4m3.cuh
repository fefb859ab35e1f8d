// E4M3 quantisation of bf16 rows for the FP8 projections.
//
// "Conditional Memory via Scalable Lookup", section 2.4: the value projection
// and the M key projections run as one dense FP8 matmul.  The pages fix
// neither the format nor the scaling; this library uses E4M3 (1 sign bit, 4
// exponent bits with bias 7, 3 mantissa bits, largest finite magnitude 448)
// with one power-of-two scale per row: 2^E, E the smallest integer with
// amax <= 448 * 2^E (E = 0 for an all-zero row), code = E4M3(x * 2^-E) rounded
// to nearest with ties to even.  x * 2^-E is exact in fp32, so the rounding
// decision is taken on the exact value; the scale is applied to the fp32
// products of the matmul.
#pragma once

#include <stdint.h>

namespace engram {

constexpr int kQuantMaxChunks = 8;  // 16-byte chunks per lane: rows of <= 2048 bf16

// 2^n as a normal fp32, -126 <= n <= 127.
__device__ __forceinline__ float e4m3_pow2(int n) { return __int_as_float((n + 127) << 23); }

// 2^E for -149 <= E <= 127 (subnormal below -126).
__device__ __forceinline__ float e4m3_scale_value(int E) {
  return E >= -126 ? e4m3_pow2(E) : __uint_as_float(1u << (E + 149));
}

// Smallest E with amax <= 448 * 2^E; amax = f 2^x with 0.5 <= f < 1 and
// 448 = 0.875 2^9, so E = x - 9 when f <= 0.875, else x - 8.
__device__ __forceinline__ int e4m3_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int x;
  const float f = frexpf(amax, &x);
  return f <= 0.875f ? x - 9 : x - 8;
}

// Two values to two E4M3 codes (lo in the low byte), nearest-even, saturating.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Quantise one row of C 16-byte chunks of bf16 (8 values each, C <= 256) with
// one warp: src(c) returns chunk c; codes go to dst (8 bytes per chunk), the
// scale 2^E to *scale (written by lane 0).
template <class Src>
__device__ __forceinline__ void quant_row_warp(Src src, int C, uint8_t* dst, float* scale,
                                               int lane) {
  uint4 v[kQuantMaxChunks];
  uint32_t amax = 0;  // |x| as the upper half of its fp32 bits: integer order = value order
#pragma unroll
  for (int i = 0; i < kQuantMaxChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < C) v[i] = src(c);
  }
#pragma unroll
  for (int i = 0; i < kQuantMaxChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < C) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) amax = max(amax, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
  }
  amax = __reduce_max_sync(0xffffffffu, amax);
  const int E = e4m3_scale_exp(__uint_as_float(amax << 16));
  // 2^-E in two exact factors (E ranges over [-142, 120] for finite bf16)
  const float s1 = e4m3_pow2((-E) / 2), s2 = e4m3_pow2(-E - (-E) / 2);
#pragma unroll
  for (int i = 0; i < kQuantMaxChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < C) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t q[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = __uint_as_float(w[j] << 16) * s1 * s2;
        const float hi = __uint_as_float(w[j] & 0xFFFF0000u) * s1 * s2;
        q[j] = e4m3x2(lo, hi);
      }
      *reinterpret_cast<uint2*>(dst + (int64_t)c * 8) =
          make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
    }
  }
  if (lane == 0) *scale = e4m3_scale_value(E);
}

}  // namespace engram
