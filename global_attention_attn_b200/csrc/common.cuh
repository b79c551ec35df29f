// Device helpers shared by the kernels: bf16 conversion and the RoPE angle.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "internal.h"

namespace mimo {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  return uint32_t(f32_to_bf16(lo)) | (uint32_t(f32_to_bf16(hi)) << 16);
}
__device__ __forceinline__ uint32_t pack2_f16(float lo, float hi) {
  return uint32_t(__half_as_ushort(__float2half_rn(lo))) | (uint32_t(__half_as_ushort(__float2half_rn(hi))) << 16);
}

// Largest finite fp16 value.  The rotated query / key dims are kept in fp16; a component
// beyond it is stored as +-65504 and reported with MIMO_STATUS_RANGE.
constexpr float kF16Max = 65504.f;

// Two floats -> fp16x2 rounded to nearest even, saturating at +-65504 (NaN stays NaN);
// `amax` collects the largest magnitude seen so that the caller can report saturation.
__device__ __forceinline__ uint32_t pack2_f16_sat(float lo, float hi, float& amax) {
  uint32_t d;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
  return d;
}

// cos / sin of pos * inv_freq.  The angle and its reduction to [-pi, pi] are
// taken in float64 (the fastest rotary angle equals the position, up to ~1.3e5
// radians here, far past where a float32 angle keeps its digits); only the
// reduced angle goes through the float32 sincos.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float* c, float* s) {
  const double two_pi = 6.283185307179586476925286766559;
  const double theta = double(pos) * inv_freq;
  const double k = rint(theta * (1.0 / two_pi));
  const float r = float(fma(-k, two_pi, theta));
  sincosf(r, s, c);
}

// OCP E4M3 (FP8) conversions.  Two floats -> two E4M3 bytes (round to nearest even,
// saturating to +-448): `lo` lands in the low byte.
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}
// Two E4M3 bytes -> two fp16 (exact: E4M3 is a subset of fp16); the low byte lands in
// the low half.
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint16_t x) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(x));
  return d;
}

// NeoX rotate-half on one 16-byte chunk pair: lo holds dims 8u..8u+7, hi holds
// dims 8u+32..8u+39 (u in 0..3); frequency index of element i is 8u+i.
// Input bf16, output IEEE fp16: the rotated dims are kept in fp16 everywhere
// (query tiles, key copies, caches) because their rounding error enters every
// logit; fp16 has 11 significant bits against bf16's 8.  Outputs saturate at
// +-65504 and `amax` collects the largest magnitude (see pack2_f16_sat).
__device__ __forceinline__ void rope_chunk_pair(uint4& lo, uint4& hi, int u, int pos, const RopeFreqs& rf,
                                                float& amax) {
  uint32_t* a = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* b = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float x0 = lo_bf16(a[w]), x1 = hi_bf16(a[w]);
    float y0 = lo_bf16(b[w]), y1 = hi_bf16(b[w]);
    float c0, s0, c1, s1;
    rope_cos_sin(pos, rf.inv_freq[8 * u + 2 * w], &c0, &s0);
    rope_cos_sin(pos, rf.inv_freq[8 * u + 2 * w + 1], &c1, &s1);
    a[w] = pack2_f16_sat(x0 * c0 - y0 * s0, x1 * c1 - y1 * s1, amax);
    b[w] = pack2_f16_sat(y0 * c0 + x0 * s0, y1 * c1 + x1 * s1, amax);
  }
}

// Same rotation with precomputed (cos, sin) pairs: cs[i] for frequency 8u+i.
__device__ __forceinline__ void rope_chunk_pair_cs(uint4& lo, uint4& hi, const float2* cs, float& amax) {
  uint32_t* a = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* b = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float x0 = lo_bf16(a[w]), x1 = hi_bf16(a[w]);
    const float y0 = lo_bf16(b[w]), y1 = hi_bf16(b[w]);
    const float2 t0 = cs[2 * w], t1 = cs[2 * w + 1];
    a[w] = pack2_f16_sat(x0 * t0.x - y0 * t0.y, x1 * t1.x - y1 * t1.y, amax);
    b[w] = pack2_f16_sat(y0 * t0.x + x0 * t0.y, y1 * t1.x + x1 * t1.y, amax);
  }
}

// Same rotation on packed fp32 pairs: cs[w] = (cos_a, sin_a, cos_b, sin_b) for the
// two frequencies held by 32-bit word w of the chunks.
__device__ __forceinline__ void rope_chunk_pair_cs4(uint4& lo, uint4& hi, const float4* cs, float& amax) {
  uint32_t* a = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* b = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float4 t = cs[w];
    // x = (x0, x1), y = (y0, y1), c = (c0, c1), s = (s0, s1)
    uint64_t x, y, c, sn, ns, r0, r1;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(a[w] << 16), "r"(a[w] & 0xFFFF0000u));
    asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "r"(b[w] << 16), "r"(b[w] & 0xFFFF0000u));
    asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(t.x), "f"(t.z));
    asm("mov.b64 %0, {%1, %2};" : "=l"(sn) : "f"(t.y), "f"(t.w));
    asm("mov.b64 %0, {%1, %2};" : "=l"(ns) : "f"(-t.y), "f"(-t.w));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r0) : "l"(y), "l"(ns));      // -y s
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(r0) : "l"(x), "l"(c));   // x c - y s
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r1) : "l"(x), "l"(sn));      // x s
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(r1) : "l"(y), "l"(c));   // y c + x s
    float a0, a1, b0, b1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(r0));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(r1));
    a[w] = pack2_f16_sat(a0, a1, amax);
    b[w] = pack2_f16_sat(b0, b1, amax);
  }
}


}  // namespace mimo
