// quant_math.cuh -- the per-element arithmetic of the fine-grained FP8
// quantization, shared by the stand-alone quantization kernels and the GEMM
// epilogue that quantizes a layer's output for the next layer (both must give
// the same bits).
//
// scale = max(amax / 448, 2^-126) in correctly rounded float32; UE8M0 keeps
// the smallest power of two >= scale ("Transformers 中的细粒度 FP8 量化 ...",
// §七 补充: float scales round *up* to UE8M0); element = e4m3(RN_f32(x /
// scale')) with a round-to-nearest-even, saturating cast.
#pragma once

#include <cuda_fp8.h>

#include <cstdint>

namespace fg8 {
namespace qm {

constexpr float kMinScale = 1.17549435082228750797e-38f;  // 2^-126

__device__ __forceinline__ float group_scale(float amax) {
  return fmaxf(__fdiv_rn(amax, 448.0f), kMinScale);
}

// Smallest power of two >= s (s a positive normal float) as a UE8M0 byte.
__device__ __forceinline__ uint32_t e8m0_ceil_byte(float s) {
  const uint32_t b = __float_as_uint(s);
  return (b >> 23) + ((b & 0x7FFFFFu) != 0u);
}

// 2^(127 - byte): the exact reciprocal of the UE8M0 scale (byte <= 253).
__device__ __forceinline__ float e8m0_reciprocal(uint32_t byte) { return __uint_as_float((254u - byte) << 23); }

// Correctly rounded float32 a / b from y = RN(1/b): one refinement brings
// q within one ulp of a/b, and a second FMA-based correction step is then
// exact by Markstein's theorem (remainder r = a - q*b computed exactly by the
// FMA; q' = RN(q + r*y)).  The sign of a zero quotient is taken from a.
__device__ __forceinline__ float div_rn_from_rcp(float a, float b, float y) {
  float q = __fmul_rn(a, y);
  float r = __fmaf_rn(-q, b, a);
  q = __fmaf_rn(r, y, q);
  r = __fmaf_rn(-q, b, a);
  q = __fmaf_rn(r, y, q);
  return copysignf(q, a);
}

// The same correctly rounded quotient for two values at once with packed
// f32x2 arithmetic (each lane of FMUL2/FFMA2 rounds exactly like the scalar op).
__device__ __forceinline__ float2 div2_rn_from_rcp(float2 a, float b, float y) {
  const float2 Y = make_float2(y, y), nB = make_float2(-b, -b);
  float2 q = __fmul2_rn(a, Y);
  float2 r = __ffma2_rn(q, nB, a);
  q = __ffma2_rn(r, Y, q);
  r = __ffma2_rn(q, nB, a);
  q = __ffma2_rn(r, Y, q);
  return make_float2(copysignf(q.x, a.x), copysignf(q.y, a.y));
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Quantize 16 values (two 16-byte bf16 loads) with the group's scale;
// returns 16 packed e4m3 bytes.
template <int FMT>
__device__ __forceinline__ uint4 quantize16(const float (&f)[16], float s, uint32_t sbyte) {
  float q[16];
  if (FMT == 0) {
    const float y = __frcp_rn(s);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 r = div2_rn_from_rcp(make_float2(f[i], f[i + 1]), s, y);
      q[i] = r.x;
      q[i + 1] = r.y;
    }
  } else {
    const float inv = e8m0_reciprocal(sbyte);  // x * 2^-e is the correctly rounded x / 2^e
    const float2 I = make_float2(inv, inv);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 r = __fmul2_rn(make_float2(f[i], f[i + 1]), I);
      q[i] = r.x;
      q[i + 1] = r.y;
    }
  }
  return make_uint4(pack_e4m3x4(q[0], q[1], q[2], q[3]), pack_e4m3x4(q[4], q[5], q[6], q[7]),
                    pack_e4m3x4(q[8], q[9], q[10], q[11]), pack_e4m3x4(q[12], q[13], q[14], q[15]));
}

}  // namespace qm
}  // namespace fg8
