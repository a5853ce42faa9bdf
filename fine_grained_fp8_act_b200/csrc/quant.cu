// quant.cu -- activation and weight quantization kernels (sm_100a).
//
// Per-token activation groups of 1x128 and 128x128 weight blocks, as the
// Transformers fine-grained FP8 page describes ("Transformers 中的细粒度 FP8
// 量化 ... 完全指南", §一): one scale per group, scale = max(amax/448, 2^-126)
// (float32, correctly rounded), UE8M0 = that scale rounded up to a power of
// two (§七 补充), element = e4m3(x / scale) with a correctly rounded float32
// quotient and a round-to-nearest-even, saturating cast.
//
// Both kernels are HBM streams: 16-byte loads, amax by warp shuffles, packed
// e4m3 stores; no shared-memory staging is needed because every group is read
// once, reduced in registers and written once.

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fg8_internal.h"

namespace fg8 {
namespace {

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

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// Quantize 8 values with the group's scale; returns 8 packed e4m3 bytes.
template <int FMT>
__device__ __forceinline__ uint2 quantize8(const float (&f)[8], float s, uint32_t sbyte) {
  float q[8];
  if (FMT == 0) {
    const float y = __frcp_rn(s);
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = div_rn_from_rcp(f[i], s, y);
  } else {
    const float inv = e8m0_reciprocal(sbyte);  // x * 2^-e is the correctly rounded x / 2^e
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(f[i], inv);
  }
  return make_uint2(pack_e4m3x4(q[0], q[1], q[2], q[3]), pack_e4m3x4(q[4], q[5], q[6], q[7]));
}

// ------------------------------------------------------------ act quant ----
// A half-warp owns one 128-channel group: lane l loads channels [8l, 8l+8)
// with one 16-byte load.  Each warp takes 8 groups per iteration (4 per half,
// loads issued before any arithmetic) and strides over the grid.
//   kScaleRowMajor: group g -> (m = g / Kb, kb = g % Kb)  (scales [M, Kb])
//   kScaleKMajor / kScaleSfTiles: g -> (kb = g / rows, m = g % rows), so the
//   scale writes of neighbouring half-warps are neighbouring addresses.
template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(256) act_quant_kernel(const ActQuantArgs a, const int64_t total, const int rows,
                                                        const int cols) {
  const int lane = threadIdx.x & 31, half = lane >> 4, l = lane & 15;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const uint16_t* x = static_cast<const uint16_t*>(a.x);

  for (int64_t base = warp * 8; base < total; base += nwarps * 8) {
    uint4 v[4];
    int m[4], kb[4];
    bool has[4], real[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t g = base + u * 2 + half;
      has[u] = g < total;
      if (LAYOUT == kScaleRowMajor) {
        m[u] = static_cast<int>(g / cols);
        kb[u] = static_cast<int>(g % cols);
      } else {
        kb[u] = static_cast<int>(g / rows);
        m[u] = static_cast<int>(g % rows);
      }
      real[u] = has[u] && m[u] < a.M && kb[u] < a.Kb;
      const int k = kb[u] * kGroup + l * 8;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (real[u] && k < a.K) v[u] = __ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m[u]) * a.ld_x + k));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f[8];
      unpack_bf16x8(v[u], f);
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
      const float s = group_scale(amax);
      const uint32_t sbyte = FMT == 1 ? e8m0_ceil_byte(s) : 0u;
      const uint2 packed = quantize8<FMT>(f, s, sbyte);
      const int k = kb[u] * kGroup + l * 8;
      if (real[u] && k < a.K) *reinterpret_cast<uint2*>(a.xq + static_cast<int64_t>(m[u]) * a.K + k) = packed;
      if (l == 0 && has[u]) {
        if (LAYOUT == kScaleRowMajor) {
          if (FMT == 0) static_cast<float*>(a.xs)[static_cast<int64_t>(m[u]) * a.Kb + kb[u]] = s;
          else static_cast<uint8_t*>(a.xs)[static_cast<int64_t>(m[u]) * a.Kb + kb[u]] = static_cast<uint8_t>(sbyte);
        } else if (LAYOUT == kScaleKMajor) {
          if (real[u]) static_cast<float*>(a.xs)[static_cast<int64_t>(kb[u]) * a.ld_s + m[u]] = s;
        } else {
          static_cast<uint8_t*>(a.xs)[sf_tile_offset(m[u], kb[u], a.Kq)] =
              real[u] ? static_cast<uint8_t>(sbyte) : static_cast<uint8_t>(127);
        }
      }
    }
  }
}

// ---------------------------------------------------------- weight quant ----
// One CTA per 128x128 block.  Thread t loads 8 rows (t/16 + 16i) x 8 channels
// (8*(t%16)), all held in registers across the block-wide amax reduction.
template <int FMT>
__global__ void __launch_bounds__(256) weight_quant_kernel(const uint16_t* __restrict__ w, const int64_t ld_w,
                                                           const int N, const int K, const int Kb,
                                                           uint8_t* __restrict__ wq, void* __restrict__ ws) {
  __shared__ float red[8];
  const int nb = blockIdx.y, kb = blockIdx.x;
  const int t = threadIdx.x, rg = t >> 4, c = t & 15;
  const int k = kb * 128 + c * 8;
  uint4 v[8];
  bool ok[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = nb * 128 + rg + 16 * i;
    ok[i] = n < N && k < K;
    v[i] = ok[i] ? __ldg(reinterpret_cast<const uint4*>(w + static_cast<int64_t>(n) * ld_w + k))
                 : make_uint4(0u, 0u, 0u, 0u);
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float f[8];
    unpack_bf16x8(v[i], f);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  if ((t & 31) == 0) red[t >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float s = group_scale(amax);
  const uint32_t sbyte = FMT == 1 ? e8m0_ceil_byte(s) : 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (!ok[i]) continue;
    float f[8];
    unpack_bf16x8(v[i], f);
    const int n = nb * 128 + rg + 16 * i;
    *reinterpret_cast<uint2*>(wq + static_cast<int64_t>(n) * K + k) = quantize8<FMT>(f, s, sbyte);
  }
  if (t == 0) {
    if (FMT == 0) static_cast<float*>(ws)[static_cast<int64_t>(nb) * Kb + kb] = s;
    else static_cast<uint8_t*>(ws)[static_cast<int64_t>(nb) * Kb + kb] = static_cast<uint8_t>(sbyte);
  }
}

// --------------------------------------------------------------- sf pack ----
__global__ void __launch_bounds__(256) sf_pack_kernel(const uint8_t* __restrict__ src, const int R, const int row_div,
                                                      const int Kb, const int Kq, const int64_t total,
                                                      uint8_t* __restrict__ dst) {
  const int cols = Kq * 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / cols;
    const int kb = static_cast<int>(i % cols);
    const uint8_t b = (r < R && kb < Kb) ? src[(r / row_div) * Kb + kb] : static_cast<uint8_t>(127);
    dst[sf_tile_offset(r, kb, Kq)] = b;
  }
}

}  // namespace

cudaError_t launch_act_quant(const ActQuantArgs& a, int fmt, int num_sms, cudaStream_t s) {
  int rows, cols;
  if (a.layout == kScaleSfTiles) {
    rows = a.M_pad;
    cols = a.Kq * 4;
  } else {
    rows = a.M;
    cols = a.Kb;
  }
  const int64_t total = static_cast<int64_t>(rows) * cols;
  if (total == 0) return cudaSuccess;
  const int64_t per_block = 8 * 8;  // 8 warps x 8 groups per pass
  int64_t blocks = (total + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  const dim3 grid(static_cast<unsigned>(blocks)), block(256);
#define FG8_AQ(F, L) act_quant_kernel<F, L><<<grid, block, 0, s>>>(a, total, rows, cols)
  if (fmt == 0) {
    if (a.layout == kScaleRowMajor) FG8_AQ(0, kScaleRowMajor);
    else FG8_AQ(0, kScaleKMajor);
  } else {
    if (a.layout == kScaleRowMajor) FG8_AQ(1, kScaleRowMajor);
    else FG8_AQ(1, kScaleSfTiles);
  }
#undef FG8_AQ
  return cudaGetLastError();
}

cudaError_t launch_weight_quant(const void* w, int64_t ld_w, int N, int K, uint8_t* wq, void* ws, int fmt,
                                cudaStream_t s) {
  const int Kb = (K + 127) / 128, Nb = (N + 127) / 128;
  const dim3 grid(Kb, Nb), block(256);
  if (fmt == 0) weight_quant_kernel<0><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(w), ld_w, N, K, Kb, wq, ws);
  else weight_quant_kernel<1><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(w), ld_w, N, K, Kb, wq, ws);
  return cudaGetLastError();
}

cudaError_t launch_sf_pack(const uint8_t* src, int R, int row_div, int Kb, uint8_t* dst, cudaStream_t s) {
  const int Kq = (Kb + 3) / 4;
  const int64_t R_pad = (static_cast<int64_t>(R) + 127) / 128 * 128;
  const int64_t total = R_pad * Kq * 4;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  sf_pack_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(src, R, row_div, Kb, Kq, total, dst);
  return cudaGetLastError();
}

}  // namespace fg8
