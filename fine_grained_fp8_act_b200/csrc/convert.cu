// convert.cu -- checkpoint conversions ("Transformers 中的细粒度 FP8 量化 ...
// 完全指南", §五 and §七): Fp8Dequantize, which folds each 128x128 block's
// scale back into bf16 weights, and the exact conversion of power-of-two
// scales kept in float32 containers (the ".scale" key) to UE8M0 bytes.
//
// Both are streams over the tensor: 16 weights per thread (one 16-byte load,
// two 16-byte stores), one scale word per thread.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "fg8_internal.h"

namespace fg8 {
namespace {

// UE8M0 byte b -> 2^(b - 127) as a float (b = 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_to_float(uint32_t b) {
  return b == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(b << 23);
}

// w = bf16(value(q) * s): value(q) has at most 4 significant bits and s 24,
// so the double product is exact and __double2bfloat16 rounds it once (RNE).
template <int FMT>
__global__ void __launch_bounds__(256) dequant_weight_kernel(const uint8_t* __restrict__ wq, const int64_t K,
                                                             const void* __restrict__ ws, const int Kb,
                                                             uint16_t* __restrict__ w, const int64_t ld_w,
                                                             const int64_t groups16) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < groups16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e0 = i * 16;
    const int64_t n = e0 / K, k0 = e0 - n * K;  // 16 weights of row n (K % 16 == 0), inside one 128-block
    const int64_t blk = (n >> 7) * Kb + (k0 >> 7);
    const float s = FMT == 0 ? static_cast<const float*>(ws)[blk] : e8m0_to_float(static_cast<const uint8_t*>(ws)[blk]);
    const uint4 q = *reinterpret_cast<const uint4*>(wq + e0);
    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
    uint32_t out[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __half2_raw v2 = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>((qw[j] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
        const float lo = __half2float(__half(__half_raw{v2.x}));
        const float hi = __half2float(__half(__half_raw{v2.y}));
        const uint16_t blo = __bfloat16_as_ushort(__double2bfloat16(static_cast<double>(lo) * static_cast<double>(s)));
        const uint16_t bhi = __bfloat16_as_ushort(__double2bfloat16(static_cast<double>(hi) * static_cast<double>(s)));
        out[2 * j + h] = static_cast<uint32_t>(blo) | (static_cast<uint32_t>(bhi) << 16);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(w + n * ld_w + k0);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
}

// s = 2^e (-127 <= e <= 127) -> e + 127; anything else -> 255, counted.
__global__ void __launch_bounds__(256) scale_to_e8m0_kernel(const float* __restrict__ s, const int64_t n,
                                                            uint8_t* __restrict__ out, uint32_t* __restrict__ bad) {
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x; base < n;
       base += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = base + threadIdx.x;
    uint32_t b = 255u;
    if (i < n) {
      const uint32_t bits = __float_as_uint(s[i]);
      const uint32_t e = (bits >> 23) & 0xFFu;
      if (bits == 0x00400000u) b = 0u;                                       // 2^-127, a float32 subnormal
      else if ((bits >> 31) == 0u && (bits & 0x7FFFFFu) == 0u && e >= 1u && e <= 254u) b = e;  // 2^(e-127)
      out[i] = static_cast<uint8_t>(b);
    }
    const unsigned invalid = __ballot_sync(0xFFFFFFFFu, i < n && b == 255u);
    if (bad != nullptr && (threadIdx.x & 31) == 0 && invalid != 0u) atomicAdd(bad, static_cast<uint32_t>(__popc(invalid)));
  }
}

// Batched expert layout -> the grouped layout's expert index: expert e owns
// rows [e * cap, (e + 1) * cap), of which the first counts[e] are routed.
__global__ void __launch_bounds__(256) row_expert_kernel(const int32_t* __restrict__ counts, const int E, const int cap,
                                                         int32_t* __restrict__ row_expert) {
  const int64_t total = static_cast<int64_t>(E) * cap;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(i / cap), r = static_cast<int>(i % cap);
    row_expert[i] = r < counts[e] ? e : -1;
  }
}

}  // namespace

cudaError_t launch_dequant_weight(const uint8_t* wq, int N, int K, const void* ws, int fmt, uint16_t* w, int64_t ld_w,
                                  int num_sms, cudaStream_t s) {
  const int64_t groups16 = static_cast<int64_t>(N) * K / 16;
  if (groups16 == 0) return cudaSuccess;
  int64_t blocks = (groups16 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  const int Kb = (K + 127) / 128;
  if (fmt == 0)
    dequant_weight_kernel<0><<<static_cast<unsigned>(blocks), 256, 0, s>>>(wq, K, ws, Kb, w, ld_w, groups16);
  else
    dequant_weight_kernel<1><<<static_cast<unsigned>(blocks), 256, 0, s>>>(wq, K, ws, Kb, w, ld_w, groups16);
  return cudaGetLastError();
}

cudaError_t launch_row_expert(const int32_t* counts, int E, int cap, int32_t* row_expert, int num_sms,
                              cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(E) * cap;
  if (total == 0) return cudaSuccess;
  int64_t blocks = (total + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
  row_expert_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(counts, E, cap, row_expert);
  return cudaGetLastError();
}

cudaError_t launch_scale_to_e8m0(const float* s, int64_t n, uint8_t* out, uint32_t* bad, int num_sms, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  scale_to_e8m0_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(s, n, out, bad);
  return cudaGetLastError();
}

}  // namespace fg8
