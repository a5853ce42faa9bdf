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
#include "ptx.cuh"
#include "quant_math.cuh"

namespace fg8 {
namespace {

using namespace qm;

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

// n / d and n % d for a divisor fixed per launch, by multiply-high (Granlund
// and Montgomery, "Division by invariant integers using multiplication",
// 1994): with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1,
// q = (t + ((n - t) >> 1)) >> (l - 1), t = umulhi(m, n), for all 32-bit n.
struct FastDiv {
  uint32_t d, m, l;
};

__host__ inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{d, 0u, 0u};
  while ((1ull << f.l) < d) ++f.l;
  if (d > 1) f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << f.l) - d)) / d + 1);
  return f;
}

__device__ __forceinline__ void fast_divmod(const FastDiv& f, uint32_t n, uint32_t& q, uint32_t& r) {
  if (f.d == 1) {
    q = n;
  } else {
    const uint32_t t = __umulhi(f.m, n);
    q = (t + ((n - t) >> 1)) >> (f.l - 1);
  }
  r = n - q * f.d;
}

// ------------------------------------------------------------ act quant ----
// Static activation scheme (float scales): the same arithmetic with the
// group scale replaced by one scale for the tensor (values beyond 448 times it
// saturate); the scale is still written per group, so the GEMM reads it
// exactly as it reads dynamic scales.
//
// GL lanes own one group of 16*GL channels (8 lanes for the default 128, 2
// for 1 x 32 groups): lane l loads channels [16l, 16l+16) with two 16-byte
// loads.  A warp covers 32/GL groups per pass and makes 2 passes per
// iteration (all loads issued before any arithmetic), striding over the
// grid.  amax: per-lane max, then log2(GL) xor-shuffles inside the group.
//   kScaleRowMajor: group g -> (m = g / Kb, kb = g % Kb)  (scales [M, Kb])
//   kScaleKMajor / kScaleSfTiles: g -> (kb = g / rows, m = g % rows), so the
//   scale writes of neighbouring lane-octets are neighbouring addresses.
template <int FMT, int LAYOUT, int GL>
__global__ void __launch_bounds__(256) act_quant_kernel(const ActQuantArgs a, const uint32_t total, const FastDiv div) {
  grid_wait_prerequisites();  // x may come from the preceding kernel (launched ahead of its end)
  grid_launch_dependents();   // the GEMM may set itself up meanwhile; it waits for our results
  constexpr int kPasses = 2;
  constexpr int kGpw = 32 / GL;  // groups per warp and pass
  constexpr int G = 16 * GL;     // group width
  const int lane = threadIdx.x & 31, oct = lane / GL, l = lane % GL;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint16_t* x = static_cast<const uint16_t*>(a.x);

  for (uint32_t base = warp * (kGpw * kPasses); base < total; base += nwarps * (kGpw * kPasses)) {
    uint4 v[kPasses][2];
    int m[kPasses], kb[kPasses];
    bool has[kPasses], real[kPasses];
#pragma unroll
    for (int u = 0; u < kPasses; ++u) {
      const uint32_t g = base + u * kGpw + oct;
      has[u] = g < total;
      uint32_t qt, r;
      fast_divmod(div, g, qt, r);
      if (LAYOUT == kScaleRowMajor) {
        m[u] = static_cast<int>(qt);   // div = Kb
        kb[u] = static_cast<int>(r);
      } else {
        kb[u] = static_cast<int>(qt);  // div = rows
        m[u] = static_cast<int>(r);
      }
      real[u] = has[u] && m[u] < a.M && kb[u] < a.Kb;
      const int k = kb[u] * G + l * 16;
      v[u][0] = v[u][1] = make_uint4(0u, 0u, 0u, 0u);
      if (real[u] && k < a.K) {
        const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m[u]) * a.ld_x + k);
        v[u][0] = __ldg(src);
        v[u][1] = __ldg(src + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < kPasses; ++u) {
      float f[16];
      float(&f0)[8] = *reinterpret_cast<float(*)[8]>(f);
      float(&f1)[8] = *reinterpret_cast<float(*)[8]>(f + 8);
      unpack_bf16x8(v[u][0], f0);
      unpack_bf16x8(v[u][1], f1);
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int off = GL / 2; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
      // dynamic: the group's scale; static (float only): the tensor's one scale
      const float s = (FMT == 0 && a.static_scale != nullptr) ? *a.static_scale : group_scale(amax);
      const uint32_t sbyte = FMT == 1 ? e8m0_ceil_byte(s) : 0u;
      const uint4 packed = quantize16<FMT>(f, s, sbyte);
      const int k = kb[u] * G + l * 16;
      if (real[u] && k < a.K) *reinterpret_cast<uint4*>(a.xq + static_cast<int64_t>(m[u]) * a.K + k) = packed;
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

// One warp per 32 x 32 block (weight_block_size = (32, 32)): lane i holds row
// i of the block (32 channels, four 16-byte loads; a 16-wide last block when
// K % 32 == 16), amax by 5 xor-shuffles, two 16-byte stores per row.
template <int FMT>
__global__ void __launch_bounds__(256) weight_quant32_kernel(const uint16_t* __restrict__ w, const int64_t ld_w,
                                                             const int N, const int K, const int Nb, const int Kb,
                                                             uint8_t* __restrict__ wq, void* __restrict__ ws) {
  const int lane = threadIdx.x & 31;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (blk >= static_cast<int64_t>(Nb) * Kb) return;
  const int nb = static_cast<int>(blk / Kb), kb = static_cast<int>(blk % Kb);
  const int n = nb * 32 + lane, k0 = kb * 32;
  const bool row = n < N;
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = k0 + 8 * i;
    v[i] = (row && k < K) ? __ldg(reinterpret_cast<const uint4*>(w + static_cast<int64_t>(n) * ld_w + k))
                          : make_uint4(0u, 0u, 0u, 0u);
  }
  float f[2][16];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float(&a0)[8] = *reinterpret_cast<float(*)[8]>(f[h]);
    float(&a1)[8] = *reinterpret_cast<float(*)[8]>(f[h] + 8);
    unpack_bf16x8(v[2 * h], a0);
    unpack_bf16x8(v[2 * h + 1], a1);
  }
  float amax = 0.0f;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[h][i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  const float s = group_scale(amax);
  const uint32_t sbyte = FMT == 1 ? e8m0_ceil_byte(s) : 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = k0 + 16 * h;
    if (row && k < K)
      *reinterpret_cast<uint4*>(wq + static_cast<int64_t>(n) * K + k) = quantize16<FMT>(f[h], s, sbyte);
  }
  if (lane == 0) {
    if (FMT == 0) static_cast<float*>(ws)[blk] = s;
    else static_cast<uint8_t*>(ws)[blk] = static_cast<uint8_t>(sbyte);
  }
}

// --------------------------------------------------------------- sf pack ----
// One thread per 16-byte chunk of a scale-factor tile: chunk i of tile
// (rows 128 t.., K-blocks 4 q..) holds the words of rows 128 t + 32 c + i,
// c = 0..3, byte j of each being K-block 4 q + j (sf_tile_offset's layout).
// Rows past R and K-blocks past Kb get 127 (2^0, never applied to data).
__global__ void __launch_bounds__(256) sf_pack_kernel(const uint8_t* __restrict__ src, const int R, const int row_div,
                                                      const int Kb, const int Kq, const int64_t chunks,
                                                      uint8_t* __restrict__ dst) {
  grid_wait_prerequisites();
  grid_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < chunks;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tq = i >> 5;  // (tile, K-group) index: tile * Kq + q
    const int lane = static_cast<int>(i & 31);
    const int64_t tile = tq / Kq;
    const int q = static_cast<int>(tq - tile * Kq);
    uint32_t w[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t r = tile * 128 + c * 32 + lane;
      uint32_t v = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kb = 4 * q + j;
        const uint32_t b = (r < R && kb < Kb) ? src[(r / row_div) * Kb + kb] : 127u;
        v |= b << (8 * j);
      }
      w[c] = v;
    }
    *reinterpret_cast<uint4*>(dst + tq * kSfChunkBytes + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__global__ void __launch_bounds__(256) xs_transpose_kernel(const float* __restrict__ xs, const int M, const int Kb,
                                                           const int64_t ld_s, float* __restrict__ out) {
  const int64_t total = static_cast<int64_t>(M) * Kb;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t kb = i / M, m = i % M;  // consecutive threads write consecutive m
    out[kb * ld_s + m] = xs[m * Kb + kb];
  }
}

}  // namespace

cudaError_t launch_xs_transpose(const float* xs, int M, int Kb, int64_t ld_s, float* out, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(M) * Kb;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 8192) blocks = 8192;
  xs_transpose_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(xs, M, Kb, ld_s, out);
  return cudaGetLastError();
}

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
  if (total > 0x7FFFFFF0LL) return cudaErrorInvalidValue;  // group index is 32-bit
  const FastDiv div = make_fastdiv(static_cast<uint32_t>(a.layout == kScaleRowMajor ? cols : rows));
  const int gl = a.group == 32 ? 2 : 8;  // lanes per group
  const int64_t per_block = 8 * (32 / gl) * 2;  // 8 warps x groups per warp x 2 passes
  int64_t blocks = (total + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  const dim3 grid(static_cast<unsigned>(blocks)), block(256);
  const uint32_t t32 = static_cast<uint32_t>(total);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may start behind a GEMM's tail
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
#define FG8_AQ(F, L, GL) cudaLaunchKernelEx(&cfg, act_quant_kernel<F, L, GL>, a, t32, div)
  if (gl == 8) {
    if (fmt == 0) {
      if (a.layout == kScaleRowMajor) FG8_AQ(0, kScaleRowMajor, 8);
      else FG8_AQ(0, kScaleKMajor, 8);
    } else {
      if (a.layout == kScaleRowMajor) FG8_AQ(1, kScaleRowMajor, 8);
      else FG8_AQ(1, kScaleSfTiles, 8);
    }
  } else {  // 1 x 32 groups: row-major scales, or UE8M0 scale-factor tiles for the GEMM
    if (a.layout == kScaleKMajor) return cudaErrorInvalidValue;
    if (fmt == 0) FG8_AQ(0, kScaleRowMajor, 2);
    else if (a.layout == kScaleRowMajor) FG8_AQ(1, kScaleRowMajor, 2);
    else FG8_AQ(1, kScaleSfTiles, 2);
  }
#undef FG8_AQ
  return cudaGetLastError();
}

cudaError_t launch_weight_quant32(const void* w, int64_t ld_w, int N, int K, uint8_t* wq, void* ws, int fmt,
                                  cudaStream_t s) {
  const int Kb = (K + 31) / 32, Nb = (N + 31) / 32;
  const int64_t blocks = (static_cast<int64_t>(Nb) * Kb + 7) / 8;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks)), block(256);
  if (fmt == 0)
    weight_quant32_kernel<0><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(w), ld_w, N, K, Nb, Kb, wq, ws);
  else
    weight_quant32_kernel<1><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(w), ld_w, N, K, Nb, Kb, wq, ws);
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

cudaError_t launch_sf_pack(const uint8_t* src, int R, int64_t R_pad, int row_div, int Kb, uint8_t* dst,
                           cudaStream_t s) {
  const int Kq = (Kb + 3) / 4;
  if (R_pad % 128 != 0 || R_pad < R) return cudaErrorInvalidValue;
  const int64_t chunks = R_pad / 128 * Kq * 32;  // 16-byte chunks, 32 per 512-byte tile
  int64_t blocks = (chunks + 255) / 256;
  if (blocks > 8192) blocks = 8192;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, sf_pack_kernel, src, R, row_div, Kb, Kq, chunks, dst);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fg8
