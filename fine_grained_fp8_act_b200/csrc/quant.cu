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
// GL lanes own one group of 16*GL channels (8 lanes for the default 128, 4
// for 1 x 64 groups, 2 for 1 x 32): lane l loads channels [16l, 16l+16) with two 16-byte
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
        } else if (G == 64) {
          // the tensor core takes one scale per 32 K: a 1 x 64 group's byte
          // goes to both of its steps (the same word, bytes 2j and 2j+1)
          const uint32_t b = real[u] ? sbyte : 127u;
          *reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(a.xs) + sf_tile_offset(m[u], 2 * kb[u], a.Kq)) =
              static_cast<uint16_t>(b | (b << 8));
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

// One warp per B x B block, B = 32 or 64 (weight_block_size = (B, B)): lane i
// holds rows i, i + 32, ... of the block (B channels each, B/8 16-byte loads;
// the last block of a row may be 16-wide multiples when K % B != 0), amax by
// 5 xor-shuffles, 16-byte stores of 16 codes.
template <int FMT, int B>
__global__ void __launch_bounds__(256) weight_quant_small_kernel(const uint16_t* __restrict__ w, const int64_t ld_w,
                                                                 const int N, const int K, const int Nb, const int Kb,
                                                                 uint8_t* __restrict__ wq, void* __restrict__ ws) {
  constexpr int R = B / 32;  // rows per lane
  constexpr int L = B / 8;   // 16-byte loads per row
  const int lane = threadIdx.x & 31;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (blk >= static_cast<int64_t>(Nb) * Kb) return;
  const int nb = static_cast<int>(blk / Kb), kb = static_cast<int>(blk % Kb);
  const int k0 = kb * B;
  uint4 v[R][L];
  float amax = 0.0f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int n = nb * B + lane + 32 * r;
#pragma unroll
    for (int i = 0; i < L; ++i) {
      const int k = k0 + 8 * i;
      v[r][i] = (n < N && k < K) ? __ldg(reinterpret_cast<const uint4*>(w + static_cast<int64_t>(n) * ld_w + k))
                                 : make_uint4(0u, 0u, 0u, 0u);
      float f[8];
      unpack_bf16x8(v[r][i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  const float s = group_scale(amax);
  const uint32_t sbyte = FMT == 1 ? e8m0_ceil_byte(s) : 0u;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int n = nb * B + lane + 32 * r;
#pragma unroll
    for (int h = 0; h < L / 2; ++h) {
      const int k = k0 + 16 * h;
      if (n < N && k < K) {
        float f[16];
        float(&a0)[8] = *reinterpret_cast<float(*)[8]>(f);
        float(&a1)[8] = *reinterpret_cast<float(*)[8]>(f + 8);
        unpack_bf16x8(v[r][2 * h], a0);
        unpack_bf16x8(v[r][2 * h + 1], a1);
        *reinterpret_cast<uint4*>(wq + static_cast<int64_t>(n) * K + k) = quantize16<FMT>(f, s, sbyte);
      }
    }
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
// Slot kb takes source column kb / kdiv (kdiv 2: a 64-wide block's scale for
// both of its 32-wide MMA steps).
__global__ void __launch_bounds__(256) sf_pack_kernel(const uint8_t* __restrict__ src, const int R, const int row_div,
                                                      const int Kb, const int kdiv, const int Kq, const int64_t chunks,
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
        const int kb = (4 * q + j) / kdiv;
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
  const int G = a.group == 0 ? 128 : a.group;
  if (G != 32 && G != 64 && G != 128) return cudaErrorInvalidValue;
  int rows, cols;
  if (a.layout == kScaleSfTiles) {
    rows = a.M_pad;
    // group slots of the scale-factor tiles: a chunk holds 4 K-blocks of 128
    // (groups of 128; Kq chunks per row tile), or one K-block of 128 (smaller
    // groups; Kq = K-blocks per row, 128 / G groups each)
    cols = G == 128 ? a.Kq * 4 : a.Kq * (128 / G);
  } else {
    rows = a.M;
    cols = a.Kb;
  }
  const int64_t total = static_cast<int64_t>(rows) * cols;
  if (total == 0) return cudaSuccess;
  if (total > 0x7FFFFFF0LL) return cudaErrorInvalidValue;  // group index is 32-bit
  const FastDiv div = make_fastdiv(static_cast<uint32_t>(a.layout == kScaleRowMajor ? cols : rows));
  const int gl = G / 16;  // lanes per group
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
  } else if (gl == 4) {  // 1 x 64 groups
    if (fmt == 0) {
      if (a.layout == kScaleRowMajor) FG8_AQ(0, kScaleRowMajor, 4);
      else if (a.layout == kScaleKMajor) FG8_AQ(0, kScaleKMajor, 4);
      else return cudaErrorInvalidValue;
    } else {
      if (a.layout == kScaleRowMajor) FG8_AQ(1, kScaleRowMajor, 4);
      else if (a.layout == kScaleSfTiles) FG8_AQ(1, kScaleSfTiles, 4);
      else return cudaErrorInvalidValue;
    }
  } else {  // 1 x 32 groups
    if (fmt == 0) {
      if (a.layout == kScaleRowMajor) FG8_AQ(0, kScaleRowMajor, 2);
      else if (a.layout == kScaleKMajor) FG8_AQ(0, kScaleKMajor, 2);
      else return cudaErrorInvalidValue;
    } else {
      if (a.layout == kScaleRowMajor) FG8_AQ(1, kScaleRowMajor, 2);
      else if (a.layout == kScaleSfTiles) FG8_AQ(1, kScaleSfTiles, 2);
      else return cudaErrorInvalidValue;
    }
  }
#undef FG8_AQ
  return cudaGetLastError();
}

cudaError_t launch_weight_quant_small(const void* w, int64_t ld_w, int N, int K, int block, uint8_t* wq, void* ws,
                                      int fmt, cudaStream_t s) {
  if (block != 32 && block != 64) return cudaErrorInvalidValue;
  const int Kb = (K + block - 1) / block, Nb = (N + block - 1) / block;
  const int64_t blocks = (static_cast<int64_t>(Nb) * Kb + 7) / 8;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks)), thr(256);
  const uint16_t* wp = static_cast<const uint16_t*>(w);
  if (block == 32) {
    if (fmt == 0) weight_quant_small_kernel<0, 32><<<grid, thr, 0, s>>>(wp, ld_w, N, K, Nb, Kb, wq, ws);
    else weight_quant_small_kernel<1, 32><<<grid, thr, 0, s>>>(wp, ld_w, N, K, Nb, Kb, wq, ws);
  } else {
    if (fmt == 0) weight_quant_small_kernel<0, 64><<<grid, thr, 0, s>>>(wp, ld_w, N, K, Nb, Kb, wq, ws);
    else weight_quant_small_kernel<1, 64><<<grid, thr, 0, s>>>(wp, ld_w, N, K, Nb, Kb, wq, ws);
  }
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

cudaError_t launch_sf_pack(const uint8_t* src, int R, int64_t R_pad, int row_div, int Kb, int kdiv, uint8_t* dst,
                           cudaStream_t s) {
  const int Kq = (Kb * kdiv + 3) / 4;
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, sf_pack_kernel, src, R, row_div, Kb, kdiv, Kq, chunks, dst);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fg8
