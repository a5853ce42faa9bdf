// gemm.cu -- block-scaled FP8 GEMM for sm_100a (tcgen05 + TMA + TMEM).
//
//   y[M, N] = sum_kb  sx(m, kb) * sw(n/128, kb) * (xq . wq^T over K-block kb)  + bias[n]
//
// the product the Transformers fine-grained FP8 page routes every FP8Linear
// through ("Transformers 中的细粒度 FP8 量化 ... 完全指南", §八 step 6 and the
// block (128,128) + dynamic-activation fast path of §6.1).
//
// One persistent CTA per SM walks 128 x BN output tiles.  Warp roles:
//   warp 0      TMA producer: A (128 x 128 e4m3) and B (BN x 128 e4m3) tiles
//               per 128-wide K-block into a STAGES-deep shared-memory ring
//               (128-byte swizzle), plus UE8M0 scale-factor tiles.
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma (K = 32 each) per
//               K-block into a TMEM accumulator buffer.
//   warp 2      TMEM allocator.
//   warps 4..   epilogue warpgroups; warp w reads TMEM lanes 32*(w%4)..+31,
//               warpgroup g owns columns [g*BN/EPI_WG, (g+1)*BN/EPI_WG).
//
// Float scales (FMT 0): every K-block's partial product P_kb lands in its own
// TMEM buffer (ring of 4); the epilogue promotes it in registers,
// acc += P_kb * (sx * sw), so the float32 scales are applied exactly as given
// -- they are never rounded to a power of two (§七 补充 names that hazard).
// UE8M0 scales (FMT 1): tcgen05.mma.kind::mxf8f6f4.block_scale applies the
// power-of-two scales inside the tensor core (one scale per 32 K-elements,
// every group of four equal), accumulating the whole K range in TMEM.
// Ragged edges: TMA zero-fills out-of-range rows/columns of A and B (they add
// 0), and the bf16 TMA store clips rows >= M and columns >= N.
//
// Every wait is bounded (global-timer limit, shared abort flag); on expiry
// the kernel records FG8_ERR_TIMEOUT in the status word, drains its own
// in-flight copies and tensor-core ops, frees TMEM and returns.

#include <cuda.h>
#include <cuda_bf16.h>

#include "fg8_internal.h"
#include "ptx.cuh"

namespace fg8 {
namespace {

constexpr uint32_t kStatusTimeout = 6u;      // FG8_ERR_TIMEOUT
constexpr uint64_t kTeardownNs = 1000000000ull;

struct KParams {
  int M, N, K, Kb, Kq;
  int num_m, num_n, num_tiles;
  const float* xs;
  int64_t xs_sm, xs_sk;
  const float* ws;
  const uint8_t* sfa;
  const uint8_t* sfb;
  const uint16_t* bias;
  uint32_t* status;
  uint64_t wait_limit_ns;
};

template <int BN, int FMT, int STAGES, int EPI_WG>
struct Cfg {
  static constexpr int kA = kBlockM * 128;
  static constexpr int kB = BN * 128;
  static constexpr int kSF = FMT == 1 ? 2 * kSfChunkBytes : 0;
  static constexpr int kStage = kA + kB + kSF;
  static constexpr int kEpiWarps = 4 * EPI_WG;
  static constexpr int kThreads = 128 + 32 * kEpiWarps;
  static constexpr int kCols = BN / EPI_WG;
  static constexpr int kNumAcc = FMT == 0 ? 512 / BN : (512 - 16) / BN;
  static constexpr int kTmemCols = 512;
  static constexpr int kStageOut = 32 * 32 * 2;  // one 32 x 32 bf16 box
  static constexpr int kStagingBytes = kEpiWarps * 2 * kStageOut;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = 1024 + STAGES * kStage + kStagingBytes + kBarBytes;
  static_assert(kStage % 1024 == 0, "stages must keep 1024-byte alignment for the 128B swizzle");
  static_assert(kCols % 32 == 0, "epilogue works in 32-column chunks");
  static_assert(BN == 128, "one weight block row per tile (scale sw is per tile)");
  static_assert(kSmem <= 232448, "shared memory budget");
  // instruction descriptors (M = 128, K-major A and B, e4m3 x e4m3 -> f32)
  static constexpr uint32_t kIdescF8 = (1u << 4) | (uint32_t(BN >> 3) << 17) | (uint32_t(kBlockM >> 4) << 24);
  static constexpr uint32_t kIdescMx = (uint32_t(BN >> 3) << 17) | (1u << 23) | (uint32_t(kBlockM >> 4) << 24);
};

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mb, int& nb) {
  constexpr int G = 16;  // m-blocks per raster group: a wave shares A rows and B columns in L2
  const int span = G * num_n;
  const int g = t / span;
  const int first_m = g * G;
  const int gm = min(G, num_m - first_m);
  const int r = t - g * span;
  mb = first_m + r % gm;
  nb = r / gm;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, uint32_t* status) {
  *abort_flag = 1;
  atomicExch(status, kStatusTimeout);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  uint32_t(&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(r);
  tmem_ld_32x32b_x32(taddr, a);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int BN, int FMT, int STAGES, int EPI_WG>
__global__ void __launch_bounds__(Cfg<BN, FMT, STAGES, EPI_WG>::kThreads, 1)
    fg8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmY, const KParams p) {
  using C = Cfg<BN, FMT, STAGES, EPI_WG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES * C::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::kStagingBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + C::kNumAcc;
  uint64_t* teardown = tempty + C::kNumAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Kb = p.Kb;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < C::kNumAcc; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, C::kEpiWarps);
    }
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmY);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0;
      uint32_t issued_par[STAGES];
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, p.num_m, p.num_n, mb, nb);
        for (int kb = 0; kb < Kb; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, limit, abort_flag)) {
            raise_abort(abort_flag, p.status);
            ok = false;
            break;
          }
          const bool sf = FMT == 1 && (kb & 3) == 0;
          uint8_t* sa = smem + stage * C::kStage;
          mbar_arrive_expect_tx(full + stage, C::kA + C::kB + (sf ? C::kSF : 0));
          tma_load_2d(sa, &tmA, full + stage, kb * 128, mb * kBlockM);
          tma_load_2d(sa + C::kA, &tmB, full + stage, kb * 128, nb * BN);
          if (sf) {
            bulk_load(sa + C::kA + C::kB, p.sfa + (static_cast<size_t>(mb) * p.Kq + (kb >> 2)) * kSfChunkBytes,
                      kSfChunkBytes, full + stage);
            bulk_load(sa + C::kA + C::kB + kSfChunkBytes,
                      p.sfb + (static_cast<size_t>(nb) * p.Kq + (kb >> 2)) * kSfChunkBytes, kSfChunkBytes,
                      full + stage);
          }
          issued_par[stage] = phase;
          issued |= 1u << stage;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every issued copy must have landed before the CTA's shared memory goes away.
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) (void)mbar_wait(full + s, issued_par[s], kTeardownNs, nullptr);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0, abuf = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      const uint32_t sfa_t = tmem_base + static_cast<uint32_t>(C::kNumAcc * BN);
      const uint32_t sfb_t = sfa_t + 4;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        for (int kb = 0; kb < Kb; ++kb) {
          if (!mbar_wait(full + stage, phase, limit, abort_flag)) {
            raise_abort(abort_flag, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
          if (FMT == 0 || kb == 0) {
            if (!mbar_wait(tempty + abuf, aphase ^ 1u, limit, abort_flag)) {
              raise_abort(abort_flag, p.status);
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const uint32_t a_addr = smem_u32(smem + stage * C::kStage);
          const uint32_t b_addr = a_addr + C::kA;
          const uint32_t d = tmem_base + static_cast<uint32_t>(abuf * BN);
          if (FMT == 1 && (kb & 3) == 0) {
            // 128 rows x 4 K-blocks of UE8M0 scales for A and for B into TMEM
            // (issued before the MMAs that read them; tcgen05 ops of one
            // thread execute in issue order).
            tc_cp_32x128b_warpx4(sfa_t, smem_desc(b_addr + C::kB, 128, 128, 0));
            tc_cp_32x128b_warpx4(sfb_t, smem_desc(b_addr + C::kB + kSfChunkBytes, 128, 128, 0));
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = smem_desc(a_addr + k * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(b_addr + k * 32, 16, 1024, 2);
            if (FMT == 0) {
              mma_f8f6f4(d, ad, bd, C::kIdescF8, k > 0 ? 1u : 0u);
            } else {
              const uint32_t j = static_cast<uint32_t>(kb & 3);
              mma_mxf8f6f4(d, ad, bd, C::kIdescMx | (j << 29) | (j << 4), sfa_t | (j << 30), sfb_t | (j << 30),
                           (kb > 0 || k > 0) ? 1u : 0u);
            }
          }
          tc_commit(empty + stage);
          if (FMT == 0 || kb == Kb - 1) {
            tc_commit(tfull + abuf);
            if (++abuf == C::kNumAcc) {
              abuf = 0;
              aphase ^= 1u;
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // All issued tensor-core ops must finish before TMEM is released.
      tc_commit(teardown);
      (void)mbar_wait(teardown, 0, kTeardownNs, nullptr);
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- epilogue --
    const int ew = warp - 4;
    const int q = warp & 3;
    const int col0 = (ew >> 2) * C::kCols;
    uint8_t* stg = staging + ew * 2 * C::kStageOut;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int abuf = 0, nstore = 0;
    uint32_t aphase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, p.num_m, p.num_n, mb, nb);
      const int row0 = mb * kBlockM + q * 32;
      float acc[C::kCols];
      uint32_t r[C::kCols];
      if (FMT == 0) {
#pragma unroll
        for (int j = 0; j < C::kCols; ++j) acc[j] = 0.0f;
        const int row_c = min(row0 + lane, p.M - 1);
        const float* xs_row = p.xs + static_cast<int64_t>(row_c) * p.xs_sm;
        const float* ws_row = p.ws + static_cast<int64_t>(nb) * Kb;
        float sx = __ldg(xs_row), sw = __ldg(ws_row);
        for (int kb = 0; kb < Kb; ++kb) {
          const float sc = sx * sw;
          if (kb + 1 < Kb) {
            sx = __ldg(xs_row + static_cast<int64_t>(kb + 1) * p.xs_sk);
            sw = __ldg(ws_row + kb + 1);
          }
          if (!mbar_wait(tfull + abuf, aphase, limit, abort_flag)) {
            raise_abort(abort_flag, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * BN + col0);
#pragma unroll
          for (int c = 0; c < C::kCols / 32; ++c) tmem_ld32(taddr + c * 32, r + c * 32);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty + abuf);
          if (++abuf == C::kNumAcc) {
            abuf = 0;
            aphase ^= 1u;
          }
#pragma unroll
          for (int j = 0; j < C::kCols; ++j) acc[j] = fmaf(__uint_as_float(r[j]), sc, acc[j]);
        }
        if (!ok) break;
      } else {
        if (!mbar_wait(tfull + abuf, aphase, limit, abort_flag)) {
          raise_abort(abort_flag, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * BN + col0);
#pragma unroll
        for (int c = 0; c < C::kCols / 32; ++c) tmem_ld32(taddr + c * 32, r + c * 32);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty + abuf);
        if (++abuf == C::kNumAcc) {
          abuf = 0;
          aphase ^= 1u;
        }
#pragma unroll
        for (int j = 0; j < C::kCols; ++j) acc[j] = __uint_as_float(r[j]);
      }
      // + bias, round to bf16, stage a 32 x 32 box (64-byte swizzle), TMA store.
#pragma unroll
      for (int c = 0; c < C::kCols / 32; ++c) {
        const int n0 = nb * BN + col0 + c * 32;
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 bv = make_uint4(0u, 0u, 0u, 0u);
          if (p.bias != nullptr && n0 + 8 * i < p.N) bv = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + 8 * i));
          const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int j = c * 32 + 8 * i + 2 * h;
            w[4 * i + h] = pack_bf16x2(acc[j] + __uint_as_float(bw[h] << 16), acc[j + 1] + __uint_as_float(bw[h] & 0xFFFF0000u));
          }
        }
        uint8_t* buf = stg + (nstore & 1) * C::kStageOut;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int chunk = i ^ ((lane >> 1) & 3);
          *reinterpret_cast<uint4*>(buf + lane * 64 + chunk * 16) =
              make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (n0 < p.N && row0 < p.M) tma_store_2d(&tmY, buf, n0, row0);
          bulk_commit_group();
        }
        ++nstore;
      }
    }
    if (lane == 0) bulk_wait_group<0>();
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int FMT, int STAGES, int EPI_WG>
cudaError_t launch_cfg(const GemmArgs& g, int num_sms, cudaStream_t s) {
  using C = Cfg<BN, FMT, STAGES, EPI_WG>;
  CUtensorMap tA, tB, tY;
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.xq, g.K, g.M, g.K, 128, kBlockM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.wq, g.K, g.N, g.K, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.y, g.N, g.M, static_cast<uint64_t>(g.ld_y) * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  auto kern = fg8_gemm_kernel<BN, FMT, STAGES, EPI_WG>;
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  KParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.Kb = g.Kb;
  p.Kq = g.Kq;
  p.num_m = (g.M + kBlockM - 1) / kBlockM;
  p.num_n = (g.N + BN - 1) / BN;
  p.num_tiles = p.num_m * p.num_n;
  p.xs = g.xs;
  p.xs_sm = g.xs_sm;
  p.xs_sk = g.xs_sk;
  p.ws = g.ws;
  p.sfa = g.sfa;
  p.sfb = g.sfb;
  p.bias = static_cast<const uint16_t*>(g.bias);
  p.status = g.status;
  p.wait_limit_ns = g.wait_limit_ns;
  if (p.num_tiles == 0) return cudaSuccess;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  kern<<<grid, C::kThreads, C::kSmem, s>>>(tA, tB, tY, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& g, int fmt, int num_sms, cudaStream_t s) {
  if (fmt == 0) return launch_cfg<128, 0, 5, 2>(g, num_sms, s);
  return launch_cfg<128, 1, 5, 2>(g, num_sms, s);
}

}  // namespace fg8
