// gemm.cu -- block-scaled FP8 GEMM for sm_100a (tcgen05 + TMA + TMEM).
//
//   y[M, N] = sum_kb  sx(m, kb) * sw(n/128, kb) * (xq . wq^T over K-block kb)  + bias[n]
//
// the product the Transformers fine-grained FP8 page routes every FP8Linear
// through ("Transformers 中的细粒度 FP8 量化 ... 完全指南", §八 step 6 and the
// block (128,128) + dynamic-activation fast path of §6.1).
//
// One persistent CTA per SM walks 128 x BN output tiles (BN = 128 or 256).
// 384 threads in three warpgroups; the first gives up registers
// (setmaxnreg 40-80) to the two epilogue warpgroups (setmaxnreg 208-232):
//   warp 0      producer: per 128-wide K-block, TMA loads of the A tile
//               (128 x 128 e4m3) and B tile (BN x 128 e4m3) into a STAGES-deep
//               ring (128-byte swizzle); bulk copies of UE8M0 scale-factor
//               tiles (every 4th K-block) and of the tile's bias (bias ring).
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma (K = 32) per K-block.
//   warp 2      TMEM allocator.
//   warp 3      float scales: per K-block, the 128 rows' x scales and the
//               tile's weight-block scales into a shared-memory scale ring.
//   warps 4-11  epilogue: warp w reads TMEM lanes 32*(w%4)..+31; warpgroup g
//               owns columns [g*BN/2, (g+1)*BN/2).
//
// Float scales (FMT 0): each K-block's partial product P_kb goes to its own
// TMEM buffer (512/BN of them); the epilogue promotes it in registers,
// acc += P_kb * (sx * sw) starting from acc = bias, applying the float32
// scales exactly as given --
// never rounded to a power of two (§七 补充 names that hazard).  The scales
// come from the scale ring (warp 3 runs ahead of the epilogue); P_kb is read
// from TMEM 32 columns at a time with the next 32 in flight while the current
// ones are promoted by packed two-lane FMAs (each lane rounds as a scalar FMA).
// UE8M0 scales (FMT 1): tcgen05.mma.kind::mxf8f6f4.block_scale applies the
// power-of-two scales inside the tensor core (one per 32 K-elements; four
// equal ones per 128-block), accumulating the whole K range in TMEM.
// Ragged edges: TMA zero-fills out-of-range rows/columns of A and B (they add
// 0), and the bf16 TMA store clips rows >= M and columns >= N.
// Split-K tail: when the tiles leave the last wave partly empty, each tile of
// that wave is split over K into units that run on the otherwise idle SMs
// (split_plan); the epilogues of a tile's first S-1 units write their fp32
// partials to the workspace and count themselves in, and its last unit waits
// for them, adds them in split order with its own last, and stores the tile
// as usual.
//
// Every wait is bounded (global-timer limit and a shared abort flag); on
// expiry the kernel records FG8_ERR_TIMEOUT in the status word, drains its
// own in-flight copies and tensor-core ops, frees TMEM and returns.

#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>

#include "fg8_internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace fg8 {
namespace {

constexpr uint32_t kStatusTimeout = 6u;  // FG8_ERR_TIMEOUT
constexpr uint64_t kTeardownNs = 1000000000ull;
constexpr int kMaxSmem = 232448;

struct KParams {
  int M, N, K, Kb, Kq, Nb;
  int num_m, num_n, num_tiles;
  const float* xs_t;    // float path: x scales, K-major [Kb][ld_s]
  int64_t ld_s;
  const float* w_scale; // float path: weight scales [Nb][Kb] as given
  const uint8_t* sfa;   // UE8M0 path: scale-factor tiles
  const uint8_t* sfb;
  const uint16_t* bias;
  uint32_t* status;
  uint64_t wait_limit_ns;
  int test_stall;
  // output re-quantization for a next layer (REQUANT configs)
  uint8_t* nx_xq;
  void* nx_xs;
  int64_t nx_ld_s;
  int nx_Kq;
  const void* nx_w_scale;
  void* nx_w_prep;
  int nx_N;
  // grouped (MoE experts): the expert of each row, [M]; a tile computes
  // with the expert of its first row (-1: the tile is skipped).  Weights
  // [E][N][K] (one tensor map over E*N rows), float scales [E][Nb][Kb],
  // bias [E][N], UE8M0 weight scale-factor tiles sfb_tiles per expert.
  const int32_t* row_expert;  // nullptr: a plain GEMM (expert 0)
  int E;
  int sfb_tiles;
  // UE8M0 scale granularity along K: one scale-factor chunk (4 scales per
  // row) covers 4 K-blocks of 128 (sf_shift 2, 1 x 128 groups), or one
  // K-block whose 4 MMA steps of K = 32 each take their own scale (sf_shift
  // 0, 1 x 32 or 1 x 64 groups and 32 x 32 or 64 x 64 weight blocks)
  int sf_shift;
  // float scales at block size wblk (128, 64 or 32): every K-block of 128 is
  // promoted in gsteps = 128 / wblk slices of MMA steps (kps_shift = log2 of
  // the steps per slice), Kg = ceil(K / wblk) slices in all; x scales
  // [Kg][ld_s], weight scales [Nbs = ceil(N / wblk)][Kg]
  int wblk, gsteps, kps_shift, Kg, Nbs;
  // x quantized inside the kernel (QIN configs): bf16 x, the unit flags and
  // the epoch / finished-CTA words; xq_w, xs_w: where the codes and scales go
  const uint16_t* qx;
  int64_t ld_qx;
  uint32_t* qflags;
  uint32_t* qepoch;
  uint8_t* xq_w;
  void* xs_w;
  int M_pad;
  // UE8M0 QIN: this layer's weight scales [Nb][Kb] as given, packed by phase
  // one into the scale-factor tiles the producer reads (sfb_w = sfb)
  const uint8_t* wsc_src;
  uint8_t* sfb_w;
  // split-K tail: work units 0 .. split_from-1 are whole tiles, then every
  // tile from split_from on is split_s units of split_kbs K-blocks; partials
  // of units s < split_s - 1: [(tile - split_from) * (split_s - 1) + s][BN * 128]
  // fp32; split_cnt one arrival counter per split tile (zero at rest)
  int split_from, split_s, split_kbs, num_work;
  float* partials;
  uint32_t* split_cnt;
};

// One unit of a CTA's walk: a tile, the K-blocks [kb0, kb1) it computes, and
// its split index (-1: the whole tile).
struct Work {
  int tile, kb0, kb1, s;
};

template <class C>
__device__ __forceinline__ Work work_at(const KParams& p, int u) {
  Work w;
  if (!C::SPLIT || u < p.split_from) {
    w.tile = u;
    w.kb0 = 0;
    w.kb1 = p.Kb;
    w.s = -1;
  } else {
    const int j = u - p.split_from;
    const int t = j / p.split_s;
    w.tile = p.split_from + t;
    w.s = j - t * p.split_s;
    w.kb0 = w.s * p.split_kbs;
    w.kb1 = min(p.Kb, w.kb0 + p.split_kbs);
  }
  return w;
}

constexpr uint32_t kStatusBadExpert = 1u;  // FG8_ERR_INVALID_ARG

// Expert of the tile whose first row is m0.  An index past the last expert
// skips the tile like -1; the producer also records it in the status word.
__device__ __forceinline__ int tile_expert(const KParams& p, int m0, bool report) {
  if (p.row_expert == nullptr) return 0;
  const int e = p.row_expert[m0];
  if (e >= p.E) {
    if (report) atomicExch(p.status, kStatusBadExpert);
    return -1;
  }
  return e;
}

template <int BN_, int FMT_, int STAGES_, int OUTBUFS_, bool REQUANT_ = false, bool SUBK_ = false, bool QIN_ = false,
          bool SPLIT_ = false>
struct Cfg {
  static constexpr int BN = BN_, FMT = FMT_, STAGES = STAGES_;
  // SPLIT: the launch has a split-K tail (work units past the whole tiles);
  // the instance without it carries none of the hand-over code
  static constexpr bool SPLIT = SPLIT_;
  // QIN: the kernel quantizes its own x (1 x 128 groups) before the tiles
  static constexpr bool QIN = QIN_;
  // REQUANT: the epilogue also quantizes its bf16 output rows, one 128-column
  // group per thread, for a next layer (needs the 256-wide tile).
  static constexpr bool REQUANT = REQUANT_;
  // SUBK (float scales at block 64 or 32): every K-block is promoted in
  // 64- or 32-wide slices, and the weight scale changes every 64 or 32
  // columns of a thread's row; without it, one scale per K-block and thread.
  static constexpr bool SUBK = SUBK_;
  static constexpr int kA = kBlockM * 128;
  static constexpr int kB = BN * 128;
  static constexpr int kSfBytes = FMT == 1 ? kSfChunkBytes * (1 + BN / 128) : 0;
  static constexpr int kStage = (kA + kB + kSfBytes + 1023) / 1024 * 1024;
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 384;
  static constexpr int kCols = BN / 2;  // columns per epilogue thread
  static constexpr int kChunks = kCols / 32;
  static constexpr int kNumAcc = FMT == 0 ? 512 / BN : (BN == 256 ? 1 : 3);
  // UE8M0 scale factors in TMEM: two sets (A: 4 columns, B: 4 per 128 rows),
  // alternating per copy, so that a copy never lands under an MMA that may
  // still read the previous set
  static constexpr int kSfaCol = kNumAcc * BN;
  static constexpr int kSfbCol = kSfaCol + 4;
  static constexpr int kSfSetCols = 4 + BN / 32;
  static constexpr int kBiasSlot = BN * 2;
  // float scale ring: per promotion slice the 128 rows' x scales, then the
  // weight scales of the tile's column blocks (up to 8: BN / 32)
  static constexpr int kSRing = FMT == 0 ? 8 : 0;
  static constexpr int kScaleSlot = 128 * 4 + 32;
  // register split after launch (384 x 168): the wide float epilogue holds
  // 128 accumulators + 64 TMEM registers per thread, the others need less
  static constexpr uint32_t kRegsLow = (FMT == 0 && BN == 256) ? 40 : (BN == 128 ? 80 : 56);
  static constexpr uint32_t kRegsHigh = (FMT == 0 && BN == 256) ? 232 : (BN == 128 ? 208 : 224);
  static_assert(128 * kRegsLow + 256 * kRegsHigh <= 384 * 168, "register split exceeds the launch allocation");
  static constexpr int kOutBuf = 32 * 32 * 2;  // one 32 x 32 bf16 box
  // output staging boxes per epilogue warp: with kChunks of them a warp never
  // waits for its own TMA stores inside a tile
  static constexpr int kOutBufs = OUTBUFS_;
  static_assert(kOutBufs >= 1 && kOutBufs <= kChunks && kChunks % kOutBufs == 0, "staging buffers per warp");
  // shared memory map (offsets from the 1024-aligned base)
  static constexpr int kOffStaging = STAGES * kStage;
  static constexpr int kOffBias = kOffStaging + kEpiWarps * kOutBufs * kOutBuf;
  static constexpr int kOffScale = kOffBias + 2 * kBiasSlot;
  static constexpr int kOffBar = kOffScale + kSRing * kScaleSlot;
  static constexpr int kSmem = 1024 + kOffBar + 512;
  static_assert(kSmem <= kMaxSmem, "shared memory budget");
  static_assert(kStage % 1024 == 0, "stages keep 1024-byte alignment for the 128B swizzle");
  static_assert(kOffBias % 16 == 0 && kOffScale % 16 == 0 && kOffBar % 8 == 0, "alignment of rings");
  static_assert(kNumAcc * BN + (FMT == 1 ? 2 * kSfSetCols : 0) <= 512, "TMEM columns");
  static_assert(!REQUANT || BN == 256, "output re-quantization: one 128-column group per thread");
  // bytes the stage's full barrier waits for
  static constexpr uint32_t kStageTx = kA + kB;
  // instruction descriptors (M = 128, K-major A and B, e4m3 x e4m3 -> f32)
  // (kind::f8f6f4 for float scales, kind::mxf8f6f4 block-scaled for UE8M0)
  static constexpr uint32_t kIdesc = FMT == 0
                                         ? (1u << 4) | (uint32_t(BN >> 3) << 17) | (uint32_t(kBlockM >> 4) << 24)
                                         : (uint32_t(BN >> 3) << 17) | (1u << 23) | (uint32_t(kBlockM >> 4) << 24);
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

template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  uint32_t(&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(r);
  tmem_ld_32x32b_x32(taddr, a);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Ring position: slot index and the parity of its current use.
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  template <int N>
  __device__ __forceinline__ void advance() {
    if (++slot == N) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// Quantize one output row's 128-column group (bf16-rounded values in `v`) as
// the next layer's activation group: the same arithmetic, hence the same bits,
// as the stand-alone activation quantization of the stored bf16 output.
template <class C>
__device__ __forceinline__ void requant_group(const KParams& p, const uint32_t (&v)[C::kCols], int row, int n_first) {
  static_assert(C::kCols == 128, "one group per thread");
  const int valid = p.N - n_first;  // real columns of this group (may be <= 0 past N)
  const int g = n_first / 128;      // the next layer's K-block
  // four independent max chains (max is exact in any order)
  float m4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (valid >= 128) {
#pragma unroll
    for (int j = 0; j < 128; ++j) m4[j & 3] = fmaxf(m4[j & 3], fabsf(__uint_as_float(v[j])));
  } else {
#pragma unroll
    for (int j = 0; j < 128; ++j)
      if (j < valid) m4[j & 3] = fmaxf(m4[j & 3], fabsf(__uint_as_float(v[j])));
  }
  const float amax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
  const float s = qm::group_scale(amax);
  const uint32_t sbyte = C::FMT == 1 ? qm::e8m0_ceil_byte(s) : 0u;
  const bool store = row < p.M && valid > 0;
  if (store) {
    const float y = C::FMT == 0 ? __frcp_rn(s) : qm::e8m0_reciprocal(sbyte);
    uint8_t* dst = p.nx_xq + static_cast<int64_t>(row) * p.N + n_first;
#pragma unroll
    for (int c = 0; c < 8; ++c) {  // 16 values -> 16 e4m3 bytes per store
      if (c * 16 < valid) {
        float q[16];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float2 a = make_float2(__uint_as_float(v[c * 16 + i]), __uint_as_float(v[c * 16 + i + 1]));
          const float2 r = C::FMT == 0 ? qm::div2_rn_from_rcp(a, s, y) : __fmul2_rn(a, make_float2(y, y));
          q[i] = r.x;
          q[i + 1] = r.y;
        }
        *reinterpret_cast<uint4*>(dst + c * 16) =
            make_uint4(qm::pack_e4m3x4(q[0], q[1], q[2], q[3]), qm::pack_e4m3x4(q[4], q[5], q[6], q[7]),
                       qm::pack_e4m3x4(q[8], q[9], q[10], q[11]), qm::pack_e4m3x4(q[12], q[13], q[14], q[15]));
      }
    }
  }
  if constexpr (C::FMT == 0) {
    if (store) static_cast<float*>(p.nx_xs)[static_cast<int64_t>(g) * p.nx_ld_s + row] = s;
  } else {
    // every (row, K-block) byte of the tiles the next GEMM reads must be a
    // finite scale: padding rows and groups past N get 2^0
    static_cast<uint8_t*>(p.nx_xs)[sf_tile_offset(row, g, p.nx_Kq)] =
        store ? static_cast<uint8_t>(sbyte) : static_cast<uint8_t>(127);
  }
}

// Idle warps of a REQUANT launch: put the next layer's weight scales in the
// GEMM's layout, and fill the scale-factor bytes no epilogue thread owns.
// (Float: the next GEMM reads its weight scales as given; nothing to do.)
template <class C>
__device__ __forceinline__ void prepare_next_layer(const KParams& p, int idx, int stride) {
  const int Kb_next = (p.N + 127) / 128;
  if constexpr (C::FMT == 1) {
    const int cols = p.nx_Kq * 4;
    const int64_t rows = sfb_rows(p.nx_N);
    const uint8_t* ws = static_cast<const uint8_t*>(p.nx_w_scale);
    for (int64_t i = idx; i < rows * cols; i += stride) {
      const int64_t r = i / cols;
      const int kb = static_cast<int>(i % cols);
      const uint8_t b = (r < p.nx_N && kb < Kb_next) ? ws[(r / 128) * Kb_next + kb] : static_cast<uint8_t>(127);
      static_cast<uint8_t*>(p.nx_w_prep)[sf_tile_offset(r, kb, p.nx_Kq)] = b;
    }
    // activation scale-factor K-blocks beyond the tile grid
    const int first_unowned = 2 * p.num_n;
    const int64_t m_rows = static_cast<int64_t>(p.num_m) * kBlockM;
    const int64_t extra = static_cast<int64_t>(cols > first_unowned ? cols - first_unowned : 0) * m_rows;
    for (int64_t i = idx; i < extra; i += stride) {
      const int64_t r = i % m_rows;
      const int kb = first_unowned + static_cast<int>(i / m_rows);
      static_cast<uint8_t*>(p.nx_xs)[sf_tile_offset(r, kb, p.nx_Kq)] = static_cast<uint8_t>(127);
    }
  }
}

// ------------------------------------------------- in-kernel act-quant ----
// A unit: rows [128 rb, 128 rb + 128) of x, K-block kb -- 128 groups of
// 1 x 128, eight lanes per group (two 16-byte loads each), the same
// arithmetic as the stand-alone quantizer (quant_math.cuh), written in the
// layouts the GEMM reads: codes [M, K] row stride K; float scales K-major
// [Kb][ld_s]; UE8M0 bytes in the scale-factor tiles (rows past M, and the
// K-block slots past Kb in the last chunk, get 2^0).  With 384 threads (48
// groups at a time) a unit takes kUnitPasses passes; the loads of a batch of
// kUnitBatch units are all issued before any of them is quantized.
constexpr int kUnitPasses = 3;
constexpr int kUnitBatch = 2;

struct UnitLoad {
  uint4 v[kUnitPasses][2];
};

template <class C>
__device__ __forceinline__ void load_unit(const KParams& p, int u, UnitLoad& d) {
  const int rb = u / p.Kb, kb = u - (u / p.Kb) * p.Kb;
  const int oct = static_cast<int>(threadIdx.x) >> 3, l = static_cast<int>(threadIdx.x) & 7;
#pragma unroll
  for (int i = 0; i < kUnitPasses; ++i) {
    const int r = oct + i * (C::kThreads >> 3);
    const int m = rb * kBlockM + r;
    const int k = kb * 128 + l * 16;
    d.v[i][0] = d.v[i][1] = make_uint4(0u, 0u, 0u, 0u);
    if (r < kBlockM && m < p.M && k < p.K) {
      const uint4* src = reinterpret_cast<const uint4*>(p.qx + static_cast<int64_t>(m) * p.ld_qx + k);
      d.v[i][0] = __ldg(src);
      d.v[i][1] = __ldg(src + 1);
    }
  }
}

template <class C>
__device__ __forceinline__ void quantize_unit(const KParams& p, int u, const UnitLoad& d) {
  const int rb = u / p.Kb, kb = u - (u / p.Kb) * p.Kb;
  const int oct = static_cast<int>(threadIdx.x) >> 3, l = static_cast<int>(threadIdx.x) & 7;
#pragma unroll
  for (int i = 0; i < kUnitPasses; ++i) {
    const int r = oct + i * (C::kThreads >> 3);
    if (i * (C::kThreads >> 3) + (static_cast<int>(threadIdx.x) & ~31) / 8 >= kBlockM) break;  // whole warps stop
    const int m = rb * kBlockM + r;
    const bool real = r < kBlockM && m < p.M;
    const int k = kb * 128 + l * 16;
    float f[16];
    float(&f0)[8] = *reinterpret_cast<float(*)[8]>(f);
    float(&f1)[8] = *reinterpret_cast<float(*)[8]>(f + 8);
    qm::unpack_bf16x8(d.v[i][0], f0);
    qm::unpack_bf16x8(d.v[i][1], f1);
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(f[j]));
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const float s = qm::group_scale(amax);
    const uint32_t sbyte = C::FMT == 1 ? qm::e8m0_ceil_byte(s) : 0u;
    const uint4 packed = qm::quantize16<C::FMT>(f, s, sbyte);
    if (real && k < p.K) *reinterpret_cast<uint4*>(p.xq_w + static_cast<int64_t>(m) * p.K + k) = packed;
    if (l == 0 && r < kBlockM) {
      if constexpr (C::FMT == 0) {
        if (real) static_cast<float*>(p.xs_w)[static_cast<int64_t>(kb) * p.ld_s + m] = s;
      } else {
        uint8_t* sf = static_cast<uint8_t*>(p.xs_w);
        sf[sf_tile_offset(m, kb, p.Kq)] = real ? static_cast<uint8_t>(sbyte) : static_cast<uint8_t>(127);
        if (kb == p.Kb - 1)
          for (int kx = p.Kb; kx < 4 * p.Kq; ++kx) sf[sf_tile_offset(m, kx, p.Kq)] = static_cast<uint8_t>(127);
      }
    }
  }
}

// Phase one of a QIN launch, by every thread of the CTA.  UE8M0: first its
// share of the weight scale-factor tiles (16-byte pieces, the prepare step's
// packing), counted in the header's third word.  Then its share of the
// units (unit u = rb * Kb + kb on CTA u % grid, in increasing u, so the row
// blocks the first tiles need come first), each published with the epoch.
template <class C>
__device__ __forceinline__ void quantize_own_units(const KParams& p, uint32_t epoch) {
  static_assert(kUnitPasses * (C::kThreads / 8) >= kBlockM, "a unit's 128 groups in kUnitPasses passes");
  if constexpr (C::FMT == 1) {
    const int64_t pieces = sfb_rows(p.N) / 128 * p.Kq * 32;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * C::kThreads + threadIdx.x; i < pieces;
         i += static_cast<int64_t>(gridDim.x) * C::kThreads) {
      const int64_t tq = i >> 5;
      const int lane = static_cast<int>(i & 31);
      const int64_t tile = tq / p.Kq;
      const int q = static_cast<int>(tq - tile * p.Kq);
      uint32_t w[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int64_t r = tile * 128 + c * 32 + lane;
        uint32_t v = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int kb = 4 * q + j;
          const uint32_t b = (r < p.N && kb < p.Kb) ? p.wsc_src[(r / 128) * p.Kb + kb] : 127u;
          v |= b << (8 * j);
        }
        w[c] = v;
      }
      *reinterpret_cast<uint4*>(p.sfb_w + tq * kSfChunkBytes + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_global();  // read by bulk copies (async proxy) in every CTA
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      atomicAdd(p.qepoch + 2, 1u);
    }
  }
  const int units = p.num_m * p.Kb;
  const int step = static_cast<int>(gridDim.x);
  for (int u0 = static_cast<int>(blockIdx.x); u0 < units; u0 += kUnitBatch * step) {
    UnitLoad d[kUnitBatch];
#pragma unroll
    for (int j = 0; j < kUnitBatch; ++j)
      if (u0 + j * step < units) load_unit<C>(p, u0 + j * step, d[j]);
#pragma unroll
    for (int j = 0; j < kUnitBatch; ++j) {
      const int u = u0 + j * step;
      if (u >= units) break;
      quantize_unit<C>(p, u, d[j]);
      fence_proxy_async_global();  // the codes are read by TMA (async proxy) in other CTAs
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        st_release_gpu(p.qflags + u, epoch + 1u);
      }
    }
  }
}

// Wait until unit (rb, kb) of this call is quantized (QIN configs).
template <class C>
__device__ __forceinline__ bool unit_ready(const KParams& p, uint32_t epoch, int rb, int kb,
                                           volatile int* abort_flag) {
  if constexpr (!C::QIN) {
    return true;
  } else {
    if (!flag_wait(p.qflags + rb * p.Kb + kb, epoch + 1u, p.wait_limit_ns, abort_flag)) return false;
    fence_proxy_async_global();
    return true;
  }
}

// ---------------------------------------------------------------- roles ----
template <class C>
__device__ __forceinline__ void producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const KParams& p,
                                         uint8_t* smem, uint64_t* full, uint64_t* empty, uint64_t* bfull,
                                         uint64_t* bempty, volatile int* abort_flag, uint32_t epoch) {
  const uint64_t limit = p.wait_limit_ns;
  Ring st, bi;
  // most recent issue phase per slot, for the drain at the end
  uint32_t st_issued = 0, bi_issued = 0;
  uint32_t st_par[C::STAGES], bi_par[2];
  bool ok = true;
  bool w_packed = false;
  for (int u = static_cast<int>(blockIdx.x); ok && u < p.num_work; u += static_cast<int>(gridDim.x)) {
    const Work w = work_at<C>(p, u);
    int mb, nb;
    tile_coords(w.tile, p.num_m, p.num_n, mb, nb);
    const int n0 = nb * C::BN;
    const int m0 = mb * kBlockM;
    const int e = tile_expert(p, m0, true);
    if (e < 0) continue;  // every role skips the same tiles
    const int wrow0 = e * p.N + n0;  // the expert's weight rows in the [E*N, K] tensor map
    // bias of the tile (clipped to N; nothing when there is no bias)
    if (!mbar_wait(bempty + bi.slot, bi.phase ^ 1u, limit, abort_flag)) {
      raise_abort(abort_flag, p.status);
      break;
    }
    {
      const int ncols = min(C::BN, p.N - n0);
      const uint32_t bytes = p.bias != nullptr ? static_cast<uint32_t>(ncols) * 2u : 0u;
      mbar_arrive_expect_tx(bfull + bi.slot, bytes);
      if (bytes)
        bulk_load(smem + C::kOffBias + bi.slot * C::kBiasSlot, p.bias + static_cast<int64_t>(e) * p.N + n0, bytes,
                  bfull + bi.slot);
      bi_par[bi.slot] = bi.phase;
      bi_issued |= 1u << bi.slot;
      bi.template advance<2>();
    }
    for (int kb = w.kb0; kb < w.kb1; ++kb) {
      if (!mbar_wait(empty + st.slot, st.phase ^ 1u, limit, abort_flag)) {
        raise_abort(abort_flag, p.status);
        ok = false;
        break;
      }
      const bool sf = C::FMT == 1 && (kb & ((1 << p.sf_shift) - 1)) == 0;
      if constexpr (C::QIN) {  // the A tile (and, UE8M0, the chunk's four K-blocks of scales) quantized
        bool ready = true;
        if (C::FMT == 1 && !w_packed) {  // every CTA's share of the weight scale-factor tiles is in place
          ready = flag_wait(p.qepoch + 2, gridDim.x, limit, abort_flag);
          fence_proxy_async_global();
          w_packed = true;
        }
        const int last = C::FMT == 1 && sf ? min(kb + 3, p.Kb - 1) : kb;
        for (int kx = kb; ready && kx <= last; ++kx) ready = unit_ready<C>(p, epoch, mb, kx, abort_flag);
        if (!ready) {
          raise_abort(abort_flag, p.status);
          ok = false;
          break;
        }
      }
      uint8_t* sa = smem + st.slot * C::kStage;
      mbar_arrive_expect_tx(full + st.slot, C::kStageTx + (sf ? C::kSfBytes : 0));
      tma_load_2d(sa, tmA, full + st.slot, kb * 128, m0);
      tma_load_2d(sa + C::kA, tmB, full + st.slot, kb * 128, wrow0);
      if (sf) {
        uint8_t* sfs = sa + C::kA + C::kB;
        bulk_load(sfs, p.sfa + (static_cast<size_t>(m0 / kBlockM) * p.Kq + (kb >> p.sf_shift)) * kSfChunkBytes,
                  kSfChunkBytes, full + st.slot);
#pragma unroll
        for (int h = 0; h < C::BN / 128; ++h)
          bulk_load(sfs + kSfChunkBytes * (1 + h),
                    p.sfb + (static_cast<size_t>(e * p.sfb_tiles + n0 / 128 + h) * p.Kq + (kb >> p.sf_shift)) *
                                kSfChunkBytes,
                    kSfChunkBytes,
                    full + st.slot);
      }
      st_par[st.slot] = st.phase;
      st_issued |= 1u << st.slot;
      st.template advance<C::STAGES>();
    }
  }
  // Every issued copy must have landed before the CTA's shared memory goes away.
  for (int s = 0; s < C::STAGES; ++s)
    if ((st_issued >> s) & 1u) (void)mbar_wait(full + s, st_par[s], kTeardownNs, nullptr);
  for (int s = 0; s < 2; ++s)
    if ((bi_issued >> s) & 1u) (void)mbar_wait(bfull + s, bi_par[s], kTeardownNs, nullptr);
}

template <class C>
__device__ __forceinline__ void mma_issuer(const KParams& p, uint8_t* smem, uint32_t tmem_base, uint64_t* full,
                                           uint64_t* empty, uint64_t* tfull, uint64_t* tempty, uint64_t* teardown,
                                           uint64_t* stall, volatile int* abort_flag) {
  const uint64_t limit = p.wait_limit_ns;
  Ring st, ab;
  bool ok = true;
  // test hook: a barrier nothing arrives on, so the bounded wait runs out
  if (p.test_stall && !mbar_wait(stall, 0, limit, abort_flag)) {
    raise_abort(abort_flag, p.status);
    ok = false;
  }
  uint32_t sf_set = 1;  // the set the next copy goes to is sf_set ^ 1
  uint32_t sfa_t = tmem_base + static_cast<uint32_t>(C::kSfaCol);
  uint32_t sfb_t = tmem_base + static_cast<uint32_t>(C::kSfbCol);
  for (int u = static_cast<int>(blockIdx.x); ok && u < p.num_work; u += static_cast<int>(gridDim.x)) {
    const Work w = work_at<C>(p, u);
    if (p.row_expert != nullptr) {
      int mb, nb;
      tile_coords(w.tile, p.num_m, p.num_n, mb, nb);
      if (tile_expert(p, mb * kBlockM, false) < 0) continue;
    }
    for (int kb = w.kb0; kb < w.kb1; ++kb) {
      if (!mbar_wait(full + st.slot, st.phase, limit, abort_flag)) {
        raise_abort(abort_flag, p.status);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a_addr = smem_u32(smem + st.slot * C::kStage);
      const uint32_t b_addr = a_addr + C::kA;
      if constexpr (C::FMT == 0 && !C::SUBK) {
        // float: the K-block's 4 MMA steps of K = 32 into its own TMEM buffer
        if (!mbar_wait(tempty + ab.slot, ab.phase ^ 1u, limit, abort_flag)) {
          raise_abort(abort_flag, p.status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(ab.slot * C::BN);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_f8f6f4(d, smem_desc(a_addr + k * 32, 16, 1024, 2), smem_desc(b_addr + k * 32, 16, 1024, 2), C::kIdesc,
                     k > 0 ? 1u : 0u);
        tc_commit(empty + st.slot);
        tc_commit(tfull + ab.slot);
        ab.template advance<C::kNumAcc>();
        st.template advance<C::STAGES>();
        continue;
      } else if constexpr (C::FMT == 0) {
        // float at block 64 / 32: every promotion slice (2 or 1 MMA steps of
        // K = 32) into its own TMEM buffer; slices past the last real one are skipped
        const int kps = 1 << p.kps_shift;
        const int nsl = min(p.gsteps, p.Kg - kb * p.gsteps);
        for (int k = 0; k < 4 && (k >> p.kps_shift) < nsl; ++k) {
          const int j = k & (kps - 1);
          if (j == 0) {
            if (!mbar_wait(tempty + ab.slot, ab.phase ^ 1u, limit, abort_flag)) {
              raise_abort(abort_flag, p.status);
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const uint32_t d = tmem_base + static_cast<uint32_t>(ab.slot * C::BN);
          mma_f8f6f4(d, smem_desc(a_addr + k * 32, 16, 1024, 2), smem_desc(b_addr + k * 32, 16, 1024, 2),
                     C::kIdesc, j > 0 ? 1u : 0u);
          if (j == kps - 1) {
            tc_commit(tfull + ab.slot);
            ab.template advance<C::kNumAcc>();
          }
        }
        if (!ok) break;
      } else {
        if (kb == w.kb0) {
          if (!mbar_wait(tempty + ab.slot, ab.phase ^ 1u, limit, abort_flag)) {
            raise_abort(abort_flag, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const uint32_t d = tmem_base + static_cast<uint32_t>(ab.slot * C::BN);
        if ((kb & ((1 << p.sf_shift) - 1)) == 0) {
          // UE8M0 scales of 128 rows x 4 K-blocks (or 4 K = 32 steps) for A, and for B, into TMEM;
          // issued before the MMAs that read them (tcgen05 ops of one thread
          // execute in issue order).
          const uint32_t sfs = b_addr + C::kB;
          sf_set ^= 1u;
          sfa_t = tmem_base + static_cast<uint32_t>(C::kSfaCol + sf_set * C::kSfSetCols);
          sfb_t = tmem_base + static_cast<uint32_t>(C::kSfbCol + sf_set * C::kSfSetCols);
          tc_cp_32x128b_warpx4(sfa_t, smem_desc(sfs, 128, 128, 0));
#pragma unroll
          for (int h = 0; h < C::BN / 128; ++h)
            tc_cp_32x128b_warpx4(sfb_t + 4 * h, smem_desc(sfs + kSfChunkBytes * (1 + h), 128, 128, 0));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = smem_desc(a_addr + k * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(b_addr + k * 32, 16, 1024, 2);
          // the byte of each row's scale word: the K-block's (1 x 128 groups) or the step's (1 x 32, 1 x 64)
          const uint32_t j = static_cast<uint32_t>(p.sf_shift == 0 ? k : (kb & 3));
          mma_mxf8f6f4(d, ad, bd, C::kIdesc | (j << 29) | (j << 4), sfa_t | (j << 30), sfb_t | (j << 30),
                       (kb > w.kb0 || k > 0) ? 1u : 0u);
        }
        if (kb == w.kb1 - 1) {
          tc_commit(tfull + ab.slot);
          ab.template advance<C::kNumAcc>();
        }
      }
      tc_commit(empty + st.slot);
      st.template advance<C::STAGES>();
    }
  }
  // All issued tensor-core ops must finish before TMEM is released.
  tc_commit(teardown);
  (void)mbar_wait(teardown, 0, kTeardownNs, nullptr);
}

// Float scales, one warp: for each tile of the CTA's walk and each of its
// promotion slices (the K-blocks, or their 64- / 32-wide parts for smaller
// blocks), the x scales of the tile's 128 rows (K-major layout: 512
// contiguous bytes, 16 per lane) and the weight scale of each of the tile's
// column blocks are copied asynchronously (cp.async) into the next slot of
// the scale ring; each lane's copies complete the slot's barrier as they
// land, so up to kSRing slices of scale loads are in flight and their
// latency stays off the epilogue's path.  The epilogue warps release slots.
template <class C>
__device__ __forceinline__ void scale_loader(const KParams& p, uint8_t* smem, uint64_t* sfull, uint64_t* sempty,
                                             volatile int* abort_flag, int lane, uint32_t epoch) {
  const uint64_t limit = p.wait_limit_ns;
  Ring sr;
  for (int u = static_cast<int>(blockIdx.x); u < p.num_work; u += static_cast<int>(gridDim.x)) {
    const Work w = work_at<C>(p, u);
    int mb, nb;
    tile_coords(w.tile, p.num_m, p.num_n, mb, nb);
    const int e = tile_expert(p, mb * kBlockM, false);
    if (e < 0) continue;
    const float* xs = p.xs_t + mb * kBlockM + 4 * lane;
    // the weight-scale block of lane j's slot (j < BN / wblk); a block past N
    // (ragged last tile) reads the last block: its columns are never stored
    const int nwb = C::BN / p.wblk;
    const int wb = e * p.Nbs + min(nb * C::BN / p.wblk + (lane & 7), p.Nbs - 1);
    const float* ws = p.w_scale + static_cast<int64_t>(wb) * p.Kg;
    const int g1 = min(p.Kg, w.kb1 * p.gsteps);
    for (int g = w.kb0 * p.gsteps; g < g1; ++g) {
      if (!mbar_wait_warp(sempty + sr.slot, sr.phase ^ 1u, limit, abort_flag)) {
        raise_abort(abort_flag, p.status);
        cp_async_wait_all();
        return;
      }
      if (!__all_sync(0xFFFFFFFFu, unit_ready<C>(p, epoch, mb, g, abort_flag))) {  // QIN: this unit's scales
        raise_abort(abort_flag, p.status);
        cp_async_wait_all();
        return;
      }
      float* slot = reinterpret_cast<float*>(smem + C::kOffScale + sr.slot * C::kScaleSlot);
      cp_async16(slot + 4 * lane, xs + static_cast<int64_t>(g) * p.ld_s);
      if (lane < nwb) cp_async4(slot + 128 + lane, ws + g);
      cp_async_mbar_arrive(sfull + sr.slot);  // one arrival per lane, when its copies have landed
      sr.template advance<C::kSRing>();
    }
  }
  cp_async_wait_all();  // the CTA's shared memory must outlive every copy in flight
}

template <class C>
__device__ __forceinline__ void epilogue(const CUtensorMap* tmY, const KParams& p, uint8_t* smem, uint32_t tmem_base,
                                         uint64_t* tfull, uint64_t* tempty, uint64_t* bfull, uint64_t* bempty,
                                         uint64_t* sfull, uint64_t* sempty, uint64_t* xbar, uint64_t* ybar,
                                         volatile uint32_t* xlast, volatile int* abort_flag, int warp, int lane) {
  const uint64_t limit = p.wait_limit_ns;
  const int ew = warp - 4;
  const int q = warp & 3;      // TMEM lane quadrant
  const int wg = ew >> 2;      // column half of the tile
  const int col0 = wg * C::kCols;
  uint8_t* stg = smem + C::kOffStaging + ew * C::kOutBufs * C::kOutBuf;
  const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
  Ring ab, bi, sr;
  bool ok = true;
  const int sub_row = q * 32 + lane;  // this thread's row inside a tile
  uint32_t xph = 0;                   // parity of the split hand-over barriers
  for (int u = static_cast<int>(blockIdx.x); ok && u < p.num_work; u += static_cast<int>(gridDim.x)) {
    const Work w = work_at<C>(p, u);
    int mb, nb;
    tile_coords(w.tile, p.num_m, p.num_n, mb, nb);
    if (tile_expert(p, mb * kBlockM, false) < 0) continue;
    const int row0 = mb * kBlockM + q * 32;
    // the tile's bias (bias ring; zeros past N or without bias)
    if (!mbar_wait_warp(bfull + bi.slot, bi.phase, limit, abort_flag)) {
      raise_abort(abort_flag, p.status);
      break;
    }
    const uint8_t* bias_s = smem + C::kOffBias + bi.slot * C::kBiasSlot;
    uint32_t acc[C::kCols];  // float bits
    if constexpr (C::FMT == 0) {
      // the promotion accumulates onto the bias: y = bias + sum_kb P_kb * s_kb
      // (a split tile's first unit starts from the bias, the others from 0)
#pragma unroll
      for (int i = 0; i < C::kCols / 8; ++i) {
        uint4 bv = make_uint4(0u, 0u, 0u, 0u);
        if (p.bias != nullptr && w.s <= 0 && nb * C::BN + col0 + 8 * i < p.N)
          bv = *reinterpret_cast<const uint4*>(bias_s + (col0 + 8 * i) * 2);
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          acc[8 * i + 2 * h] = bw[h] << 16;
          acc[8 * i + 2 * h + 1] = bw[h] & 0xFFFF0000u;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bempty + bi.slot);
      bi.template advance<2>();
      const int g1 = min(p.Kg, w.kb1 * p.gsteps);
      for (int g = w.kb0 * p.gsteps; g < g1; ++g) {
        // sx(m, g) * sw(block of the chunk's columns, g) from the scale ring
        if (!mbar_wait_warp(sfull + sr.slot, sr.phase, limit, abort_flag)) {
          raise_abort(abort_flag, p.status);
          ok = false;
          break;
        }
        const float* slot = reinterpret_cast<const float*>(smem + C::kOffScale + sr.slot * C::kScaleSlot);
        const float sx = slot[sub_row];
        constexpr int kScales = C::SUBK ? C::kChunks : 1;  // one per 32-column chunk, or one for the thread
        float2 s2[kScales];
#pragma unroll
        for (int c = 0; c < kScales; ++c) {
          const float sc = sx * slot[128 + ((col0 + 32 * c) >> (p.kps_shift + 5))];  // wblk = 32 << kps_shift
          s2[c] = make_float2(sc, sc);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sempty + sr.slot);
        sr.template advance<C::kSRing>();
        if (!mbar_wait_warp(tfull + ab.slot, ab.phase, limit, abort_flag)) {
          raise_abort(abort_flag, p.status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(ab.slot * C::BN + col0);
        // two 32-column TMEM loads per wait: chunks c, c+1 are promoted while
        // c+2, c+3 load into the same registers; the buffer goes back after
        // the last wait
        static_assert(C::kChunks % 2 == 0, "chunk pairs");
        uint32_t r[2][32];
        tmem_ld32(taddr, r[0]);
        tmem_ld32(taddr + 32, r[1]);
        tmem_wait_ld();
        tmem_reg_fence(r[0]);
        tmem_reg_fence(r[1]);
#pragma unroll
        for (int c = 0; c < C::kChunks; c += 2) {
          const bool more = c + 2 < C::kChunks;
          if (!more) {  // every column of this K-block is in registers: hand the buffer back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + ab.slot);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {  // acc += P * s, two lanes per packed FMA
              uint32_t* a = acc + (c + h) * 32 + j;
              const float2 o = __ffma2_rn(make_float2(__uint_as_float(r[h][j]), __uint_as_float(r[h][j + 1])),
                                          s2[C::SUBK ? c + h : 0],
                                          make_float2(__uint_as_float(a[0]), __uint_as_float(a[1])));
              a[0] = __float_as_uint(o.x);
              a[1] = __float_as_uint(o.y);
            }
            if (more) tmem_ld32(taddr + (c + 2 + h) * 32, r[h]);
          }
          if (more) {
            tmem_wait_ld();
            tmem_reg_fence(r[0]);
            tmem_reg_fence(r[1]);
          }
        }
        ab.template advance<C::kNumAcc>();
      }
      if (!ok) break;
    } else {
      if (!mbar_wait_warp(tfull + ab.slot, ab.phase, limit, abort_flag)) {
        raise_abort(abort_flag, p.status);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(ab.slot * C::BN + col0);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c) tmem_ld32(taddr + c * 32, acc + c * 32);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c) tmem_reg_fence(acc + c * 32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + ab.slot);
      ab.template advance<C::kNumAcc>();
    }

    if (C::SPLIT && w.s >= 0) {
      // A unit of a split tile.  Units 0 .. S-2 write their partial sums
      // (fp32, each thread's columns as float4s, contiguous per warp) and
      // count themselves in; unit S-1 waits for that count, adds the others'
      // partials in split order and its own last, and goes on to store the
      // tile.  All units of a split tile are in the last wave (one per CTA).
      constexpr int kVec = C::kCols / 4;
      const int j = w.tile - p.split_from;
      const int et = ew * 32 + lane;
      const bool reducer = w.s == p.split_s - 1;
      const float4* part = reinterpret_cast<const float4*>(p.partials) +
                           static_cast<int64_t>(j) * (p.split_s - 1) * (kVec * 256) + et;
      if (!reducer) {
        float4* mine = const_cast<float4*>(part) + static_cast<int64_t>(w.s) * (kVec * 256);
#pragma unroll
        for (int i = 0; i < kVec; ++i)
          __stcg(mine + i * 256, make_float4(__uint_as_float(acc[4 * i]), __uint_as_float(acc[4 * i + 1]),
                                             __uint_as_float(acc[4 * i + 2]), __uint_as_float(acc[4 * i + 3])));
        __threadfence();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar);
      if (ew == 0 && lane == 0) {
        bool fine = mbar_wait(xbar, xph, limit, abort_flag);
        if (fine && !reducer) {
          __threadfence();
          atomicAdd(p.split_cnt + j, 1u);
        } else if (fine) {  // every other unit's partial is out; zero the counter for the next call
          fine = flag_wait(p.split_cnt + j, static_cast<uint32_t>(p.split_s - 1), limit, abort_flag);
          if (fine) {
            __threadfence();
            atomicExch(p.split_cnt + j, 0u);
          }
        }
        *xlast = fine ? 1u : 2u;
        mbar_arrive(ybar);
      }
      const bool got = mbar_wait_warp(ybar, xph, limit, abort_flag);
      xph ^= 1u;
      if (!got || *xlast == 2u) {
        raise_abort(abort_flag, p.status);
        break;
      }
      if (!reducer) {
        if constexpr (C::FMT == 1) {  // the bias slot is not needed
          __syncwarp();
          if (lane == 0) mbar_arrive(bempty + bi.slot);
          bi.template advance<2>();
        }
        continue;
      }
      constexpr int kBatch = 4;  // float4s per thread in flight per partial
#pragma unroll
      for (int i0 = 0; i0 < kVec; i0 += kBatch) {
        float4 t[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) t[i] = __ldcg(part + (i0 + i) * 256);
        for (int sp = 1; sp < p.split_s - 1; ++sp) {
          const float4* ps = part + static_cast<int64_t>(sp) * (kVec * 256);
          float4 r[kBatch];
#pragma unroll
          for (int i = 0; i < kBatch; ++i) r[i] = __ldcg(ps + (i0 + i) * 256);
#pragma unroll
          for (int i = 0; i < kBatch; ++i) {
            t[i].x = __fadd_rn(t[i].x, r[i].x);
            t[i].y = __fadd_rn(t[i].y, r[i].y);
            t[i].z = __fadd_rn(t[i].z, r[i].z);
            t[i].w = __fadd_rn(t[i].w, r[i].w);
          }
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
          uint32_t* a = acc + 4 * (i0 + i);
          a[0] = __float_as_uint(__fadd_rn(t[i].x, __uint_as_float(a[0])));
          a[1] = __float_as_uint(__fadd_rn(t[i].y, __uint_as_float(a[1])));
          a[2] = __float_as_uint(__fadd_rn(t[i].z, __uint_as_float(a[2])));
          a[3] = __float_as_uint(__fadd_rn(t[i].w, __uint_as_float(a[3])));
        }
      }
    }

    // (UE8M0: + bias), round to bf16, stage 32 x 32 boxes (64-byte swizzle),
    // store them with TMA: one proxy fence and one bulk group per batch of
    // kOutBufs boxes.
    if (lane == 0) bulk_wait_group_read<0>();  // the previous tile's stores have read the boxes
    __syncwarp();
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c) {
      const int b = c % C::kOutBufs;
      if (c >= C::kOutBufs && b == 0) {  // reusing the boxes: the previous batch must have been read
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
      }
      const int nloc = col0 + c * 32;
      const int n0 = nb * C::BN + nloc;
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 bv = make_uint4(0u, 0u, 0u, 0u);
        if (C::FMT == 1 && p.bias != nullptr && n0 + 8 * i < p.N)
          bv = *reinterpret_cast<const uint4*>(bias_s + (nloc + 8 * i) * 2);
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int j = c * 32 + 8 * i + 2 * h;
          w[4 * i + h] = C::FMT == 0 ? pack_bf16x2(__uint_as_float(acc[j]), __uint_as_float(acc[j + 1]))
                                     : pack_bf16x2(__uint_as_float(acc[j]) + __uint_as_float(bw[h] << 16),
                                                   __uint_as_float(acc[j + 1]) + __uint_as_float(bw[h] & 0xFFFF0000u));
          if constexpr (C::REQUANT) {  // keep the bf16-rounded values: they are the next layer's input
            acc[j] = w[4 * i + h] << 16;
            acc[j + 1] = w[4 * i + h] & 0xFFFF0000u;
          }
        }
      }
      uint8_t* buf = stg + b * C::kOutBuf;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int chunk = i ^ ((lane >> 1) & 3);
        *reinterpret_cast<uint4*>(buf + lane * 64 + chunk * 16) =
            make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
      if (b == C::kOutBufs - 1) {  // the batch is staged: make it visible to TMA and store it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int cc = c - b; cc <= c; ++cc) {
            const int nn = nb * C::BN + col0 + cc * 32;
            if (nn < p.N && row0 < p.M) tma_store_2d(tmY, stg + (cc % C::kOutBufs) * C::kOutBuf, nn, row0);
          }
          bulk_commit_group();
        }
      }
    }
    if constexpr (C::FMT == 1) {  // the bias slot was read in the store phase
      __syncwarp();
      if (lane == 0) mbar_arrive(bempty + bi.slot);
      bi.template advance<2>();
    }
    if constexpr (C::REQUANT) requant_group<C>(p, acc, row0 + lane, nb * C::BN + col0);
  }
  if (lane == 0) bulk_wait_group<0>();
}

template <class C>
__global__ void __launch_bounds__(384, 1)
    fg8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmY, const KParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + C::kNumAcc;
  uint64_t* bfull = tempty + C::kNumAcc;
  uint64_t* bempty = bfull + 2;
  uint64_t* sfull = bempty + 2;
  uint64_t* sempty = sfull + C::kSRing;
  uint64_t* teardown = sempty + C::kSRing;
  uint64_t* stall = teardown + 1;
  uint64_t* xbar = stall + 1;  // split tiles: the epilogue warps' partials are out
  uint64_t* ybar = xbar + 1;   // ... and the unit has been counted (verdict in xlast)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ybar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile uint32_t* xlast = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);
  static_assert(C::kOffBar + 8 * (2 * C::STAGES + 2 * C::kNumAcc + 4 + 2 * C::kSRing + 4) + 16 <= C::kOffBar + 512,
                "barrier block");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    // the descriptors' fetch overlaps the barrier set-up before the first copy
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmY);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < C::kNumAcc; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, C::kEpiWarps);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bfull + s, 1);
      mbar_init(bempty + s, C::kEpiWarps);
    }
    for (int s = 0; s < C::kSRing; ++s) {
      mbar_init(sfull + s, 32);             // every lane of the scale warp
      mbar_init(sempty + s, C::kEpiWarps);
    }
    mbar_init(teardown, 1);
    mbar_init(stall, 1);
    mbar_init(xbar, C::kEpiWarps);
    mbar_init(ybar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above overlapped the preceding kernel (programmatic dependent
  // launch); from here on its outputs (quantized activations, scales) are read.
  grid_wait_prerequisites();
  grid_launch_dependents();  // the next kernel may take SMs as this grid's CTAs finish
  uint32_t epoch = 0;
  if constexpr (C::QIN) {
    epoch = ld_acquire_gpu(p.qepoch);
    quantize_own_units<C>(p, epoch);
  }

  if (warp < 4) {
    setmaxnreg_dec<C::kRegsLow>();
    if (warp == 0 && lane == 0)
      producer<C>(&tmA, &tmB, p, smem, full, empty, bfull, bempty, abort_flag, epoch);
    else if (warp == 1 && lane == 0)
      mma_issuer<C>(p, smem, tmem_base, full, empty, tfull, tempty, teardown, stall, abort_flag);
    if constexpr (C::FMT == 0) {
      if (warp == 3) scale_loader<C>(p, smem, sfull, sempty, abort_flag, lane, epoch);
    }
    if constexpr (C::REQUANT && C::FMT == 1) {
      if (warp == 2 || warp == 3)
        prepare_next_layer<C>(p, static_cast<int>(blockIdx.x) * 64 + (warp - 2) * 32 + lane,
                              static_cast<int>(gridDim.x) * 64);
    }
  } else {
    setmaxnreg_inc<C::kRegsHigh>();
    epilogue<C>(&tmY, p, smem, tmem_base, tfull, tempty, bfull, bempty, sfull, sempty, xbar, ybar, xlast, abort_flag,
                warp, lane);
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }

  if constexpr (C::QIN) {
    // the last CTA out advances the epoch: every CTA has read it and every
    // unit flag of this call holds epoch + 1, which no later call waits for
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(p.qepoch + 1, 1u) == gridDim.x - 1) {
        p.qepoch[1] = 0u;
        p.qepoch[2] = 0u;
        __threadfence();
        atomicAdd(p.qepoch, 1u);
      }
    }
  }
}

// ------------------------------------------------------------------ host ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // looked up once per process (thread-safe static initialisation)
  static const EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
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

template <class C>
cudaError_t launch_cfg(const GemmArgs& g, int num_sms, cudaStream_t s) {
  CUtensorMap tA, tB, tY;
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.xq, g.K, g.M, g.K, 128, kBlockM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.wq, g.K,
                    static_cast<uint64_t>(g.N) * (g.row_expert != nullptr ? g.E : 1), g.K, 128, C::BN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.y, g.N, g.M, static_cast<uint64_t>(g.ld_y) * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  auto kern = fg8_gemm_kernel<C>;
  KParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.Kb = g.Kb;
  p.Kq = g.Kq;
  p.Nb = (g.N + 127) / 128;
  p.num_m = (g.M + kBlockM - 1) / kBlockM;
  p.num_n = (g.N + C::BN - 1) / C::BN;
  p.num_tiles = p.num_m * p.num_n;
  p.xs_t = g.xs_t;
  p.ld_s = g.ld_s;
  p.w_scale = g.w_scale;
  p.sfa = g.sfa;
  p.sfb = g.sfb;
  p.bias = static_cast<const uint16_t*>(g.bias);
  p.status = g.status;
  p.wait_limit_ns = g.wait_limit_ns;
  p.test_stall = g.test_stall;
  p.nx_xq = g.nx_xq;
  p.nx_xs = g.nx_xs;
  p.nx_ld_s = g.nx_ld_s;
  p.nx_Kq = g.nx_Kq;
  p.nx_w_scale = g.nx_w_scale;
  p.nx_w_prep = g.nx_w_prep;
  p.nx_N = g.nx_N;
  p.row_expert = g.row_expert;
  p.E = g.row_expert != nullptr ? g.E : 1;
  p.sfb_tiles = g.sfb_tiles;
  p.sf_shift = g.sf32 ? 0 : 2;
  p.wblk = g.wblk == 0 ? 128 : g.wblk;
  p.gsteps = 128 / p.wblk;
  p.kps_shift = p.wblk == 128 ? 2 : (p.wblk == 64 ? 1 : 0);
  p.Kg = (g.K + p.wblk - 1) / p.wblk;
  p.Nbs = (g.N + p.wblk - 1) / p.wblk;
  p.qx = static_cast<const uint16_t*>(g.qx);
  p.ld_qx = g.ld_qx;
  p.qflags = g.qflags;
  p.qepoch = g.qepoch;
  p.xq_w = static_cast<uint8_t*>(const_cast<void*>(g.xq));
  p.xs_w = C::FMT == 0 ? static_cast<void*>(const_cast<float*>(g.xs_t))
                       : static_cast<void*>(const_cast<uint8_t*>(g.sfa));
  p.M_pad = (g.M + kBlockM - 1) / kBlockM * kBlockM;
  p.wsc_src = static_cast<const uint8_t*>(g.qwsc);
  p.sfb_w = const_cast<uint8_t*>(g.sfb);
  if (p.num_tiles == 0) return cudaSuccess;
  // the split-K tail: tiled GEMMs with room for the partials (not the
  // expert-grouped or sliced-promotion variants)
  p.split_from = p.num_tiles;
  p.split_s = 1;
  p.split_kbs = p.Kb;
  p.partials = nullptr;
  p.split_cnt = nullptr;
  static_assert(!C::SPLIT || !C::QIN, "the in-launch quantization runs short K, which never splits");
  if (C::SPLIT && g.row_expert == nullptr && g.split_ws != nullptr) {
    const SplitPlan pl = split_plan(p.num_tiles, p.num_m, p.Kb, C::FMT == 1 && !g.sf32 ? 4 : 1, num_sms);
    if (pl.from < p.num_tiles && split_area_bytes(pl, p.num_tiles, C::BN) <= g.split_bytes &&
        p.num_tiles - pl.from <= kHeaderCounters) {
      p.split_from = pl.from;
      p.split_s = pl.s;
      p.split_kbs = pl.kbs;
      p.partials = reinterpret_cast<float*>(g.split_ws);
      p.split_cnt = g.status + kHeaderCounterOffset / 4;
    }
  }
  p.num_work = p.split_from + (p.num_tiles - p.split_from) * p.split_s;

  // the shared-memory opt-in once per device: one bit per device; calls from
  // several host threads may repeat it, which is harmless
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if ((configured.load(std::memory_order_acquire) & bit) == 0) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  // start early behind the activation quantization (the kernel waits for its
  // results before reading them)
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(p.num_work < num_sms ? p.num_work : num_sms);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tA, tB, tY, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <class Plain, class Split>
cudaError_t launch_either(bool split, const GemmArgs& g, int num_sms, cudaStream_t s) {
  return split ? launch_cfg<Split>(g, num_sms, s) : launch_cfg<Plain>(g, num_sms, s);
}

// Estimated time of a split tail: units of k K-blocks, se of them per tile
// (K-block periods; see split_plan).
double split_cost(int k, int se) { return k + 4.0 + 3.0 * (se - 1); }

}  // namespace

SplitPlan split_plan(int tiles, int m_blocks, int Kb, int kb_align, int sms) {
  SplitPlan pl;
  pl.from = tiles;
  pl.kbs = Kb;
  // Measured on the B200: with fewer than 64 K-blocks per tile the CTAs'
  // spread in finishing their whole tiles eats the gain; with a single row
  // block the tiles stream distinct weights and are bound by that, split or
  // not.  The spread grows with the whole waves before the tail: past 6 of
  // them a split has to save 60 K-block periods (it then gained 1-3% on
  // 3584- to 8192-token layers of 96 and 144 K-blocks with a nearly empty
  // last wave, and lost ~0.5% where it saved 41), past 16 none is tried.
  const int waves = sms > 0 ? tiles / sms : 0;
  if (tiles <= 0 || sms <= 0 || Kb < 64 || m_blocks < 2 || waves > 16) return pl;
  const int rem = tiles % sms;
  if (rem == 0) return pl;
  // Cost of the tail in K-block periods: unsplit, a whole tile's K loop;
  // split, a unit's K-blocks plus the write-back of the partials, the wait
  // and the last unit's reading of the other S - 1 partials (128 KB each
  // from L2 at ~0.1 TB/s per SM against ~0.6 us per 128 x 256 x 128
  // K-block), fitted to timings of 2048- to 8192-token layers.
  double best = waves > 6 ? Kb - 60 : Kb;
  for (int S = 2; S <= Kb && rem * S <= sms; ++S) {
    const int kbs = (Kb + S - 1) / S;
    const int k = (kbs + kb_align - 1) / kb_align * kb_align;
    const int se = (Kb + k - 1) / k;
    if (se < 2 || rem * se > sms) continue;
    const double cost = split_cost(k, se);
    if (cost < best) {
      best = cost;
      pl.from = tiles - rem;
      pl.s = se;
      pl.kbs = k;
    }
  }
  return pl;
}

size_t split_area_bytes(const SplitPlan& pl, int tiles, int bn) {
  if (pl.from >= tiles) return 0;
  // the last unit of a tile keeps its partial in registers
  return static_cast<size_t>(tiles - pl.from) * (pl.s - 1) * bn * kBlockM * sizeof(float);
}

size_t gemm_split_area(int64_t M, int64_t N, int64_t K, int fmt, int sms) {
  const int64_t m_tiles = (M + kBlockM - 1) / kBlockM;
  const int Kb = static_cast<int>((K + 127) / 128);
  size_t area = 0;
  for (int bn : {128, 256}) {
    const int64_t tiles = m_tiles * ((N + bn - 1) / bn);
    if (tiles > (int64_t(1) << 30)) continue;
    const int t = static_cast<int>(tiles);
    const SplitPlan pl = split_plan(t, static_cast<int>(m_tiles), Kb, fmt == 1 ? 4 : 1, sms);
    if (t - pl.from > kHeaderCounters) continue;
    const size_t a = split_area_bytes(pl, t, bn);
    if (a > area) area = a;
  }
  return area;
}

int choose_block_n(int M, int N, int Kb, int kb_align, int num_sms, bool split) {
  const int m_blocks = static_cast<int>((M + kBlockM - 1) / kBlockM);
  // Per-CTA time in K-block periods of the tile: the whole waves' K loops
  // plus the tail (unsplit: one more K loop; split: the plan's estimate).
  // The 256-wide tile moves ~1.6x more MMA work per operand byte and per
  // epilogue instruction, so a 128-wide K-block costs ~0.6 / 0.5 of one.
  const int64_t m_tiles = (M + kBlockM - 1) / kBlockM;
  auto cost = [&](int bn) {
    const int64_t tiles64 = m_tiles * ((N + bn - 1) / bn);
    const int tiles = static_cast<int>(tiles64 < (int64_t(1) << 30) ? tiles64 : (int64_t(1) << 30));
    double t = static_cast<double>((tiles + num_sms - 1) / num_sms) * Kb;
    if (split) {
      const SplitPlan pl = split_plan(tiles, m_blocks, Kb, kb_align, num_sms);
      if (pl.from < tiles && tiles - pl.from <= kHeaderCounters)
        t = static_cast<double>(pl.from / num_sms) * Kb + split_cost(pl.kbs, pl.s);
    }
    return t * (bn == 128 ? 128.0 / 0.6 : 256.0);
  };
  return cost(128) < cost(256) ? 128 : 256;
}

cudaError_t launch_gemm(const GemmArgs& g, int fmt, int num_sms, cudaStream_t s) {
  // Short K: few K-blocks per tile, so the tile's output path dominates --
  // give every output chunk its own staging box and keep one stage fewer.
  // Long K: four stages (the float path's scale ring takes the shared memory
  // of the second staging box per warp).  Measured crossover: float up to 32
  // K-blocks per tile; UE8M0, whose MMAs run faster and want the deeper
  // ring, up to 8 (12 to 32 K-blocks ran 7-18% faster with four stages).
  const bool short_k = g.Kb <= (fmt == 1 ? 8 : 32);
  const int align = fmt == 1 ? 4 : 1;
  // (the split-K tail only runs for block-128 scales with room for it)
  const bool may_split = g.split_ws != nullptr && g.row_expert == nullptr && !g.sf32 && (g.wblk == 0 || g.wblk == 128);
  // does the plan for bn-wide tiles split (and fit the room)?  Then the
  // launch takes the instance with the hand-over code.
  auto splits = [&](int bn) {
    if (!may_split) return false;
    const int m_tiles = (g.M + kBlockM - 1) / kBlockM;
    const int tiles = m_tiles * ((g.N + bn - 1) / bn);
    const SplitPlan pl = split_plan(tiles, m_tiles, g.Kb, align, num_sms);
    return pl.from < tiles && tiles - pl.from <= kHeaderCounters && split_area_bytes(pl, tiles, bn) <= g.split_bytes;
  };
  if (g.qx != nullptr) {  // x quantized inside the kernel: short K only (see can_quantize_in_gemm)
    if (g.Kb > 32 || g.wblk > 0 && g.wblk != 128 || g.row_expert != nullptr) return cudaErrorInvalidValue;
    const bool requant = g.nx_xq != nullptr;
    // the tile width fg8_linear picks, so that both give the same bits (short
    // K never splits: the split-K tail needs at least 64 K-blocks)
    const int bnq = requant ? 256 : choose_block_n(g.M, g.N, g.Kb, align, num_sms, may_split);
    if (fmt == 0) {
      if (requant) return launch_cfg<Cfg<256, 0, 3, 4, true, false, true>>(g, num_sms, s);
      if (bnq == 256) return launch_cfg<Cfg<256, 0, 3, 4, false, false, true>>(g, num_sms, s);
      return launch_cfg<Cfg<128, 0, 5, 2, false, false, true>>(g, num_sms, s);
    }
    if (requant) return launch_cfg<Cfg<256, 1, 3, 4, true, false, true>>(g, num_sms, s);
    if (bnq == 256) return launch_cfg<Cfg<256, 1, 3, 4, false, false, true>>(g, num_sms, s);
    return launch_cfg<Cfg<128, 1, 5, 2, false, false, true>>(g, num_sms, s);
  }
  if (g.nx_xq != nullptr) {  // output re-quantization needs the 256-wide tile
    if (fmt == 0) {
      if (short_k) return launch_cfg<Cfg<256, 0, 3, 4, true>>(g, num_sms, s);
      return launch_either<Cfg<256, 0, 4, 1, true>, Cfg<256, 0, 4, 1, true, false, false, true>>(splits(256), g,
                                                                                               num_sms, s);
    }
    if (short_k) return launch_cfg<Cfg<256, 1, 3, 4, true>>(g, num_sms, s);
    return launch_either<Cfg<256, 1, 4, 1, true>, Cfg<256, 1, 4, 1, true, false, false, true>>(splits(256), g,
                                                                                             num_sms, s);
  }
  const int bn = choose_block_n(g.M, g.N, g.Kb, align, num_sms, may_split);
  if (fmt == 0 && g.wblk != 0 && g.wblk != 128) {  // float at block 64 / 32 (never split)
    if (bn == 256) {
      if (short_k) return launch_cfg<Cfg<256, 0, 3, 4, false, true>>(g, num_sms, s);
      return launch_cfg<Cfg<256, 0, 4, 1, false, true>>(g, num_sms, s);
    }
    return launch_cfg<Cfg<128, 0, 5, 2, false, true>>(g, num_sms, s);
  }
  const bool sp = splits(bn);
  if (fmt == 0) {
    if (bn == 256) {
      if (short_k) return launch_cfg<Cfg<256, 0, 3, 4>>(g, num_sms, s);
      return launch_either<Cfg<256, 0, 4, 1>, Cfg<256, 0, 4, 1, false, false, false, true>>(sp, g, num_sms, s);
    }
    return launch_either<Cfg<128, 0, 5, 2>, Cfg<128, 0, 5, 2, false, false, false, true>>(sp, g, num_sms, s);
  }
  if (bn == 256) {
    if (short_k) return launch_cfg<Cfg<256, 1, 3, 4>>(g, num_sms, s);
    return launch_either<Cfg<256, 1, 4, 1>, Cfg<256, 1, 4, 1, false, false, false, true>>(sp, g, num_sms, s);
  }
  return launch_either<Cfg<128, 1, 5, 2>, Cfg<128, 1, 5, 2, false, false, false, true>>(sp, g, num_sms, s);
}

}  // namespace fg8
