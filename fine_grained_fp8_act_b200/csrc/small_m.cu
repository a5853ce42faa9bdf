// small_m.cu -- the fine-grained FP8 linear for few tokens (M <= 128):
// block-scaled GEMM, split-K reduction, bias and bf16 output on the
// activation groups of the prepare step, or for M <= 16 with UE8M0 scales
// with the activation quantization fused in ("Transformers 中的细粒度 FP8 量化
// ... 完全指南", §八 step 6 with the dynamic per-token activation groups of
// §6.1).
//
// With few tokens the layer is bound by reading the weights once (N x K
// e4m3 bytes).  The tile-per-output GEMM would give one 128-token row of
// tiles, N/256 CTAs, most SMs idle.  Here the operands swap roles: the
// weights are the tensor core's M side.  A CTA owns 128 weight rows -- one
// weight block, so one weight scale per K-block -- and a range of K-blocks;
// the MMA is M = 128 weight rows x N = MP tokens (padded to 16, 32, 64 or
// 128) x K = 32, and the K-ranges of a weight tile are spread over several
// CTAs (split-K) so that every SM streams weights.
//
// Roles (192 threads; 320 with fused quantization):
//   warp 0      producer: per K-block, TMA loads of the weight box (128 x 128
//               e4m3, 128-byte swizzle) and of the activation block into one
//               stage of a ring.  Pre-quantized: the e4m3 box (MP x 128,
//               rows past M zero-filled) straight into the MMA's B operand,
//               the UE8M0 scale-factor tiles of x and W every fourth K-block,
//               float x scales into a token-scale ring; the first stages'
//               weight boxes go out before the preceding kernel has finished.
//               Fused: the bf16 block.
//   warp 1      MMA issuer (one thread)
//   warps 2-5   fused only: quantizers, one K-block per warp (four in
//               flight): the staged bf16 block (8 lanes per token, 16
//               channels each), amax by shuffles, the UE8M0 scale and e4m3
//               codes of quant_math.cuh -- the same bits as the stand-alone
//               activation quantization -- written as the MMA's B operand
//               (128-byte swizzle) and its scale-factor chunks
//   last 4 warps epilogue: thread = weight row.  Float: each K-block's
//               partial P lands in its own TMEM buffer (4 of them) and is
//               promoted, acc[m] += P[m] * (sx[m] * sw).  UE8M0: the
//               block-scaled MMA accumulates the whole K-range.  The idle
//               ring then stages the outputs, which leave by bulk copies
//               (plain stores from the epilogue threads run at a fraction of
//               that rate beside a ring this size): with one split, the bf16
//               rows of y = acc + bias; with several, the fp32 partial rows
//               to the workspace, and the last CTA of the weight tile to
//               finish reads all S partial blocks back, sums them in split
//               order, adds the bias and writes y.
//
// Every wait is bounded; on expiry the kernel records FG8_ERR_TIMEOUT in the
// status word, drains its copies and tensor-core ops, frees TMEM and returns.

#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>

#include "fg8_internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace fg8 {
namespace {

constexpr uint32_t kTimeoutStatus = 6u;  // FG8_ERR_TIMEOUT
constexpr uint64_t kDrainNs = 1000000000ull;
constexpr int kQuantWarp0 = 2;

struct SmParams {
  const uint16_t* x;  // bf16 [M, K], row stride ld_x (fused quantization)
  int64_t ld_x;
  // pre-quantized activations (the prepare step's layouts): float x scales
  // K-major [Kb][ld_s]; UE8M0 scale-factor tiles of x (sfa) and W (sfb)
  const float* xs_t;
  int64_t ld_s;
  const uint8_t* sfa;
  const uint8_t* sfb;
  int Kq;
  int M, N, K, Kb, S;
  const float* ws_f;    // float weight scales [Nb][Kb]
  const uint8_t* ws_b;  // UE8M0 weight scales [Nb][Kb]
  const uint16_t* bias;
  uint16_t* y;
  int64_t ld_y;
  float* part;          // split-K partials [Nb][S][M][128]
  uint32_t* counters;   // [Nb], zero at launch; the last CTA of a tile resets its own
  uint32_t* status;
  uint64_t wait_limit_ns;
  int test_stall;
};

template <int FMT_, int MP_, bool PREQ_ = false>
struct SmCfg {
  static constexpr int FMT = FMT_, MP = MP_;
  // PREQ: the activations come quantized (the prepare step's e4m3 codes and
  // scales, TMA-loaded straight into the MMA's B operand); no quantizer warps
  static constexpr bool PREQ = PREQ_;
  // one ring stage: weight box | fused: bf16 activation block | the e4m3
  // codes (the MMA's B operand) | UE8M0: scale-factor chunks of the tokens
  // and the weight rows
  static constexpr int kW = 128 * 128;
  static constexpr int kXb = PREQ ? 0 : MP * 256;
  static constexpr int kX = MP * 128;
  static constexpr int kOffXb = kW, kOffXq = kW + kXb, kOffSf = kOffXq + kX;
  static constexpr int kStage = (kOffSf + (FMT == 1 ? 2 * kSfChunkBytes : 0) + 1023) / 1024 * 1024;
  static constexpr int kScSlots = FMT == 0 ? 8 : 1;
  static constexpr int kStagesFit = (220 * 1024 - kScSlots * MP * 4) / kStage;
  // fused: kQ quantizer warps work on K-blocks i = w (mod kQ); the ring depth
  // is a multiple of kQ (and divides the 8 scale slots' period) so that each
  // ring slot and scale slot is only ever waited on by one quantizer warp
  static constexpr int kQ = kStagesFit >= 8 ? 4 : 2;
  static constexpr int STAGES = PREQ ? (kStagesFit > 10 ? 10 : kStagesFit)
                                     : (kQ == 4 ? 8 : (kStagesFit >= 6 ? 6 : 4));
  static constexpr int kNumAcc = FMT == 0 ? 4 : 1;
  static constexpr int kCols = MP;
  static constexpr int kChunk = MP < 32 ? MP : 32;  // TMEM columns per load
  static constexpr int kEpiWarp0 = PREQ ? 2 : 6;
  static constexpr int kEpiThreads = 128;
  static constexpr int kThreads = kEpiWarp0 * 32 + kEpiThreads;
  static constexpr int kSfCol = 256;  // UE8M0: scale factors in TMEM, two sets of 8 columns
  static constexpr int kOffSc = STAGES * kStage;
  static constexpr int kOffBar = kOffSc + kScSlots * MP * 4;
  static constexpr int kSmemUsed = 1024 + kOffBar + 512;
  // at least 120 KB so that one CTA holds an SM (and its 512 TMEM columns)
  static constexpr int kSmem = kSmemUsed < 120 * 1024 ? 120 * 1024 : kSmemUsed;
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(STAGES >= 4 && (PREQ || (STAGES % kQ == 0 && 8 % kQ == 0)), "ring depth");
  static_assert(MP % 16 == 0 && MP >= 16 && MP <= (PREQ ? 128 : 32), "token padding");
  static_assert(kOffXq % 1024 == 0 && kOffXb == kW, "the swizzled B operand starts on a 1024-byte boundary");
  static_assert(kNumAcc * MP <= (FMT == 0 ? 512 : 256), "TMEM columns");
  // barriers, the TMEM slot and three flags fit the 512 bytes after the scale ring
  static_assert((3 * STAGES + 2 * kNumAcc + 2 * kScSlots + 3) * 8 + 16 <= 512, "barrier area");
  // the idle ring stages the outputs: partials [MP][128] fp32, and for the
  // reduction at least one token of all 64 splits beside [MP][128] bf16 rows
  static_assert(STAGES * kStage >= MP * 512 && STAGES * kStage - MP * 256 >= 64 * 512, "output staging");
  // M = 128 (weight rows), N = MP (tokens), K-major e4m3 operands, f32 accumulate
  static constexpr uint32_t kIdescF8 = (1u << 4) | (uint32_t(MP >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static constexpr uint32_t kIdescMx = (uint32_t(MP >> 3) << 17) | (1u << 23) | (uint32_t(128 >> 4) << 24);
};

__device__ __forceinline__ void sm_raise(volatile int* abort_flag, uint32_t* status) {
  *abort_flag = 1;
  atomicExch(status, kTimeoutStatus);
}

struct SmRing {
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

// W (16 or 32) consecutive TMEM columns of the warp's 32 lanes into registers, waited for.
template <int W>
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 16) {
    tmem_ld_32x32b_x16(taddr, r);
    tmem_wait_ld();
    tmem_reg_fence16(r);
  } else {
    tmem_ld_32x32b_x32(taddr, r);
    tmem_wait_ld();
    tmem_reg_fence(r);
  }
}

template <class C>
__device__ __forceinline__ void sm_producer(const CUtensorMap* tmW, const CUtensorMap* tmX, const SmParams& p,
                                            uint8_t* smem, uint64_t* wfull, uint64_t* sempty, int nt, int kb0, int kb1,
                                            volatile int* abort_flag) {
  SmRing st;
  uint32_t issued = 0, par[C::STAGES];
  for (int kb = kb0; kb < kb1; ++kb) {
    if (!mbar_wait(sempty + st.slot, st.phase ^ 1u, p.wait_limit_ns, abort_flag)) {
      sm_raise(abort_flag, p.status);
      break;
    }
    uint8_t* stage = smem + st.slot * C::kStage;
    mbar_arrive_expect_tx(wfull + st.slot, C::kW + C::kXb);
    tma_load_2d(stage, tmW, wfull + st.slot, kb * 128, nt * 128);
    tma_load_2d(stage + C::kOffXb, tmX, wfull + st.slot, kb * 128, 0);
    par[st.slot] = st.phase;
    issued |= 1u << st.slot;
    st.template advance<C::STAGES>();
  }
  for (int s = 0; s < C::STAGES; ++s)  // every issued copy lands before shared memory goes away
    if ((issued >> s) & 1u) (void)mbar_wait(wfull + s, par[s], kDrainNs, nullptr);
}

// PREQ producer: per K-block the weight box and the e4m3 activation box
// (the prepare step's codes, rows past M zero-filled) on the stage's
// barrier, UE8M0 scale-factor chunks of x and W whenever a group of four
// K-blocks starts, float x scales (MP of the K-major column) into the scale
// ring.  The weight boxes of the first stages go out before the activation
// quantization of the preceding kernel has finished.
template <class C>
__device__ __forceinline__ void sm_producer_pq(const CUtensorMap* tmW, const CUtensorMap* tmX, const SmParams& p,
                                               uint8_t* smem, uint64_t* full, uint64_t* empty, uint64_t* scfull,
                                               uint64_t* scempty, int nt, int kb0, int kb1, volatile int* abort_flag) {
  const int nk = kb1 - kb0;
  const int pre = nk < C::STAGES ? nk : C::STAGES;
  auto sf = [&](int i) { return C::FMT == 1 && (i == 0 || ((kb0 + i) & 3) == 0); };
  auto xpart = [&](int i) {  // the stage's activation-side copies
    const int kb = kb0 + i;
    uint8_t* stage = smem + (i % C::STAGES) * C::kStage;
    uint64_t* bar = full + i % C::STAGES;
    tma_load_2d(stage + C::kOffXq, tmX, bar, kb * 128, 0);
    if (sf(i)) {
      bulk_load(stage + C::kOffSf, p.sfa + static_cast<size_t>(kb >> 2) * kSfChunkBytes, kSfChunkBytes, bar);
      bulk_load(stage + C::kOffSf + kSfChunkBytes, p.sfb + (static_cast<size_t>(nt) * p.Kq + (kb >> 2)) * kSfChunkBytes,
                kSfChunkBytes, bar);
    }
  };
  auto scales = [&](int i) -> bool {  // float: this K-block's x scales into the scale ring
    if (C::FMT != 0) return true;
    const int slot = i % C::kScSlots;
    if (!mbar_wait(scempty + slot, static_cast<uint32_t>((i / C::kScSlots) & 1) ^ 1u, p.wait_limit_ns, abort_flag))
      return false;
    mbar_arrive_expect_tx(scfull + slot, C::MP * 4);
    bulk_load(smem + C::kOffSc + slot * C::MP * 4, p.xs_t + static_cast<int64_t>(kb0 + i) * p.ld_s, C::MP * 4,
              scfull + slot);
    return true;
  };
  bool ok = true;
  int issued = 0;      // K-blocks whose stage copies were issued
  int sc_issued = 0;   // K-blocks whose scale copies were issued
  for (int i = 0; i < pre; ++i) {  // weights first: they do not depend on the preceding kernel
    mbar_arrive_expect_tx(full + i, C::kW + C::kX + (sf(i) ? 2 * kSfChunkBytes : 0));
    tma_load_2d(smem + i * C::kStage, tmW, full + i, (kb0 + i) * 128, nt * 128);
  }
  grid_wait_prerequisites();  // the activations' codes and scales come from the preceding kernel
  for (int i = 0; i < pre; ++i) xpart(i);
  issued = pre;
  for (int i = 0; ok && i < pre; ++i) ok = scales(i), sc_issued += ok ? 1 : 0;
  for (int i = pre; ok && i < nk; ++i) {
    const int slot = i % C::STAGES;
    if (!mbar_wait(empty + slot, static_cast<uint32_t>((i / C::STAGES) & 1) ^ 1u, p.wait_limit_ns, abort_flag)) {
      ok = false;
      break;
    }
    mbar_arrive_expect_tx(full + slot, C::kW + C::kX + (sf(i) ? 2 * kSfChunkBytes : 0));
    tma_load_2d(smem + slot * C::kStage, tmW, full + slot, (kb0 + i) * 128, nt * 128);
    xpart(i);
    issued = i + 1;
    ok = scales(i);
    sc_issued += ok ? 1 : 0;
  }
  if (!ok) sm_raise(abort_flag, p.status);
  // every issued copy lands before shared memory goes away
  for (int i = issued > C::STAGES ? issued - C::STAGES : 0; i < issued; ++i)
    (void)mbar_wait(full + i % C::STAGES, static_cast<uint32_t>((i / C::STAGES) & 1), kDrainNs, nullptr);
  for (int i = sc_issued > C::kScSlots ? sc_issued - C::kScSlots : 0; C::FMT == 0 && i < sc_issued; ++i)
    (void)mbar_wait(scfull + i % C::kScSlots, static_cast<uint32_t>((i / C::kScSlots) & 1), kDrainNs, nullptr);
}

// The quantizer warps: warp w < kQ quantizes K-blocks kb0 + w, kb0 + w + kQ,
// ... (kQ K-blocks in flight at once), 8 lanes per token, 4 tokens per pass.
template <class C>
__device__ __forceinline__ void sm_quantizer(const SmParams& p, uint8_t* smem, uint64_t* wfull, uint64_t* xfull,
                                             uint64_t* scfull, uint64_t* scempty, int nt, int kb0, int kb1,
                                             volatile int* abort_flag) {
  const int qw = (static_cast<int>(threadIdx.x) >> 5) - kQuantWarp0;
  const int lane = static_cast<int>(threadIdx.x) & 31, l = lane & 7, r_in = lane >> 3;
  if (qw >= C::kQ) return;
  for (int i = qw; kb0 + i < kb1; i += C::kQ) {
    const int kb = kb0 + i;
    const int slot = i % C::STAGES;
    const uint32_t phase = static_cast<uint32_t>((i / C::STAGES) & 1);
    // the stage's activation block has landed (and the MMA that last used
    // the stage, hence its B operand, is done: the producer refilled it after)
    if (!mbar_wait_warp(wfull + slot, phase, p.wait_limit_ns, abort_flag)) {
      sm_raise(abort_flag, p.status);
      break;
    }
    uint8_t* stage = smem + slot * C::kStage;
    uint8_t* xs = stage + C::kOffXq;
    const uint8_t* xb = stage + C::kOffXb;
    // float: the K-block's token scales go to the epilogue's scale ring (slot
    // i % 8: with kQ dividing 8, always this warp's), once the epilogue has
    // released the slot's previous K-block
    const int sc_slot = i % C::kScSlots;
    float* scs = reinterpret_cast<float*>(smem + C::kOffSc + sc_slot * C::MP * 4);
    if (C::FMT == 0 && !mbar_wait_warp(scempty + sc_slot, static_cast<uint32_t>((i / C::kScSlots) & 1) ^ 1u,
                                       p.wait_limit_ns, abort_flag)) {
      sm_raise(abort_flag, p.status);
      break;
    }
    constexpr int kPasses = C::MP / 4;
    constexpr int kBatch = kPasses < 4 ? kPasses : 4;
#pragma unroll
    for (int u0 = 0; u0 < kPasses; u0 += kBatch) {
      uint4 v[kBatch][2];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {  // channels 16 l .. 16 l + 15 of the row (zeros past M and K)
        const int row = (u0 + u) * 4 + r_in;
        const uint4* src = reinterpret_cast<const uint4*>(xb + row * 256 + l * 32);
        v[u][0] = src[0];
        v[u][1] = src[1];
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int row = (u0 + u) * 4 + r_in;
        float f[16];
        {
          float f0[8], f1[8];
          qm::unpack_bf16x8(v[u][0], f0);
          qm::unpack_bf16x8(v[u][1], f1);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            f[k] = f0[k];
            f[8 + k] = f1[k];
          }
        }
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(f[k]));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
        const float s = qm::group_scale(amax);
        const uint32_t sb = C::FMT == 1 ? qm::e8m0_ceil_byte(s) : 0u;
        const uint4 q = qm::quantize16<C::FMT>(f, s, sb);
        // row `row`, 16-byte chunk l of the 128-byte row, 128-byte swizzle (8-row atoms)
        *reinterpret_cast<uint4*>(xs + (row >> 3) * 1024 + (row & 7) * 128 + ((l ^ (row & 7)) << 4)) = q;
        if (l == 0) {
          if constexpr (C::FMT == 1)  // tcgen05.cp source: token row r -> word (r % 32) * 16 + (r / 32) * 4, byte 0
            *reinterpret_cast<uint32_t*>(xs + C::kX + (row & 31) * 16 + (row >> 5) * 4) = row < p.M ? sb : 127u;
          else
            scs[row] = s;  // rows past M: a finite scale whose products are never stored
        }
      }
    }
    if constexpr (C::FMT == 1) {
      // every weight row of the tile has the block's scale; token rows past
      // MP get a finite scale the MMA never uses
      const uint32_t wb = p.ws_b[static_cast<int64_t>(nt) * p.Kb + kb];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = k * 32 + lane;
        *reinterpret_cast<uint32_t*>(xs + C::kX + kSfChunkBytes + (r & 31) * 16 + (r >> 5) * 4) = wb;
        if (r >= C::MP) *reinterpret_cast<uint32_t*>(xs + C::kX + (r & 31) * 16 + (r >> 5) * 4) = 127u;
      }
    }
    fence_proxy_async_smem();  // the tensor core reads what these threads wrote
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(xfull + slot);
      if (C::FMT == 0) mbar_arrive(scfull + sc_slot);  // the epilogue reads the scales
    }
  }
}

template <class C>
__device__ __forceinline__ void sm_mma(const SmParams& p, uint8_t* smem, uint32_t tmem, uint64_t* wfull,
                                       uint64_t* xfull, uint64_t* sempty, uint64_t* tfull, uint64_t* tempty,
                                       uint64_t* teardown, uint64_t* stall, int kb0, int kb1,
                                       volatile int* abort_flag) {
  SmRing st, ab;
  // test hook: a barrier nothing arrives on, so the bounded wait runs out
  if (p.test_stall && !mbar_wait(stall, 0, p.wait_limit_ns, abort_flag)) {
    sm_raise(abort_flag, p.status);
    kb1 = kb0;
  }
  int sf_loads = 0;
  for (int kb = kb0; kb < kb1; ++kb) {
    if (!mbar_wait(wfull + st.slot, st.phase, p.wait_limit_ns, abort_flag) ||
        (!C::PREQ && !mbar_wait(xfull + st.slot, st.phase, p.wait_limit_ns, abort_flag))) {
      sm_raise(abort_flag, p.status);
      break;
    }
    tc_fence_after();
    if (C::FMT == 0) {
      if (!mbar_wait(tempty + ab.slot, ab.phase ^ 1u, p.wait_limit_ns, abort_flag)) {
        sm_raise(abort_flag, p.status);
        break;
      }
      tc_fence_after();
    }
    const uint32_t a = smem_u32(smem + st.slot * C::kStage);
    const uint32_t b = a + C::kOffXq;
    // UE8M0: the scale factors into one of two TMEM column sets (alternating,
    // so a copy never lands under an MMA still reading the last one): every
    // K-block (fused: byte 0 of each word) or whenever a group of four
    // K-blocks starts (PREQ: the prepare step's tiles, byte kb % 4)
    const bool load_sf = C::FMT == 1 && (!C::PREQ || kb == kb0 || (kb & 3) == 0);
    if (load_sf) ++sf_loads;
    const uint32_t sf = tmem + static_cast<uint32_t>(C::kSfCol + ((sf_loads - 1) & 1) * 8);
    const uint32_t j = C::PREQ ? static_cast<uint32_t>(kb & 3) : 0u;
    if (load_sf) {
      tc_cp_32x128b_warpx4(sf, smem_desc(b + C::kX, 128, 128, 0));                      // tokens (B)
      tc_cp_32x128b_warpx4(sf + 4, smem_desc(b + C::kX + kSfChunkBytes, 128, 128, 0));  // weight rows (A)
    }
    const uint32_t d = tmem + static_cast<uint32_t>(C::FMT == 0 ? ab.slot * C::MP : 0);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint64_t ad = smem_desc(a + k * 32, 16, 1024, 2);
      const uint64_t bd = smem_desc(b + k * 32, 16, 1024, 2);
      if (C::FMT == 0) mma_f8f6f4(d, ad, bd, C::kIdescF8, k > 0 ? 1u : 0u);
      else
        mma_mxf8f6f4(d, ad, bd, C::kIdescMx | (j << 29) | (j << 4), (sf + 4) | (j << 30), sf | (j << 30),
                     (kb > kb0 || k > 0) ? 1u : 0u);
    }
    tc_commit(sempty + st.slot);  // frees the weight box and the activation block
    if (C::FMT == 0) {
      tc_commit(tfull + ab.slot);
      ab.template advance<C::kNumAcc>();
    }
    st.template advance<C::STAGES>();
  }
  if (C::FMT == 1) tc_commit(tfull);
  tc_commit(teardown);  // all tensor-core ops done before TMEM is released
  (void)mbar_wait(teardown, 0, kDrainNs, nullptr);
}

// bf16 rows staged in shared memory ([j][128], 256 bytes each) to y: one
// bulk store per token row (the tile's valid columns; N % 8 == 0 keeps every
// size and address a multiple of 16 bytes).  Shared memory is read before
// the thread leaves; the stores complete with the grid.
template <class C>
__device__ __forceinline__ void sm_store_rows(const SmParams& p, const uint16_t* ys, int nt, int et,
                                              volatile int* abort_flag) {
  fence_proxy_async_smem();  // this thread's staged values are visible to the bulk copies
  named_barrier_sync(1, C::kEpiThreads);
  if (*abort_flag) return;
  const int ncols = p.N - nt * 128 < 128 ? p.N - nt * 128 : 128;
  bool any = false;
  for (int j = et; j < p.M; j += C::kEpiThreads) {
    bulk_store(p.y + static_cast<int64_t>(j) * p.ld_y + nt * 128, ys + j * 128, static_cast<uint32_t>(ncols) * 2u);
    any = true;
  }
  if (any) {
    bulk_commit_group();
    bulk_wait_group_read<0>();
  }
}

// The last CTA of a weight tile: the S partial blocks of its [S][M][128]
// region come into the (idle) ring in chunks of G tokens, one bulk copy per
// split and one barrier wait per chunk; the sum runs in split order (the same
// whichever CTA finishes last), thread = 4 adjacent columns of one token;
// bias, bf16, then the rows go out as bulk stores.  Every epilogue warp runs
// the same barrier sequence, including after a timed-out wait.
template <class C>
__device__ __forceinline__ void sm_reduce_tile(const SmParams& p, uint8_t* smem, const float* tp, int nt, int et,
                                               uint64_t* rbar, volatile int* go_flag, volatile int* abort_flag) {
  constexpr int kRing = C::STAGES * C::kStage;
  uint16_t* ys = reinterpret_cast<uint16_t*>(smem + kRing - C::MP * 256);  // [MP][128] bf16
  const int S = p.S, M = p.M;
  const int G = (kRing - C::MP * 256) / 512 / S < M ? (kRing - C::MP * 256) / 512 / S : M;
  const int ew = et >> 5, c = (et & 31) * 4;
  const int n0 = nt * 128 + c;
  float4 b = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (p.bias != nullptr && n0 < p.N) {  // N % 8 == 0: a column quad is wholly inside or outside
    const uint2 bb = *reinterpret_cast<const uint2*>(p.bias + n0);
    b = make_float4(__uint_as_float(bb.x << 16), __uint_as_float(bb.x & 0xFFFF0000u), __uint_as_float(bb.y << 16),
                    __uint_as_float(bb.y & 0xFFFF0000u));
  }
  fence_proxy_async_global();  // the partials, written by bulk copies, are read by bulk copies
  uint32_t phase = 0;
  bool pending = false;  // loads issued whose arrival nobody saw
  for (int j0 = 0; j0 < M; j0 += G) {
    const int g = M - j0 < G ? M - j0 : G;
    named_barrier_sync(1, C::kEpiThreads);  // the chunk buffer is free
    if (et == 0) {
      const int go = !*abort_flag;
      *go_flag = go;
      if (go) {
        mbar_arrive_expect_tx(rbar, static_cast<uint32_t>(S * g * 512));
        for (int s = 0; s < S; ++s)
          bulk_load(smem + s * g * 512, tp + (static_cast<int64_t>(s) * M + j0) * 128, static_cast<uint32_t>(g) * 512u,
                    rbar);
        pending = true;
      }
    }
    named_barrier_sync(1, C::kEpiThreads);
    if (!*go_flag) break;  // read by every warp after the same barrier: a uniform exit
    if (!mbar_wait_warp(rbar, phase, p.wait_limit_ns, abort_flag)) {
      sm_raise(abort_flag, p.status);
    } else {
      if (et == 0) pending = false;
      for (int jj = ew; jj < g; jj += 4) {
        float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        for (int s = 0; s < S; ++s) {
          const float4 l = *reinterpret_cast<const float4*>(smem + (s * g + jj) * 512 + c * 4);
          v.x += l.x;
          v.y += l.y;
          v.z += l.z;
          v.w += l.w;
        }
        const uint32_t lo = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.x + b.x))) |
                            (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y + b.y))) << 16);
        const uint32_t hi = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.z + b.z))) |
                            (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.w + b.w))) << 16);
        *reinterpret_cast<uint2*>(ys + (j0 + jj) * 128 + c) = make_uint2(lo, hi);
      }
    }
    phase ^= 1u;
  }
  // copies still in flight land before the ring is reused or released
  if (et == 0 && pending) (void)mbar_wait(rbar, phase ^ 1u, kDrainNs, nullptr);
  sm_store_rows<C>(p, ys, nt, et, abort_flag);
}

template <class C>
__device__ __forceinline__ void sm_epilogue(const SmParams& p, uint8_t* smem, uint32_t tmem, uint64_t* tfull,
                                            uint64_t* tempty, uint64_t* scfull, uint64_t* scempty, uint64_t* rbar,
                                            int nt, int sp, int kb0, int kb1, volatile int* abort_flag,
                                            volatile int* last_flag, volatile int* go_flag) {
  const int warp = static_cast<int>(threadIdx.x) >> 5, lane = static_cast<int>(threadIdx.x) & 31;
  const int q = warp & 3;  // TMEM lane quadrant
  const int t = q * 32 + lane;
  const int n = nt * 128 + t;
  const int m0 = 0;  // first token of this thread's columns
  const int et = static_cast<int>(threadIdx.x) - C::kEpiWarp0 * 32;
  const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
  float acc[C::kCols];
#pragma unroll
  for (int j = 0; j < C::kCols; ++j) acc[j] = 0.0f;
  bool ok = true;
  if constexpr (C::FMT == 0) {
    SmRing ab, sc;
    // the ring holds sx; the weight block's sw comes from global memory
    const float* wsr = p.ws_f + static_cast<int64_t>(nt) * p.Kb;
    float sw_next = wsr[kb0];
    for (int kb = kb0; kb < kb1; ++kb) {
      const float sw = sw_next;
      if (kb + 1 < kb1) sw_next = wsr[kb + 1];
      if (!mbar_wait_warp(scfull + sc.slot, sc.phase, p.wait_limit_ns, abort_flag) ||
          !mbar_wait_warp(tfull + ab.slot, ab.phase, p.wait_limit_ns, abort_flag)) {
        sm_raise(abort_flag, p.status);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + lane_base + static_cast<uint32_t>(ab.slot * C::MP + m0);
      const float* scs = reinterpret_cast<const float*>(smem + C::kOffSc + sc.slot * C::MP * 4) + m0;
#pragma unroll
      for (int c = 0; c < C::kCols / C::kChunk; ++c) {
        uint32_t r[C::kChunk];
        tmem_ld_chunk<C::kChunk>(taddr + c * C::kChunk, r);
        if (c + 1 == C::kCols / C::kChunk) {  // the K-block's columns are all read: hand the buffer back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty + ab.slot);
        }
#pragma unroll
        for (int j = 0; j < C::kChunk; ++j)
          acc[c * C::kChunk + j] = __fmaf_rn(__uint_as_float(r[j]), scs[c * C::kChunk + j] * sw, acc[c * C::kChunk + j]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(scempty + sc.slot);
      ab.template advance<C::kNumAcc>();
      sc.template advance<C::kScSlots>();
    }
  } else {
    if (!mbar_wait_warp(tfull, 0, p.wait_limit_ns, abort_flag)) {
      sm_raise(abort_flag, p.status);
      ok = false;
    } else {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < C::kCols / C::kChunk; ++c) {
        uint32_t r[C::kChunk];
        tmem_ld_chunk<C::kChunk>(tmem + lane_base + static_cast<uint32_t>(m0 + c * C::kChunk), r);
#pragma unroll
        for (int j = 0; j < C::kChunk; ++j) acc[c * C::kChunk + j] = __uint_as_float(r[j]);
      }
    }
  }
  tc_fence_before();
  // Every epilogue warp takes the same path from here on (the named barriers
  // below count all of them): a warp that timed out joins them, writing
  // nothing.  The ring is idle now -- every copy into it was consumed by an
  // MMA that has completed -- and stages the outputs.
  if (p.S == 1) {
    uint16_t* ys = reinterpret_cast<uint16_t*>(smem);  // [MP][128] bf16
    const float bias_n = (p.bias != nullptr && n < p.N) ? __uint_as_float(static_cast<uint32_t>(p.bias[n]) << 16) : 0.0f;
    if (ok) {
#pragma unroll
      for (int j = 0; j < C::kCols; ++j)
        if (m0 + j < p.M) ys[(m0 + j) * 128 + t] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j] + bias_n));
    }
    sm_store_rows<C>(p, ys, nt, et, abort_flag);
    return;
  }
  // this tile's partials, [S][M][128] (columns past N are written, never read back)
  float* tp = p.part + static_cast<int64_t>(nt) * p.S * p.M * 128;
  float* pa = reinterpret_cast<float*>(smem);  // [M][128]
  if (ok) {
#pragma unroll
    for (int j = 0; j < C::kCols; ++j)
      if (m0 + j < p.M) pa[(m0 + j) * 128 + t] = acc[j];
  }
  fence_proxy_async_smem();
  named_barrier_sync(1, C::kEpiThreads);
  if (!*abort_flag && et < p.M) {  // one bulk store per token row, completed before the arrival is counted
    bulk_store(tp + (static_cast<int64_t>(sp) * p.M + et) * 128, pa + et * 128, 512u);
    bulk_commit_group();
    bulk_wait_group<0>();
    fence_proxy_async_global();
  }
  __threadfence();
  named_barrier_sync(1, C::kEpiThreads);
  if (et == 0) {
    const uint32_t done = ok && !*abort_flag ? atomicAdd(p.counters + nt, 1u) + 1u : 0u;
    *last_flag = done == static_cast<uint32_t>(p.S) ? 1 : 0;
    // every CTA of the tile has arrived: zero the counter for the next call
    if (done == static_cast<uint32_t>(p.S)) p.counters[nt] = 0u;
  }
  named_barrier_sync(1, C::kEpiThreads);
  if (*last_flag) {
    __threadfence();
    sm_reduce_tile<C>(p, smem, tp, nt, et, rbar, go_flag, abort_flag);
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    fg8_small_m_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const SmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* xfull = wfull + C::STAGES;
  uint64_t* sempty = xfull + C::STAGES;
  uint64_t* tfull = sempty + C::STAGES;
  uint64_t* tempty = tfull + C::kNumAcc;
  uint64_t* scfull = tempty + C::kNumAcc;
  uint64_t* scempty = scfull + C::kScSlots;
  uint64_t* teardown = scempty + C::kScSlots;
  uint64_t* stall = teardown + 1;
  uint64_t* rbar = stall + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* go_flag = reinterpret_cast<volatile int*>(tmem_slot + 3);

  const int warp = static_cast<int>(threadIdx.x) >> 5, lane = static_cast<int>(threadIdx.x) & 31;
  const int nt = static_cast<int>(blockIdx.x) / p.S, sp = static_cast<int>(blockIdx.x) % p.S;
  const int kb0 = static_cast<int>(static_cast<int64_t>(sp) * p.Kb / p.S);
  const int kb1 = static_cast<int>(static_cast<int64_t>(sp + 1) * p.Kb / p.S);
  if (threadIdx.x == 0) {
    // the descriptors' fetch overlaps the barrier set-up before the first copy
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(wfull + s, 1);
      mbar_init(xfull + s, 1);
      mbar_init(sempty + s, 1);
    }
    for (int a = 0; a < C::kNumAcc; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, C::kEpiThreads / 32);
    }
    for (int s = 0; s < C::kScSlots; ++s) {
      mbar_init(scfull + s, 1);
      mbar_init(scempty + s, C::kEpiThreads / 32);
    }
    mbar_init(teardown, 1);
    mbar_init(stall, 1);
    mbar_init(rbar, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // fused: x may come from the preceding kernel; PREQ: only the producer
  // reads that kernel's output, and it waits itself after its first weights
  if constexpr (!C::PREQ) grid_wait_prerequisites();
  grid_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      if constexpr (C::PREQ) sm_producer_pq<C>(&tmW, &tmX, p, smem, wfull, sempty, scfull, scempty, nt, kb0, kb1,
                                               abort_flag);
      else sm_producer<C>(&tmW, &tmX, p, smem, wfull, sempty, nt, kb0, kb1, abort_flag);
    }
  } else if (warp == 1) {
    if (lane == 0)
      sm_mma<C>(p, smem, tmem, wfull, xfull, sempty, tfull, tempty, teardown, stall, kb0, kb1, abort_flag);
  } else if (warp < C::kEpiWarp0) {
    if constexpr (!C::PREQ) sm_quantizer<C>(p, smem, wfull, xfull, scfull, scempty, nt, kb0, kb1, abort_flag);
  } else {
    sm_epilogue<C>(p, smem, tmem, tfull, tempty, scfull, scempty, rbar, nt, sp, kb0, kb1, abort_flag, last_flag,
                   go_flag);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

typedef CUresult (*EncodeTiledFnSm)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnSm encode_fn_sm() {
  // looked up once per process (thread-safe static initialisation)
  static const EncodeTiledFnSm fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFnSm>(ptr);
    return static_cast<EncodeTiledFnSm>(nullptr);
  }();
  return fn;
}

template <class C>
cudaError_t launch_small_m_cfg(const SmallMArgs& a, cudaStream_t s) {
  EncodeTiledFnSm fn = encode_fn_sm();
  if (fn == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tmW, tmX;
  const cuuint32_t estr[2] = {1, 1};
  {  // weights e4m3 [N, K]: 128 x 128 boxes, 128-byte swizzle
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K)};
    const cuuint32_t box[2] = {128, 128};
    if (fn(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.wq), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if constexpr (C::PREQ) {  // quantized activations e4m3 [M, K] (row stride K): MP x 128 boxes, 128-byte swizzle
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K)};
    const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(C::MP)};
    if (fn(&tmX, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.xq), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {  // activations bf16 [M, K] (row stride ld_x): MP x 128 boxes, rows past M zero-filled
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.ld_x) * 2};
    const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(C::MP)};
    if (fn(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.x), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  SmParams p;
  p.x = static_cast<const uint16_t*>(a.x);
  p.ld_x = a.ld_x;
  p.xs_t = a.xs_t;
  p.ld_s = a.ld_s;
  p.sfa = a.sfa;
  p.sfb = a.sfb;
  p.Kq = a.Kq;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.Kb = (a.K + 127) / 128;
  p.S = a.splits;
  p.ws_f = static_cast<const float*>(a.w_scale);
  p.ws_b = static_cast<const uint8_t*>(a.w_scale);
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.y = static_cast<uint16_t*>(a.y);
  p.ld_y = a.ld_y;
  p.part = a.part;
  p.counters = a.counters;
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  p.test_stall = a.test_stall;
  const int nt = (a.N + 127) / 128;
  auto kern = fg8_small_m_kernel<C>;
  // the shared-memory opt-in, once per device (one bit per device; calls from
  // several host threads may repeat it, which is harmless)
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if ((configured.load(std::memory_order_acquire) & bit) == 0) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_release);
  }
  if (a.splits > 1 && a.zero_counters) {  // arrival counters outside the header start at zero
    const cudaError_t e = cudaMemsetAsync(a.counters, 0, static_cast<size_t>(nt) * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(nt * a.splits));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmW, tmX, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int small_m_splits(int M, int N, int K) {
  // One wave of work units (weight tile, K-range): as many K-splits as fit
  // next to the other tiles on the 148 SMs (about 100 streaming SMs already
  // reach the HBM bandwidth; a second wave would only add its ramp), and at
  // most 512 / M, which bounds what the last CTA of a tile reads back
  // (S x M x 512 bytes).  Depends on the shape only, so the workspace size
  // never depends on the device.
  constexpr int kSms = 148;
  const int nt = (N + 127) / 128, kb = (K + 127) / 128;
  int s = kSms / nt;
  if (s > kb) s = kb;
  if (s > 64) s = 64;
  if (M > 0 && s > 512 / M) s = 512 / M;
  return s < 1 ? 1 : s;
}

size_t small_m_partial_bytes(int64_t M, int64_t N, int64_t K) {
  const int s = small_m_splits(static_cast<int>(M), static_cast<int>(N), static_cast<int>(K));
  return s > 1 ? static_cast<size_t>(s) * M * ((N + 127) / 128) * 128 * 4 : 0;
}

cudaError_t launch_small_m(const SmallMArgs& a, int fmt, cudaStream_t s) {
  if (a.preq) {
    if (a.M < 1 || a.M > kSmallMMax) return cudaErrorInvalidValue;
    const int mp = a.M <= 16 ? 16 : a.M <= 32 ? 32 : a.M <= 64 ? 64 : 128;
    if (fmt == 0) {
      if (mp == 16) return launch_small_m_cfg<SmCfg<0, 16, true>>(a, s);
      if (mp == 32) return launch_small_m_cfg<SmCfg<0, 32, true>>(a, s);
      if (mp == 64) return launch_small_m_cfg<SmCfg<0, 64, true>>(a, s);
      return launch_small_m_cfg<SmCfg<0, 128, true>>(a, s);
    }
    if (mp == 16) return launch_small_m_cfg<SmCfg<1, 16, true>>(a, s);
    if (mp == 32) return launch_small_m_cfg<SmCfg<1, 32, true>>(a, s);
    if (mp == 64) return launch_small_m_cfg<SmCfg<1, 64, true>>(a, s);
    return launch_small_m_cfg<SmCfg<1, 128, true>>(a, s);
  }
  // fused quantization: M <= 16 (one token padding)
  if (a.M < 1 || a.M > kFusedMMax) return cudaErrorInvalidValue;
  if (fmt == 0) return launch_small_m_cfg<SmCfg<0, 16>>(a, s);
  return launch_small_m_cfg<SmCfg<1, 16>>(a, s);
}

}  // namespace fg8
