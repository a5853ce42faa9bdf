// fg8_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace fg8 {

constexpr int kGroup = 128;      // activation group width = weight block width
constexpr int kBlockM = 128;     // GEMM tile rows (tokens)
constexpr int kSfChunkBytes = 512;  // one scale-factor tile: 128 rows x 4 K-blocks, UE8M0

enum ScaleLayout : int {
  kScaleRowMajor = 0,   // [M, Kb] row-major (the public layout)
  kScaleKMajor = 1,     // float32 [Kb, ld] (column m contiguous): what the float GEMM epilogue reads
  kScaleSfTiles = 2,    // UE8M0 tensor-core scale-factor tiles (see sf_tile_offset)
};

// Byte offset of the UE8M0 scale of (row r, K-block kb) inside the tensor-core
// scale-factor tile stream: tiles of 128 rows x 4 K-blocks, 512 bytes each,
// tile (r/128, kb/4) at ((r/128)*Kq + kb/4)*512, inside a tile the word for
// row 32c + i (i < 32) is at i*16 + c*4 and K-block kb%4 is byte kb%4 of it.
// That is the shared-memory source shape of tcgen05.cp.32x128b.warpx4, which
// lands row 32c + i in TMEM lane i (of every sub-partition), column c.
__host__ __device__ inline size_t sf_tile_offset(int64_t r, int kb, int Kq) {
  const int64_t tile = r / 128, rr = r % 128;
  return static_cast<size_t>((tile * Kq + kb / 4) * kSfChunkBytes + (rr % 32) * 16 + (rr / 32) * 4 + (kb % 4));
}

struct ActQuantArgs {
  const void* x;      // bf16 [M, K], row stride ld_x
  int64_t ld_x;
  int M, K, Kb;       // Kb: groups per row, ceil(K / group)
  int group;          // group width: 128 (0 means 128), 64 or 32
  uint8_t* xq;        // e4m3 [M, K], row stride K
  void* xs;           // scales, layout below
  int layout;         // ScaleLayout
  int64_t ld_s;       // kScaleKMajor: column stride (>= M)
  int Kq;             // kScaleSfTiles: ceil(Kb / 4) chunks of four groups per row tile
  int M_pad;          // kScaleSfTiles: rows rounded up to 128 (padding rows get scale 2^0)
  // static activation scheme (float scales only): one precomputed scale for
  // the whole tensor, read from device memory; nullptr = dynamic groups
  const float* static_scale;
};

cudaError_t launch_act_quant(const ActQuantArgs& a, int fmt, int num_sms, cudaStream_t s);

cudaError_t launch_weight_quant(const void* w, int64_t ld_w, int N, int K, uint8_t* wq, void* ws, int fmt,
                                cudaStream_t s);
// block x block weight blocks, block 32 or 64 (weight_block_size = (block,
// block)): scales [ceil(N/block), ceil(K/block)].
cudaError_t launch_weight_quant_small(const void* w, int64_t ld_w, int N, int K, int block, uint8_t* wq, void* ws,
                                      int fmt, cudaStream_t s);

// Pack a UE8M0 [R_src, Kb] row-major scale matrix into scale-factor tiles for
// R rows, written for R_pad rows (a multiple of 128): row r, slot j takes
// src[(r / row_div) * Kb + j / kdiv]; padding rows and slots get byte 127 (2^0).
cudaError_t launch_sf_pack(const uint8_t* src, int R, int64_t R_pad, int row_div, int Kb, int kdiv, uint8_t* dst,
                           cudaStream_t s);

// Rows of weight scale-factor tiles: N rounded up to the widest GEMM tile.
__host__ __device__ inline int64_t sfb_rows(int64_t N) { return (N + 255) / 256 * 256; }

struct GemmArgs {
  const void* xq;     // e4m3 [M, K] row stride K
  const void* wq;     // e4m3 [N, K] row stride K
  void* y;            // bf16 [M, N] row stride ld_y
  int64_t ld_y;
  int M, N, K, Kb;
  // float path: x scales K-major [Kb][ld_s] (ld_s a multiple of 256, >= M),
  // weight scales as given, [ceil(N/128)][Kb] row-major
  const float* xs_t;
  int64_t ld_s;
  const float* w_scale;
  // UE8M0 path: scale-factor tiles of x (rows M) and W (rows N)
  const uint8_t* sfa;
  const uint8_t* sfb;
  int Kq;
  const void* bias;   // bf16 [N] or nullptr
  uint32_t* status;   // device status word (0 = ok)
  uint64_t wait_limit_ns;
  int test_stall;     // test hook: the MMA thread first waits on a barrier nothing completes
  // Optional: also quantize this layer's bf16 output as the activation of a
  // next layer (K_next = N, N_next outputs) straight into that layer's
  // workspace, exactly as its prepare step would.
  uint8_t* nx_xq;         // e4m3 [M, N] row stride N; nullptr = off
  void* nx_xs;            // float: K-major [N/128][nx_ld_s]; UE8M0: scale-factor tiles
  int64_t nx_ld_s;
  int nx_Kq;              // UE8M0: ceil(ceil(N/128) / 4)
  const void* nx_w_scale; // next layer's weight scales [ceil(N_next/128), ceil(N/128)]
  void* nx_w_prep;        // UE8M0: ... packed into scale-factor tiles (unused for float)
  int nx_N;               // N_next
  // Optional: grouped (MoE experts) -- the expert of each row [M] (a tile
  // computes with its first row's expert; -1 skips it); wq [E][N][K],
  // w_scale [E][Nb][Kb], bias [E][N]; sfb holds sfb_tiles 128-row
  // scale-factor tiles per expert.  nullptr: one weight matrix.
  const int32_t* row_expert;
  int E;
  int sfb_tiles;
  // UE8M0 with 1 x 32 / 1 x 64 activation groups and 32 x 32 / 64 x 64
  // weight blocks: the scale-factor tiles hold one scale per 32 K per row,
  // one chunk per K-block (Kq = ceil(K/128) chunks per row tile)
  bool sf32;
  // float scales: the block size b (0 means 128; 32 or 64): 1 x b x-scale
  // groups, K-major [ceil(K/b)][ld_s], and b x b weight blocks
  // [ceil(N/b)][ceil(K/b)]; the GEMM promotes every b-wide slice of K
  int wblk;
  // Optional: quantize x inside the GEMM kernel (1 x 128 groups) instead of
  // reading a prepare step's output.  Before their tiles, all CTAs
  // quantize 128-row x 128-channel units of bf16 x (unit rb * Kb + kb on CTA
  // unit % grid) into xq and the x scales (sfa / xs_t, the prepare step's
  // layouts), and mark each unit done in qflags[unit] with the call's epoch
  // + 1; the roles that read a unit wait for its flag.  The last CTA to
  // finish advances the epoch in the workspace header.
  const void* qx;         // bf16 [M, K], row stride ld_qx; nullptr = off
  int64_t ld_qx;
  uint32_t* qflags;       // [ceil(M/128) * Kb]
  uint32_t* qepoch;       // the header's words: epoch, finished-CTA count, weight-packing CTA count
  const void* qwsc;       // UE8M0: this layer's weight scales [Nb][Kb], packed into sfb by phase one
  // Optional: room for the split-K tail (split_plan below): the fp32 partial
  // sums of the split tiles.  Used when split_bytes covers the plan's
  // split_area_bytes; its arrival counters are the header's split-K counters
  // (one per split tile, zero at rest).
  uint8_t* split_ws;
  size_t split_bytes;
};

// Split-K tail of the tiled GEMM.  With T tiles on `sms` persistent CTAs the
// last wave holds T mod sms tiles and leaves the other SMs idle for a whole
// tile's K loop.  The plan splits each of those tiles into S work units of
// kbs consecutive K-blocks (one wave of at most `sms` units); each unit
// writes its fp32 partial sum, and the tile's last unit to finish adds the S
// partials in split order (so the result does not depend on which unit
// finishes last) and stores the tile.  from == tiles: no split.
struct SplitPlan {
  int from = 0;  // first split tile (tiles before it run whole)
  int s = 1;     // units per split tile
  int kbs = 0;   // K-blocks per unit (the last unit may have fewer)
};
SplitPlan split_plan(int tiles, int m_blocks, int Kb, int kb_align, int sms);
// Bytes of fp32 partials a plan needs with bn-wide tiles.
size_t split_area_bytes(const SplitPlan& pl, int tiles, int bn);
// The split-K area a tiled GEMM of this shape may use on a device with `sms`
// SMs (the larger of the 128- and 256-wide tiles' plans).
size_t gemm_split_area(int64_t M, int64_t N, int64_t K, int fmt, int sms);

// Rows of the K-major float x-scale matrix: M rounded up to the tallest GEMM
// tile (256 rows for a CTA pair), so every tile's 128-row slices are in range.
__host__ __device__ inline int64_t kmajor_ld(int64_t M) { return (M + 255) / 256 * 256; }

// Float x scales row-major [M, Kb] -> K-major [Kb][ld_s].
cudaError_t launch_xs_transpose(const float* xs, int M, int Kb, int64_t ld_s, float* out, cudaStream_t s);

// Workspace header: the sticky device status word at byte 0 and, from byte
// kHeaderCounterOffset, split-K arrival counters: the few-token path's (one
// per 128-row weight tile) or the tiled GEMM's split tail (one per split
// tile); zero at rest, the last CTA of a tile resets its counter.  Zeroed by
// the caller before first use.
constexpr size_t kWorkspaceHeaderBytes = 1024;
constexpr size_t kHeaderEpochOffset = 8;  // fused act-quant: epoch word, then the finished-CTA count
constexpr size_t kHeaderCounterOffset = 64;
constexpr int kHeaderCounters = static_cast<int>((kWorkspaceHeaderBytes - kHeaderCounterOffset) / 4);

// Few tokens: a swap-AB split-K GEMM that streams the weights as the tensor
// core's M side (small_m.cu), either on the prepare step's quantized
// activations (preq) or, with UE8M0 scales and M <= kFusedMMax, with the
// activation quantization fused into it.  fg8_linear takes it for
// M <= kSmallMAlways, and up to kSmallMMax tokens while the tiled GEMM's grid
// (ceil(N / 256) tiles of 128 tokens) would cover at most a quarter of the
// 148 SMs; both rules depend on the shape only.
constexpr int kSmallMMax = 128;
constexpr int kSmallMAlways = 32;
constexpr int kFusedMMax = 16;

inline bool use_small_m(int64_t M, int64_t N) {
  return M >= 1 && (M <= kSmallMAlways || (M <= kSmallMMax && (N + 255) / 256 * 4 <= 148));
}
inline bool use_fused_small_m(int64_t M, int fmt) { return fmt == 1 && M <= kFusedMMax; }

struct SmallMArgs {
  const void* x;          // bf16 [M, K], row stride ld_x (fused)
  int64_t ld_x;
  bool preq;              // activations already quantized (the prepare step's layouts below)
  const void* xq;         // e4m3 [M, K], row stride K
  const float* xs_t;      // float: x scales K-major [Kb][ld_s]
  int64_t ld_s;
  const uint8_t* sfa;     // UE8M0: scale-factor tiles of x, and of W (sfb)
  const uint8_t* sfb;
  int Kq;
  int M, N, K;
  const void* wq;         // e4m3 [N, K]
  const void* w_scale;    // [ceil(N/128), ceil(K/128)] float32 or UE8M0 bytes
  const void* bias;       // bf16 [N] or nullptr
  void* y;                // bf16 [M, N], row stride ld_y
  int64_t ld_y;
  int splits;             // small_m_splits(M, N, K)
  uint32_t* counters;     // [ceil(N/128)], zero at rest (or zeroed by the launch, below)
  bool zero_counters;     // counters outside the header: clear them before the kernel
  float* part;            // [ceil(N/128)][splits][M][128] fp32 when splits > 1
  uint32_t* status;
  uint64_t wait_limit_ns;
  int test_stall;         // test hook, as GemmArgs::test_stall
};

int small_m_splits(int M, int N, int K);
// Bytes of fp32 split-K partials the small-M path needs (0 with one split).
size_t small_m_partial_bytes(int64_t M, int64_t N, int64_t K);
cudaError_t launch_small_m(const SmallMArgs& a, int fmt, cudaStream_t s);

// Checkpoint conversions (convert.cu).
cudaError_t launch_dequant_weight(const uint8_t* wq, int N, int K, const void* ws, int fmt, uint16_t* w, int64_t ld_w,
                                  int num_sms, cudaStream_t s);
// Batched expert layout (E slabs of cap rows, counts[e] routed) -> row_expert.
cudaError_t launch_row_expert(const int32_t* counts, int E, int cap, int32_t* row_expert, int num_sms,
                              cudaStream_t st);
cudaError_t launch_scale_to_e8m0(const float* s, int64_t n, uint8_t* out, uint32_t* bad, int num_sms, cudaStream_t st);

int choose_block_n(int M, int N, int Kb, int kb_align, int num_sms, bool split);

// fg8_linear's host-side argument checks, workspace excepted (api.cu); an
// fg8_status value.  Entry points built on fg8_linear run them before their
// own set-up so that a bad call touches no device state.
int check_linear_args_status(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x, const void* wq_e4m3,
                             const void* w_scale_inv, const void* bias_bf16, const void* y_bf16, int64_t ld_y,
                             int fmt);

cudaError_t launch_gemm(const GemmArgs& g, int fmt, int num_sms, cudaStream_t s);

}  // namespace fg8
