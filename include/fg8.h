/*
 * fg8.h -- C ABI of the B200 (sm_100a) fine-grained FP8 linear layer.
 *
 * The method is the one the Transformers fine-grained FP8 pages describe:
 *   [zh] "Transformers 中的细粒度 FP8 量化：配置、DeepGEMM 加速路径与 UE8M0 缩放格式完全指南"
 *   [pt] "FP8 de granularidade fina" (Transformers documentation)
 * Weights are e4m3fn with one scale per 128x128 block ([zh] §一, [pt]);
 * activations are quantized dynamically per token in groups of 128 input
 * channels aligned with the weight blocks ([zh] §一); scales are float32 or
 * UE8M0 powers of two ([zh] §四 scale_fmt, §七); the layer computes
 *   y = dequant(xq) . dequant(Wq)^T + bias   (bf16 out; bias not quantized, [zh] §三).
 *
 * Arithmetic (the pages print none; the readings used):
 *   scale s = max(amax / 448, 2^-126), a float32 division, amax over the real
 *   elements of the group/block; UE8M0 stores s rounded up to a power of two
 *   ([zh] §七 补充: float scales are rounded *up* to UE8M0); every element is
 *   q = e4m3(x / s) with the quotient a correctly rounded float32 and the cast
 *   round-to-nearest-even, saturating at +-448, sign kept.
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers on the current CUDA device; the
 *     caller allocates and owns them.  The library allocates no device memory.
 *   - `stream` is a cudaStream_t (passed as void*); work is enqueued on it and
 *     the call returns without synchronizing (except fg8_check_device_status).
 *   - bf16 / e4m3 / UE8M0 buffers are raw bytes (uint16 / uint8 per element).
 *   - Matrices are row-major.  ld_* are row strides in ELEMENTS.
 *   - Host-detectable problems return an error before anything is launched:
 *       FG8_ERR_INVALID_ARG        bad format, non-positive size (M may be 0),
 *                                  NULL required pointer, ld < row length,
 *                                  size beyond 2^31-1
 *       FG8_ERR_ALIGNMENT          K % 16 != 0, N % 8 != 0, ld % 8 != 0 for
 *                                  bf16 operands, or a pointer not 16-byte aligned
 *       FG8_ERR_UNSUPPORTED_DEVICE current device is not compute capability 10.0
 *       FG8_ERR_WORKSPACE          workspace NULL, misaligned (256 B) or too small
 *     A failed launch returns FG8_ERR_CUDA.  There is no fallback path.
 *   - Inputs must be finite; NaN/Inf inputs give unspecified outputs.
 */
#ifndef FG8_H_
#define FG8_H_

#include <stddef.h>
#include <stdint.h>

/* Symbols of the C ABI are the only ones the shared library exports. */
#if defined(__GNUC__)
#define FG8_API __attribute__((visibility("default")))
#else
#define FG8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* [zh] §四: scale_fmt is "float" or "ue8m0". One format per call governs both
 * the activation and the weight scales. */
typedef enum fg8_scale_fmt {
  FG8_SCALE_FLOAT = 0, /* float32 scales */
  FG8_SCALE_UE8M0 = 1  /* one byte: biased exponent b, scale = 2^(b-127) */
} fg8_scale_fmt;

typedef enum fg8_status {
  FG8_OK = 0,
  FG8_ERR_INVALID_ARG = 1,
  FG8_ERR_ALIGNMENT = 2,
  FG8_ERR_UNSUPPORTED_DEVICE = 3,
  FG8_ERR_WORKSPACE = 4,
  FG8_ERR_CUDA = 5,
  FG8_ERR_TIMEOUT = 6 /* a device-side bounded wait expired (see fg8_check_device_status) */
} fg8_status;

/* Quantize a weight once, on load ([zh] §八 step 4, Fp8Quantize; [zh] §一).
 *   w_bf16      [N, K] bf16, row stride ld_w elements (nn.Linear [out, in])
 *   wq_e4m3     [N, K] e4m3fn bytes, row stride K (output)
 *   w_scale_inv [ceil(N/128), ceil(K/128)] row-major (output): float32 for
 *               FG8_SCALE_FLOAT, UE8M0 bytes for FG8_SCALE_UE8M0.
 * W ~= value(wq) * scale_inv per 128x128 block; edge blocks use their real
 * elements only.  One CTA per block on a 2-D grid, so N <= 65535 * 128
 * rows (8,388,480): a larger N returns FG8_ERR_INVALID_ARG before any
 * launch; quantize such a matrix in row slices that start at multiples of
 * 128 rows and are at most that high. */
FG8_API fg8_status fg8_quantize_weight(const void* w_bf16, int64_t N, int64_t K, int64_t ld_w,
                               void* wq_e4m3, void* w_scale_inv, fg8_scale_fmt fmt, void* stream);

/* Dynamic per-token activation quantization ([zh] §一 "激活按每个 token 一组";
 * [pt] first list): each row is cut into groups of 128 channels (the last
 * group holds K mod 128 real channels), one scale per group.
 *   x_bf16  [M, K] bf16, row stride ld_x elements
 *   xq_e4m3 [M, K] e4m3fn bytes, row stride K (output)
 *   x_scale [M, ceil(K/128)] row-major (output): float32 or UE8M0 bytes. */
FG8_API fg8_status fg8_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x,
                            void* xq_e4m3, void* x_scale, fg8_scale_fmt fmt, void* stream);

/* Bytes of caller-owned device workspace fg8_linear needs for this shape
 * (quantized activations, their scales in the GEMM's layout, the scale-factor
 * tiles of the UE8M0 path, a device status word, and the fp32 partial sums of
 * the few-token kernel's split K or of the tiled GEMM's split-K tail, see
 * fg8_linear_plan).  The tail is planned for the current device's SM count
 * (148 when no device is visible); a workspace sized on a device with another
 * count is still accepted, the tail then runs unsplit.  0 on bad arguments. */
FG8_API size_t fg8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt);

/* How fg8_linear runs this shape on the current device (148 SMs when none
 * is visible), for callers that size launches or read profiles:
 *   plan[0]  kernel: 0 the tiled GEMM, 1 the few-token split-K kernel on the
 *            prepare step's activations, 2 the few-token kernel that also
 *            quantizes x (no prepare launch)
 *   plan[1]  tiled GEMM: tile width (128 or 256 output columns; 128 rows)
 *   plan[2]  tiled GEMM: tiles of the last wave split over K (0: none)
 *   plan[3]  tiled GEMM: work units per split tile (1: none).  The tiles of
 *            the last, partial wave of persistent CTAs are each cut into
 *            plan[3] runs of consecutive K-blocks on otherwise idle SMs; a
 *            tile's last unit adds the fp32 partials in split order (the
 *            same bits whichever unit finishes last), so these tiles' sums
 *            round differently from a whole tile's, within the tolerance.
 * fg8_linear_run_chain always uses 256-wide tiles (and its own tail plan);
 * fg8_gemm_prequant, fg8_linear_static and fg8_linear_fused use fg8_linear's.
 * Returns FG8_ERR_INVALID_ARG on bad arguments or a NULL plan. */
FG8_API fg8_status fg8_linear_plan(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt, int32_t* plan);

/* The layer ([zh] §八 step 6, FP8Linear.forward -> fp8_linear; [zh] §6.1 the
 * block (128,128) + dynamic-activation fast path):
 *   y[M, N] = dequant(quantize_act(x)) . dequant(wq, w_scale_inv)^T + bias
 *   x_bf16      [M, K] bf16, row stride ld_x
 *   wq_e4m3     [N, K] e4m3fn, row stride K; w_scale_inv as fg8_quantize_weight
 *   bias_bf16   [N] bf16 or NULL
 *   y_bf16      [M, N] bf16, row stride ld_y (output; written once, RNE)
 *   workspace   >= fg8_linear_workspace_bytes(M, N, K, fmt), 256-byte aligned,
 *               caller-owned device memory.  Its first 1024 bytes are a
 *               header: a sticky device status word and the few-token path's
 *               split-K arrival counters, which the kernels leave at zero.
 *               Zero the header once before first use (e.g. allocate the
 *               workspace zero-filled); fg8_check_device_status reads and
 *               clears the status word, and after a failed call the rest of
 *               the header but the epoch word of fg8_linear_fused.  Calls sharing a workspace must not overlap on the
 *               device.
 * fg8_linear is fg8_linear_prepare (quantize x into the workspace) then
 * fg8_linear_run (the GEMM), which picks its kernel by shape: for M <= 32,
 * and for M <= 128 while ceil(N / 256) <= 37 (the tiled grid would cover at
 * most a quarter of the SMs), the few-token kernel, which streams the
 * weights as the tensor core's M side (128 weight rows per CTA, split over
 * K) and reduces the splits; otherwise the tiled GEMM.  With UE8M0 scales
 * and M <= 16 fg8_linear instead runs one few-token kernel that also
 * quantizes x (no prepare launch).
 * Float scales are applied exactly per 128-K block in float32 (never rounded
 * to a power of two, [zh] §七 补充); UE8M0 scales go through the tensor
 * core's block-scaled MMA.  M == 0 is a no-op. */
FG8_API fg8_status fg8_linear(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x,
                      const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16,
                      void* y_bf16, int64_t ld_y, fg8_scale_fmt fmt,
                      void* workspace, size_t workspace_bytes, void* stream);

/* fg8_linear in two halves, for callers that reuse one quantized activation
 * for several weights (same K) or time the GEMM on its own:
 *   fg8_linear_prepare  quantizes x into the workspace in the GEMM's layouts
 *                       (and, for UE8M0, packs w_scale_inv's scale-factor tiles);
 *   fg8_linear_run      runs the GEMM from that workspace.
 * prepare followed by run on the same stream and workspace is fg8_linear
 * (bit for bit), except with UE8M0 scales and M <= 16, where fg8_linear
 * quantizes inside its few-token kernel (same codes and scales; its sums
 * may round differently within the stated tolerance).  The workspace is
 * fg8_linear_workspace_bytes, as for fg8_linear.
 * Arguments and checks are those of fg8_linear. */
FG8_API fg8_status fg8_linear_prepare(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x,
                                      const void* w_scale_inv, fg8_scale_fmt fmt, void* workspace,
                                      size_t workspace_bytes, void* stream);
FG8_API fg8_status fg8_linear_run(const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16,
                                  void* y_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_y,
                                  fg8_scale_fmt fmt, void* workspace, size_t workspace_bytes, void* stream);

/* Two consecutive layers, the second fed by the first's output: runs this
 * layer's GEMM from `workspace` (after fg8_linear_prepare) and, in the same
 * kernel's epilogue, quantizes each bf16 output row group exactly as
 * fg8_linear_prepare(y_bf16, M, next_N, N, ...) would, writing the result into
 * `next_workspace` together with the next layer's weight scales
 * (`next_w_scale_inv`, [ceil(next_N/128), ceil(N/128)]).  A following
 * fg8_linear_run(next layer, next_workspace) then computes the second layer
 * without its own activation-quantization pass over y.  y_bf16 is still
 * written.  Checks as fg8_linear for both layers (N % 16 == 0, since N is the
 * next layer's K).  Same results, bit for bit, as prepare + run per layer. */
FG8_API fg8_status fg8_linear_run_chain(const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16,
                                        void* y_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_y,
                                        fg8_scale_fmt fmt, void* workspace, size_t workspace_bytes, int64_t next_N,
                                        const void* next_w_scale_inv, void* next_workspace,
                                        size_t next_workspace_bytes, void* stream);

/* fg8_linear with the activation quantization inside the GEMM kernel ([zh]
 * §八 step 6 / §6.1 make the per-token quantization part of fp8_linear; here
 * it is fused into the tiled GEMM's launch instead of running as a separate
 * prepare kernel).  Before its tiles, every CTA of the GEMM quantizes a share
 * of x in 128-row x 128-channel units (the same codes and scales as
 * fg8_quantize_act, in the GEMM's layouts) and publishes each unit with a
 * flag; the roles that read a unit wait for its flag (bounded waits).  This
 * covers the tiled path (M above the few-token range) with K <= 4096 (up to
 * 32 K-blocks).  With M <= 16 (and no next layer) the few-token kernel
 * quantizes x itself, in quantizer warps, for either scale format.  Other
 * shapes run exactly fg8_linear (or, with a next layer, fg8_linear_prepare +
 * fg8_linear_run_chain).  Measured on B200, the separate quantization launch
 * that fg8_linear overlaps with the GEMM is faster for float scales, which is
 * why fg8_linear keeps it; this entry point is for callers that want a single
 * launch per layer.
 *   Arguments as fg8_linear, plus an optional next layer as in
 *   fg8_linear_run_chain: with next_w_scale_inv non-NULL the epilogue also
 *   quantizes y for a layer with next_N outputs into next_workspace
 *   (>= fg8_linear_workspace_bytes(M, next_N, N, fmt)), after which
 *   fg8_linear_run(next layer, next_workspace) computes that layer.  With
 *   next_w_scale_inv NULL, next_N, next_workspace and next_workspace_bytes
 *   are ignored.
 *   workspace   >= fg8_linear_fused_workspace_bytes(M, N, K, fmt), 256-byte
 *               aligned, ZERO-FILLED IN FULL before its first use: beyond
 *               fg8_linear's layout it holds one flag per unit of x, and the
 *               header holds the call epoch the flags are compared with (an
 *               epoch that only advances; fg8_check_device_status keeps it).
 *               Do not zero the header alone between fused calls on one
 *               workspace.  Calls sharing a workspace must not overlap.
 * The tiled path gives fg8_linear's results bit for bit (and
 * fg8_linear_run_chain's); the few-token kernel's sums may round differently
 * within the stated tolerance. */
FG8_API size_t fg8_linear_fused_workspace_bytes(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt);
FG8_API fg8_status fg8_linear_fused(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x,
                                    const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16,
                                    void* y_bf16, int64_t ld_y, fg8_scale_fmt fmt, void* workspace,
                                    size_t workspace_bytes, int64_t next_N, const void* next_w_scale_inv,
                                    void* next_workspace, size_t next_workspace_bytes, void* stream);

/* fg8_linear without a caller workspace, for callers that cannot allocate
 * device memory (for example a host framework that owns all device memory
 * through its own pool, or code that must never call cudaMalloc because it
 * can synchronize the device).  The pages have no counterpart of this entry
 * point; it computes exactly what fg8_linear computes, with the same
 * arguments minus the workspace.
 *   - Scratch: a fixed 64 MiB array in this library's device memory (a
 *     file-scope __device__ array; every device that loads the library keeps
 *     it until the process exits).  No call allocates or frees anything.
 *   - Size limit: shapes whose fg8_linear_workspace_bytes(M, N, K, fmt)
 *     exceeds 64 MiB return FG8_ERR_WORKSPACE without launching.
 *   - The first call on each device looks up the scratch's device address
 *     (this may load the library's device module); make that first call
 *     before any stream capture on that device.
 *   - All calls on a device share the one scratch, which keeps the previous
 *     call's contents; each call clears the part that must start at zero.
 *     Calls that overlap on the GPU (different streams, or concurrent host
 *     threads) race on it: serialize them.
 *   - Arguments are checked exactly as fg8_linear checks them, before the
 *     scratch is looked up or touched: a refused call changes nothing.
 *   - Device-side wait timeouts are not reported through this entry point. */
FG8_API fg8_status fg8_linear_noalloc(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x,
                                      const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16,
                                      void* y_bf16, int64_t ld_y, fg8_scale_fmt fmt, void* stream);

/* Bytes of workspace fg8_gemm_prequant needs (with room for the tiled GEMM's
 * split-K tail, as fg8_linear_workspace_bytes).  0 on bad arguments. */
FG8_API size_t fg8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt);

/* The GEMM alone on already-quantized activations (the layouts
 * fg8_quantize_act writes): same result as fg8_linear for the same xq/x_scale.
 *   xq_e4m3 [M, K] row stride K; x_scale [M, ceil(K/128)] row-major. */
FG8_API fg8_status fg8_gemm_prequant(const void* xq_e4m3, const void* x_scale, const void* wq_e4m3,
                             const void* w_scale_inv, const void* bias_bf16, void* y_bf16,
                             int64_t M, int64_t N, int64_t K, int64_t ld_y, fg8_scale_fmt fmt,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Static activation scheme ([zh] §四 activation_scheme "static", §6.3; float
 * scales only): x is quantized with one precomputed scale for the whole
 * tensor, q = e4m3_rn_satfinite(RN_f32(x / *act_scale)) (values beyond 448
 * times the scale saturate), instead of per-group dynamic scales.
 *   act_scale   one float32 in device memory, > 0 and finite (4-byte aligned)
 *   fg8_quantize_act_static: xq_e4m3 [M, K] and x_scale [M, ceil(K/128)]
 *               float32, every entry set to the scale (the layout
 *               fg8_gemm_prequant reads)
 *   fg8_linear_static: as fg8_linear with scale_fmt FLOAT (the same
 *               workspace, fg8_linear_workspace_bytes(M, N, K, FLOAT), checked
 *               in full before anything is launched).
 * Checks and errors as fg8_quantize_act / fg8_linear. */
FG8_API fg8_status fg8_quantize_act_static(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x,
                                           const float* act_scale, void* xq_e4m3, void* x_scale, void* stream);
FG8_API fg8_status fg8_linear_static(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x,
                                     const float* act_scale, const void* wq_e4m3, const void* w_scale_inv,
                                     const void* bias_bf16, void* y_bf16, int64_t ld_y, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* Non-default block sizes ([zh] §八: the tests cover weight_block_size such
 * as (32, 32)).  Reading: the activation groups follow the weight's
 * input-channel block, so block = b means 1 x b activation groups and b x b
 * weight blocks; scales are shaped [M, ceil(K/b)] and [ceil(N/b), ceil(K/b)].
 * block is 32, 64 or 128 (128 forwards to the calls above); every call takes
 * either scale format.  In fg8_linear_block, UE8M0 scales go through the
 * tensor core's block-scaled MMA (one scale per 32 K per row; a 64-block's
 * scale on both of its steps), and float32 scales are promoted in float32
 * registers per b-wide slice of K, exactly as the 128 layer promotes per
 * K-block: y = bias + sum over slices of P_slice * (sx * sw).  It always runs
 * the tiled GEMM (no few-token kernel).  Other checks and errors as the 128
 * versions (block sizes other than 32, 64 and 128 are FG8_ERR_INVALID_ARG);
 * the workspace is fg8_linear_block_workspace_bytes (0 for an unsupported
 * combination), with the header rules of fg8_linear. */
FG8_API fg8_status fg8_quantize_act_block(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, void* xq_e4m3,
                                          void* x_scale, fg8_scale_fmt fmt, int block, void* stream);
FG8_API fg8_status fg8_quantize_weight_block(const void* w_bf16, int64_t N, int64_t K, int64_t ld_w, void* wq_e4m3,
                                             void* w_scale_inv, fg8_scale_fmt fmt, int block, void* stream);
FG8_API size_t fg8_linear_block_workspace_bytes(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt, int block);
FG8_API fg8_status fg8_linear_block(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x,
                                    const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16,
                                    void* y_bf16, int64_t ld_y, fg8_scale_fmt fmt, int block, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* MoE experts ([zh] §6.4 and [pt] "Caminho rápido do DeepGEMM": FP8Experts
 * sends each expert's tokens through this layer with that expert's e4m3
 * weights and block scales; on Blackwell the expert kernels take UE8M0
 * scales, float32 scales being the grouped_mm alternative -- both work here).
 * The pages print no kernel interface; the layout taken is the contiguous
 * grouped one: the routed rows of x are sorted by expert and each expert's
 * run is padded to whole blocks of 128 rows.
 *   x_bf16       [M, K] bf16, row stride ld_x: the routed rows
 *   row_expert   [M] int32 (device, 4-byte aligned): block t = rows
 *                [128 t, 128 t + 128) is computed with expert
 *                row_expert[128 t]; -1 there skips the block (its y rows are
 *                not written).  The other rows' entries are not read (padding
 *                rows inside a computed block are computed with it).  An
 *                entry >= E also skips its block and leaves
 *                FG8_ERR_INVALID_ARG in the workspace's status word.
 *   wq_e4m3      [E, N, K] e4m3fn (expert e's [N, K] matrix at e*N*K bytes)
 *   w_scale_inv  [E, ceil(N/128), ceil(K/128)] float32 or UE8M0 bytes
 *   bias_bf16    [E, N] bf16 or NULL
 *   y_bf16       [M, N] bf16, row stride ld_y
 *   workspace    >= fg8_grouped_linear_workspace_bytes(M, E, N, K, fmt),
 *                with the header rules of fg8_linear
 * y[r] = fg8_linear of row r with expert e's weights, bit for bit the dense
 * layer's arithmetic (per-token activation groups, exact float scale
 * promotion or the block-scaled MMA for UE8M0).  Checks as fg8_linear, plus
 * 1 <= E <= 65535 and E*N + 256 <= 2^31 - 1. */
FG8_API size_t fg8_grouped_linear_workspace_bytes(int64_t M, int64_t E, int64_t N, int64_t K, fg8_scale_fmt fmt);
FG8_API fg8_status fg8_grouped_linear(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x,
                                      const int32_t* row_expert, int64_t E, int64_t N, const void* wq_e4m3,
                                      const void* w_scale_inv, const void* bias_bf16, void* y_bf16, int64_t ld_y,
                                      fg8_scale_fmt fmt, void* workspace, size_t workspace_bytes, void* stream);
/* The batched expert layout ([zh] §6.4's batched_mm alternative: each
 * expert's tokens in a slab of `cap` rows, x [E * cap, K]) as the grouped
 * layout: writes row_expert [E * cap] (device int32), row e * cap + r =
 * e for r < counts[e] (device int32 [E]) and -1 beyond, so blocks past an
 * expert's count are skipped.  cap % 128 == 0 (FG8_ERR_ALIGNMENT otherwise:
 * a 128-row block must not straddle two slabs); counts[e] > cap computes
 * the whole slab.  Then fg8_grouped_linear on M = E * cap rows. */
FG8_API fg8_status fg8_grouped_row_expert(const int32_t* counts, int64_t E, int64_t cap, int32_t* row_expert,
                                          void* stream);

/* fg8_grouped_linear in two halves (as fg8_linear_prepare / fg8_linear_run):
 * the prepare step quantizes x into the workspace (and, for UE8M0, packs
 * every expert's weight scales into scale-factor tiles); the run step is
 * the grouped GEMM.  prepare then run on one stream and workspace is
 * fg8_grouped_linear, bit for bit.  Arguments and checks as there. */
FG8_API fg8_status fg8_grouped_linear_prepare(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, int64_t E,
                                              int64_t N, const void* w_scale_inv, fg8_scale_fmt fmt, void* workspace,
                                              size_t workspace_bytes, void* stream);
FG8_API fg8_status fg8_grouped_linear_run(const int32_t* row_expert, int64_t E, const void* wq_e4m3,
                                          const void* w_scale_inv, const void* bias_bf16, void* y_bf16, int64_t M,
                                          int64_t N, int64_t K, int64_t ld_y, fg8_scale_fmt fmt, void* workspace,
                                          size_t workspace_bytes, void* stream);

/* Fp8Dequantize ([zh] §五 and §八 step 4: a pre-quantized checkpoint loaded
 * with dequantize=True folds each block's scale back into the weight):
 *   w[n, k] = bf16(value(wq[n, k]) * w_scale_inv[n / 128][k / 128]),
 * the product exact, rounded once to nearest even.
 *   wq_e4m3      [N, K] e4m3fn, row stride K (16-byte aligned)
 *   w_scale_inv  [ceil(N/128), ceil(K/128)] float32 (FLOAT) or UE8M0 bytes
 *   w_bf16       [N, K] bf16 output, row stride ld_w (16-byte aligned)
 * K % 16 == 0 and ld_w % 8 == 0 (FG8_ERR_ALIGNMENT otherwise).  Caller owns
 * all buffers; nothing is allocated. */
FG8_API fg8_status fg8_dequantize_weight(const void* wq_e4m3, int64_t N, int64_t K, const void* w_scale_inv,
                                         fg8_scale_fmt fmt, void* w_bf16, int64_t ld_w, void* stream);

/* The checkpoint scale conversion of [zh] §七: power-of-two UE8M0 scales
 * kept in float32 containers (key ".scale") become UE8M0 bytes exactly,
 * s = 2^e with -127 <= e <= 127 -> byte e + 127.  Any other value is no
 * UE8M0 scale: its byte is 255 (the UE8M0 NaN) and it is added to
 * *invalid_count (a device uint32; may be NULL).
 *   scale_f32 [n] float32 (4-byte aligned), scale_e8m0 [n] bytes. */
FG8_API fg8_status fg8_scale_to_ue8m0(const void* scale_f32, int64_t n, void* scale_e8m0, uint32_t* invalid_count,
                                      void* stream);

/* Synchronizes `stream`, reads and clears the status word a previous
 * fg8_linear / fg8_gemm_prequant / fg8_grouped_linear left in `workspace`:
 * FG8_OK; FG8_ERR_TIMEOUT if one of its device-side waits gave up (the
 * kernel then returned early; y is unspecified); FG8_ERR_INVALID_ARG if
 * fg8_grouped_linear met an expert index >= E (those blocks were skipped). */
FG8_API fg8_status fg8_check_device_status(void* workspace, void* stream);

/* Upper bound, in nanoseconds, on any single device-side wait of the GEMM
 * before it gives up with FG8_ERR_TIMEOUT (default 2e9).  Process-wide. */
FG8_API void fg8_set_wait_limit_ns(uint64_t ns);

/* Test hook for the timeout path (process-wide, off by default): when on,
 * the MMA thread of every GEMM launched afterwards first waits on an
 * mbarrier that nothing completes, so its bounded wait runs out after the
 * wait limit; the kernel then records FG8_ERR_TIMEOUT in the status word,
 * drains its own copies and tensor-core ops, frees TMEM and returns.  No
 * fault and no unbounded wait are involved.  Not for production use. */
FG8_API void fg8_set_test_stall(int on);

/* Static description of a status code. */
FG8_API const char* fg8_status_string(fg8_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
FG8_API int fg8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FG8_H_ */
