// fg8_oracle.cpp -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, obviously-correct CPU statement of what the fine-grained FP8
// linear layer computes.  It exists to check the CUDA library against; nothing
// in the product path may link, load or call it (only tests/, the smoke check
// and the bench's CPU-baseline leg do).  It shares no code, header, table or
// constant generator with the CUDA sources.
//
// Sources (the web pages this method is described on):
//   [zh] "Transformers 中的细粒度 FP8 量化：配置、DeepGEMM 加速路径与 UE8M0 缩放格式完全指南"
//   [pt] "FP8 de granularidade fina" (Transformers documentation, Portuguese)
// The pages name the scheme (per-token 1x128 activation groups, 128x128 weight
// blocks, e4m3fn storage, float32 or UE8M0 scales) but print no arithmetic.
// Every step below that the pages leave open carries the reading used here.
//
// e4m3fn is taken from its published definition (OCP 8-bit floating point
// specification, "E4M3" with no infinities): 1 sign bit, 4 exponent bits with
// bias 7, 3 mantissa bits; S.1111.111 is NaN; largest finite 448, smallest
// subnormal 2^-9.  UE8M0 is the OCP MX scale type: an 8-bit biased exponent,
// value 2^(b-127), b = 255 is NaN.
//
// Floating point: the pages fix float32 scales ([zh] §一: "weight_scale_inv"
// is a float32 tensor unless UE8M0), so the scale and the quotient x/scale are
// float32 operations, correctly rounded (round-to-nearest-even).  The GEMM is
// dequantize-then-accumulate in double, in increasing k.
//
// No blocking, fusion or reordering: every loop below is the definition.

#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include <omp.h>

static_assert(FLT_EVAL_METHOD == 0, "float expressions must evaluate in float");

namespace {

constexpr int kGroup = 128;       // [zh] §一: activation group width = weight input-channel block (128)
constexpr int kBlock = 128;       // [zh] §一 / [pt]: weight_block_size = (128, 128)
constexpr double kE4m3Max = 448.0;  // largest finite e4m3fn magnitude (S.1111.110)

// ---------------------------------------------------------------- e4m3fn ----
// Value of one e4m3fn code (OCP definition).  NaN for S.1111.111.
double e4m3_value(uint8_t code) {
  const int sign = code >> 7;
  const int expo = (code >> 3) & 0xF;
  const int mant = code & 0x7;
  if (expo == 0xF && mant == 0x7) return NAN;
  double mag;
  if (expo == 0) {
    mag = std::ldexp(static_cast<double>(mant), -9);          // 0.mmm * 2^(1-7)
  } else {
    mag = std::ldexp(8.0 + mant, expo - 7 - 3);              // 1.mmm * 2^(e-7)
  }
  return sign ? -mag : mag;
}

// Decoded non-negative codes 0x00..0x7E (increasing with the code).
struct E4m3Table {
  double v[0x7F];
  E4m3Table() {
    for (int c = 0; c <= 0x7E; ++c) v[c] = e4m3_value(static_cast<uint8_t>(c));
  }
};
const E4m3Table& e4m3_table() {
  static const E4m3Table t;
  return t;
}

// Round a float32 to e4m3fn: nearest finite code, ties to the code whose
// mantissa LSB is 0 (round-to-nearest-even), magnitudes >= 448 saturate to
// 448 (never NaN), the sign of f is kept (so -0 and negatives that round to
// zero give 0x80).  lo = the largest non-negative code whose value is <= |f|
// (binary search over the increasing table), hi = lo + 1; pick the nearer,
// the even one on a tie.
uint8_t e4m3_encode(float f) {
  const uint8_t sign = std::signbit(f) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(f));
  if (a >= kE4m3Max) return sign | 0x7E;
  const double* v = e4m3_table().v;
  int lo = 0, hi_excl = 0x7F;  // invariant: v[lo] <= a < v[hi_excl] (v[0x7F] taken as +inf)
  while (hi_excl - lo > 1) {
    const int mid = (lo + hi_excl) / 2;
    if (v[mid] <= a) lo = mid; else hi_excl = mid;
  }
  if (v[lo] == a) return sign | static_cast<uint8_t>(lo);
  const int hi = lo + 1;  // a < 448 = v[0x7E] so hi <= 0x7E
  const double mid = 0.5 * (v[lo] + v[hi]);  // exact: few significant bits
  int pick;
  if (a < mid) {
    pick = lo;
  } else if (a > mid) {
    pick = hi;
  } else {
    pick = (lo & 1) == 0 ? lo : hi;  // tie: even mantissa
  }
  return sign | static_cast<uint8_t>(pick);
}

// Value of a code through the table (same as e4m3_value; NaN codes never occur
// in quantizer output).
double e4m3_signed(uint8_t code) {
  if ((code & 0x7F) == 0x7F) return NAN;
  const double mag = e4m3_table().v[code & 0x7F];
  return (code & 0x80) ? -mag : mag;
}

// ----------------------------------------------------------------- UE8M0 ----
float e8m0_value(uint8_t b) { return std::ldexp(1.0f, static_cast<int>(b) - 127); }

// Smallest power of two >= s, as a UE8M0 byte.  s must be a positive normal
// float.  Reading of [zh] §七 补充 (DeepGEMM rounds float32 scales *up* to
// UE8M0): the UE8M0 scale is the float scale rounded up to a power of two.
uint8_t e8m0_ceil_byte(float s) {
  uint32_t bits;
  std::memcpy(&bits, &s, sizeof bits);
  const int biased = static_cast<int>((bits >> 23) & 0xFF);
  const uint32_t mant = bits & 0x7FFFFFu;
  return static_cast<uint8_t>(mant == 0 ? biased : biased + 1);
}

// ------------------------------------------------------------------ bf16 ----
float bf16_to_float(uint16_t h) {
  const uint32_t bits = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return f;
}

// Round a double to bf16 (8 significant bits) with round-to-nearest-even,
// directly from the double (no detour through float).  Finite inputs within
// the bf16 range only.
uint16_t bf16_from_double(double v) {
  if (v == 0.0) return std::signbit(v) ? 0x8000 : 0x0000;
  int e;
  std::frexp(std::fabs(v), &e);                    // |v| = f * 2^e, f in [0.5, 1)
  int q = e - 8;                                   // quantum exponent for 8 significant bits
  if (q < -133) q = -133;                          // bf16 subnormal quantum 2^-133
  const double scaled = std::ldexp(std::fabs(v), -q);
  const double r = std::nearbyint(scaled);         // default rounding mode: ties to even
  const float f = static_cast<float>(std::ldexp(r, q));  // exact (fits bf16, hence float)
  uint32_t bits;
  std::memcpy(&bits, &f, sizeof bits);
  uint16_t h = static_cast<uint16_t>(bits >> 16);
  if (v < 0) h |= 0x8000;
  return h;
}

// ----------------------------------------------------------- group scale ----
// Reading (the pages print no formula): the scale maps the group's largest
// magnitude onto the largest e4m3fn value, scale = amax / 448, a float32
// division; it is floored at 2^-126 (smallest normal float32, exactly a UE8M0
// value) so that an all-zero group has a finite, positive scale.
float group_scale(float amax) {
  float s = amax / 448.0f;
  const float floor_s = std::ldexp(1.0f, -126);
  if (s < floor_s) s = floor_s;
  return s;
}

int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

}  // namespace

extern "C" {

enum { ORC_FMT_FLOAT = 0, ORC_FMT_UE8M0 = 1 };

double orc_e4m3_value(uint8_t code) { return e4m3_value(code); }
uint8_t orc_e4m3_encode(float f) { return e4m3_encode(f); }
float orc_e8m0_value(uint8_t b) { return e8m0_value(b); }
uint8_t orc_e8m0_ceil_byte(float s) { return e8m0_ceil_byte(s); }
float orc_group_scale(float amax) { return group_scale(amax); }
uint16_t orc_bf16_from_double(double v) { return bf16_from_double(v); }

void orc_e4m3_encode_many(const float* f, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(f[i]);
}

// Dynamic per-token activation quantization ([zh] §一, [pt]): token row m is
// split into groups of `group` consecutive input channels (128 by default; the
// weight block's input-channel size, so (32, 32) blocks give 1x32 groups --
// [zh] §八 lists such non-default block sizes among the tested ones); the last
// group holds the remaining real channels; each group gets one scale from its
// own amax and its elements are cast to e4m3fn.
//   x      : bf16 bits, row m at x + m*ld_x
//   xq     : e4m3fn bytes [M, K] row-major
//   x_scale: [M, ceil(K/group)] row-major; float32 (fmt 0) or UE8M0 bytes (fmt 1)
// Returns 0, or -1 on a bad argument.
int orc_quantize_act_g(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, int fmt, int group,
                       uint8_t* xq, void* x_scale) {
  if (M < 0 || K <= 0 || ld_x < K || group <= 0 || (fmt != ORC_FMT_FLOAT && fmt != ORC_FMT_UE8M0)) return -1;
  const int Kb = ceil_div(K, group);
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int g = 0; g < Kb; ++g) {
      const int64_t k0 = static_cast<int64_t>(g) * group;
      const int64_t k1 = std::min<int64_t>(k0 + group, K);
      float amax = 0.0f;
      for (int64_t k = k0; k < k1; ++k) amax = std::fmax(amax, std::fabs(bf16_to_float(x[m * ld_x + k])));
      const float s = group_scale(amax);
      float s_used;
      if (fmt == ORC_FMT_FLOAT) {
        s_used = s;
        static_cast<float*>(x_scale)[m * Kb + g] = s;
      } else {
        const uint8_t b = e8m0_ceil_byte(s);
        s_used = e8m0_value(b);
        static_cast<uint8_t*>(x_scale)[m * Kb + g] = b;
      }
      for (int64_t k = k0; k < k1; ++k) {
        const float quotient = bf16_to_float(x[m * ld_x + k]) / s_used;
        xq[m * K + k] = e4m3_encode(quotient);
      }
    }
  }
  return 0;
}

int orc_quantize_act(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, int fmt, uint8_t* xq, void* x_scale) {
  return orc_quantize_act_g(x, M, K, ld_x, fmt, kGroup, xq, x_scale);
}

// 2-D block weight quantization ([zh] §一: one scale per block x block
// sub-matrix, 128 by default, weight_scale_inv shaped (ceil(out/block),
// ceil(in/block)); [zh] §三: bias is not
// quantized).  W is nn.Linear's [out=N, in=K].  Edge blocks use their real
// elements only.  W ~= dequant(wq) = value(wq) * scale_inv.
int orc_quantize_weight_b(const uint16_t* w, int64_t N, int64_t K, int64_t ld_w, int fmt, int block,
                          uint8_t* wq, void* w_scale_inv) {
  if (N <= 0 || K <= 0 || ld_w < K || block <= 0 || (fmt != ORC_FMT_FLOAT && fmt != ORC_FMT_UE8M0)) return -1;
  const int Nb = ceil_div(N, block);
  const int Kb = ceil_div(K, block);
#pragma omp parallel for collapse(2) schedule(static)
  for (int nb = 0; nb < Nb; ++nb) {
    for (int kb = 0; kb < Kb; ++kb) {
      const int64_t n0 = static_cast<int64_t>(nb) * block, n1 = std::min<int64_t>(n0 + block, N);
      const int64_t k0 = static_cast<int64_t>(kb) * block, k1 = std::min<int64_t>(k0 + block, K);
      float amax = 0.0f;
      for (int64_t n = n0; n < n1; ++n)
        for (int64_t k = k0; k < k1; ++k) amax = std::fmax(amax, std::fabs(bf16_to_float(w[n * ld_w + k])));
      const float s = group_scale(amax);
      float s_used;
      if (fmt == ORC_FMT_FLOAT) {
        s_used = s;
        static_cast<float*>(w_scale_inv)[nb * Kb + kb] = s;
      } else {
        const uint8_t b = e8m0_ceil_byte(s);
        s_used = e8m0_value(b);
        static_cast<uint8_t*>(w_scale_inv)[nb * Kb + kb] = b;
      }
      for (int64_t n = n0; n < n1; ++n)
        for (int64_t k = k0; k < k1; ++k) wq[n * K + k] = e4m3_encode(bf16_to_float(w[n * ld_w + k]) / s_used);
    }
  }
  return 0;
}

int orc_quantize_weight(const uint16_t* w, int64_t N, int64_t K, int64_t ld_w, int fmt, uint8_t* wq,
                        void* w_scale_inv) {
  return orc_quantize_weight_b(w, N, K, ld_w, fmt, kBlock, wq, w_scale_inv);
}

// The linear layer on quantized operands ([zh] §八 step 6: FP8Linear.forward
// hands quantized weights to fp8_linear):
//   y[m,n] = sum_k xhat[m,k] * what[n,k] + bias[n],
//   xhat = value(xq) * x_scale(m, k/block),  what = value(wq) * w_scale_inv(n/block, k/block),
// summed in double in increasing k; bias (bf16, may be NULL) added in double.
// Outputs, for each requested row (rows == NULL means all M rows, in order):
//   y64   [R, N] the double result, bound [R, N] = sum_k |xhat*what|,
//   y_bf16[R, N] the double result rounded once to bf16 (RNE).
int orc_linear_dequant_b(const uint8_t* xq, const void* x_scale, const uint8_t* wq, const void* w_scale_inv,
                         const uint16_t* bias, int64_t M, int64_t N, int64_t K, int fmt, int block,
                         const int64_t* rows, int64_t n_rows, double* y64, double* bound, uint16_t* y_bf16) {
  if (M < 0 || N <= 0 || K <= 0 || block <= 0 || (fmt != ORC_FMT_FLOAT && fmt != ORC_FMT_UE8M0)) return -1;
  const int Kb = ceil_div(K, block);
  const int64_t R = rows ? n_rows : M;
  auto xs_at = [&](int64_t m, int64_t g) -> double {
    return fmt == ORC_FMT_FLOAT ? static_cast<double>(static_cast<const float*>(x_scale)[m * Kb + g])
                                : static_cast<double>(e8m0_value(static_cast<const uint8_t*>(x_scale)[m * Kb + g]));
  };
  auto ws_at = [&](int64_t nb, int64_t kb) -> double {
    return fmt == ORC_FMT_FLOAT ? static_cast<double>(static_cast<const float*>(w_scale_inv)[nb * Kb + kb])
                                : static_cast<double>(e8m0_value(static_cast<const uint8_t*>(w_scale_inv)[nb * Kb + kb]));
  };
  // Dequantized weight rows, once (pure hoisting of value(wq)*scale).
  std::vector<double> what(static_cast<size_t>(N * K));
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) what[n * K + k] = e4m3_signed(wq[n * K + k]) * ws_at(n / block, k / block);

  for (int64_t r = 0; r < R; ++r) {
    const int64_t m = rows ? rows[r] : r;
    if (m < 0 || m >= M) return -1;
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < R; ++r) {
    const int64_t m = rows ? rows[r] : r;
    std::vector<double> xhat(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) xhat[k] = e4m3_signed(xq[m * K + k]) * xs_at(m, k / block);
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0, mag = 0.0;
      const double* wr = &what[n * K];
      for (int64_t k = 0; k < K; ++k) {
        const double p = xhat[k] * wr[k];
        acc += p;
        mag += std::fabs(p);
      }
      if (bias) acc += static_cast<double>(bf16_to_float(bias[n]));
      y64[r * N + n] = acc;
      bound[r * N + n] = mag;
      y_bf16[r * N + n] = bf16_from_double(acc);
    }
  }
  return 0;
}

int orc_linear_dequant(const uint8_t* xq, const void* x_scale, const uint8_t* wq, const void* w_scale_inv,
                       const uint16_t* bias, int64_t M, int64_t N, int64_t K, int fmt, const int64_t* rows,
                       int64_t n_rows, double* y64, double* bound, uint16_t* y_bf16) {
  return orc_linear_dequant_b(xq, x_scale, wq, w_scale_inv, bias, M, N, K, fmt, kBlock, rows, n_rows, y64, bound,
                              y_bf16);
}

// Fp8Dequantize ([zh] §五 and §八 step 4: a pre-quantized checkpoint loaded
// with dequantize=True folds each 128x128 block's scale back into the
// weight): w[n,k] = value(wq[n,k]) * scale_inv(n/128, k/128), the product
// formed exactly in double and rounded once to bf16 (RNE).
//   wq: e4m3fn [N, K] row-major; w_scale_inv as orc_quantize_weight writes;
//   w: bf16 bits, row n at w + n*ld_w.
int orc_dequantize_weight(const uint8_t* wq, int64_t N, int64_t K, const void* w_scale_inv, int fmt, uint16_t* w,
                          int64_t ld_w) {
  if (N <= 0 || K <= 0 || ld_w < K || (fmt != ORC_FMT_FLOAT && fmt != ORC_FMT_UE8M0)) return -1;
  const int Kb = ceil_div(K, kBlock);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      const int64_t blk = (n / kBlock) * Kb + k / kBlock;
      const double s = fmt == ORC_FMT_FLOAT ? static_cast<double>(static_cast<const float*>(w_scale_inv)[blk])
                                            : static_cast<double>(e8m0_value(static_cast<const uint8_t*>(w_scale_inv)[blk]));
      w[n * ld_w + k] = bf16_from_double(e4m3_signed(wq[n * K + k]) * s);
    }
  }
  return 0;
}

// The checkpoint scale conversion ([zh] §七: some checkpoints keep
// power-of-two UE8M0 scales in float32 containers under the key ".scale";
// after loading they are converted exactly to the UE8M0 dtype).  A UE8M0
// byte b is 2^(b-127), so s = 2^e with -127 <= e <= 127 becomes e + 127.
// Any other input is no UE8M0 value: it becomes 255 (the UE8M0 NaN) and is
// counted.  Returns the count.
int64_t orc_scale_to_e8m0(const float* s, int64_t n, uint8_t* out) {
  int64_t bad = 0;
  for (int64_t i = 0; i < n; ++i) {
    const float v = s[i];
    uint8_t b = 255;
    if (std::isfinite(v) && v > 0.0f) {
      int e2;
      const double f = std::frexp(static_cast<double>(v), &e2);  // v = f * 2^e2, f in [0.5, 1)
      const int e = e2 - 1;
      if (f == 0.5 && e >= -127 && e <= 127) b = static_cast<uint8_t>(e + 127);
    }
    if (b == 255) ++bad;
    out[i] = b;
  }
  return bad;
}

// Static activation scheme ([zh] §四: activation_scheme is "dynamic" or
// "static"; §6.3: static activation quantization).  The pages print no
// formula; the reading here: one precomputed float32 scale s > 0 for the
// whole tensor, q = e4m3_rn_satfinite(RN_f32(x / s)) -- the dynamic rule with
// the group scale replaced by s (values beyond 448 s saturate).
int orc_quantize_act_static(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, float s, uint8_t* xq) {
  if (M < 0 || K <= 0 || ld_x < K || !(s > 0.0f) || !std::isfinite(s)) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) xq[m * K + k] = e4m3_encode(bf16_to_float(x[m * ld_x + k]) / s);
  return 0;
}

// Team size of the OpenMP loops above (OMP_NUM_THREADS, else the CPUs this
// process may run on), for reporting how many host threads a timing used.
int orc_num_threads(void) { return omp_get_max_threads(); }

}  // extern "C"
