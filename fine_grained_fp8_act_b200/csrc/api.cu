// api.cu -- the extern "C" boundary of libfg8 (declared in include/fg8.h).
//
// Host-side argument checks happen before anything is launched; every
// accepted call enqueues its kernels on the caller's stream and returns.  No
// device memory is allocated here: fg8_linear / fg8_gemm_prequant carve their
// scratch out of the caller's workspace.

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "fg8.h"
#include "fg8_internal.h"

namespace {

using namespace fg8;

constexpr int64_t kMaxDim = 2147483647LL;
constexpr size_t kHeaderBytes = kWorkspaceHeaderBytes;  // status word, split-K counters
constexpr size_t kAlign = 256;

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<int> g_test_stall{0};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
  bool ok = false;
  int sms = 0;
};

// Compute capability 10.0 (B200) and SM count of the current device, cached.
fg8_status current_device(DeviceInfo* out) {
  static std::atomic<int> cached_cc[64];
  static std::atomic<int> cached_sms[64];
  static std::atomic<bool> init{false};
  if (!init.load()) {
    for (int i = 0; i < 64; ++i) {
      cached_cc[i].store(-1);
      cached_sms[i].store(0);
    }
    init.store(true);
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return FG8_ERR_UNSUPPORTED_DEVICE;
  }
  int cc = dev < 64 ? cached_cc[dev].load() : -1;
  int sms = dev < 64 ? cached_sms[dev].load() : 0;
  if (cc < 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return FG8_ERR_UNSUPPORTED_DEVICE;
    }
    cc = major * 10 + minor;
    if (dev < 64) {
      cached_cc[dev].store(cc);
      cached_sms[dev].store(sms);
    }
  }
  if (cc != 100) return FG8_ERR_UNSUPPORTED_DEVICE;
  out->ok = true;
  out->sms = sms;
  return FG8_OK;
}

bool fmt_ok(int fmt) { return fmt == FG8_SCALE_FLOAT || fmt == FG8_SCALE_UE8M0; }

// Shared shape checks of the GEMM entry points.
fg8_status check_gemm_shape(int64_t M, int64_t N, int64_t K, int fmt) {
  if (!fmt_ok(fmt)) return FG8_ERR_INVALID_ARG;
  if (M < 0 || N <= 0 || K <= 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return FG8_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % 8 != 0) return FG8_ERR_ALIGNMENT;
  return FG8_OK;
}

// Workspace of fg8_linear: [header | xq (M*K) | x scales | W scales].
//   float: x scales K-major [Kb][ld_s] float32 (the GEMM reads the caller's
//          weight scales as given: no W-scale region)
//   UE8M0: x and W scale-factor tiles (512 bytes per 128 rows x 4 K-blocks)
struct LinearWs {
  size_t xq_off, xs_off, wsc_off, total;
  int64_t ld_s;
};

LinearWs linear_ws_layout(int64_t M, int64_t N, int64_t K, int fmt) {
  LinearWs w;
  const int Kb = ceil_div(K, kGroup);
  const int Kq = ceil_div(Kb, 4);
  w.xq_off = kHeaderBytes;
  size_t off = align_up(w.xq_off + static_cast<size_t>(M) * K, kAlign);
  w.xs_off = off;
  w.ld_s = kmajor_ld(M);
  if (fmt == FG8_SCALE_FLOAT) {
    off = align_up(off + static_cast<size_t>(Kb) * w.ld_s * sizeof(float), kAlign);
    w.wsc_off = off;
  } else {
    off = align_up(off + static_cast<size_t>(ceil_div(M, 128)) * Kq * kSfChunkBytes, kAlign);
    w.wsc_off = off;
    off = align_up(off + static_cast<size_t>(sfb_rows(N) / 128) * Kq * kSfChunkBytes, kAlign);
  }
  w.total = off;
  return w;
}

// Workspace of fg8_gemm_prequant: [header | x scales | W scales] in the GEMM's
// layouts (as fg8_linear's).
struct GemmWs {
  size_t xs_off, wsc_off, total;
  int64_t ld_s;
};

GemmWs gemm_ws_layout(int64_t M, int64_t N, int64_t K, int fmt) {
  GemmWs w;
  const int Kb = ceil_div(K, kGroup);
  const int Kq = ceil_div(Kb, 4);
  size_t off = kHeaderBytes;
  w.xs_off = off;
  w.ld_s = kmajor_ld(M);
  if (fmt == FG8_SCALE_FLOAT) {
    off = align_up(off + static_cast<size_t>(Kb) * w.ld_s * sizeof(float), kAlign);
    w.wsc_off = off;
  } else {
    off = align_up(off + static_cast<size_t>(ceil_div(M, 128)) * Kq * kSfChunkBytes, kAlign);
    w.wsc_off = off;
    off = align_up(off + static_cast<size_t>(sfb_rows(N) / 128) * Kq * kSfChunkBytes, kAlign);
  }
  w.total = off;
  return w;
}

// Split-K counters of the few-token path that do not fit in the header
// (more than kHeaderCounters weight tiles) go after it, cleared per call.
size_t small_counter_bytes(int64_t N) {
  const int64_t nt = (N + 127) / 128;
  return nt > kHeaderCounters ? align_up(static_cast<size_t>(nt) * 4, kAlign) : 0;
}

// SM count the workspace sizes plan the tiled GEMM's split-K tail for: the
// current device's (a B200's 148 when there is none to ask).
int sizing_sms() {
  DeviceInfo d;
  if (current_device(&d) == FG8_OK && d.sms > 0) return d.sms;
  return 148;
}

// fg8_linear's workspace: the prepare/run layout, then for few tokens the
// small-M path's (counters beyond the header) and split-K partials, and for
// the tiled GEMM the partials of its split-K tail (none for most shapes).
size_t linear_workspace_need(int64_t M, int64_t N, int64_t K, int fmt) {
  size_t need = linear_ws_layout(M, N, K, fmt).total;
  if (use_small_m(M, N)) return align_up(need, kAlign) + small_counter_bytes(N) + small_m_partial_bytes(M, N, K);
  const size_t area = gemm_split_area(M, N, K, fmt, sizing_sms());
  return area > 0 ? align_up(need, kAlign) + area : need;
}

// fg8_gemm_prequant's workspace: its layout, then the split-K tail's partials.
size_t gemm_workspace_need(int64_t M, int64_t N, int64_t K, int fmt) {
  const size_t need = gemm_ws_layout(M, N, K, fmt).total;
  const size_t area = gemm_split_area(M, N, K, fmt, sizing_sms());
  return area > 0 ? align_up(need, kAlign) + area : need;
}

// The split-K tail's room inside a workspace whose own layout ends at `base`.
void set_split_area(GemmArgs& g, void* workspace, size_t workspace_bytes, size_t base) {
  const size_t off = align_up(base, kAlign);
  g.split_ws = workspace_bytes > off ? static_cast<uint8_t*>(workspace) + off : nullptr;
  g.split_bytes = workspace_bytes > off ? workspace_bytes - off : 0;
}

fg8_status check_workspace(void* ws, size_t bytes, size_t need) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || bytes < need) return FG8_ERR_WORKSPACE;
  return FG8_OK;
}

fg8_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FG8_OK;
  cudaGetLastError();
  return FG8_ERR_CUDA;
}

}  // namespace

// x's codes and scales into the workspace in the GEMM's layouts (the
// activation half of fg8_linear_prepare).
fg8_status prepare_act(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, int fmt, uint8_t* ws,
                       const LinearWs& L, const DeviceInfo& dev, cudaStream_t s) {
  ActQuantArgs a{};
  a.x = x_bf16;
  a.ld_x = ld_x;
  a.M = static_cast<int>(M);
  a.K = static_cast<int>(K);
  a.Kb = ceil_div(K, kGroup);
  a.xq = ws + L.xq_off;
  a.xs = ws + L.xs_off;
  a.layout = fmt == FG8_SCALE_FLOAT ? kScaleKMajor : kScaleSfTiles;
  a.ld_s = L.ld_s;
  a.Kq = ceil_div(a.Kb, 4);
  a.M_pad = ceil_div(M, 128) * 128;
  return cuda_status(launch_act_quant(a, fmt, dev.sms, s));
}

// Grouped (MoE) workspace: fg8_linear's layout for the M routed rows, with
// the UE8M0 weight scale-factor region holding every expert's tiles -- E x
// ceil(N/128) tiles of 128 rows, plus one spare the 256-wide tile of the
// last expert may read past its last block.
int64_t grouped_sf_rows(int64_t E, int64_t N) { return (E * ceil_div(N, 128) + 1) * 128; }

fg8_status check_grouped_shape(int64_t M, int64_t E, int64_t N, int64_t K, int fmt) {
  if (fg8_status st = check_gemm_shape(M, N, K, fmt); st != FG8_OK) return st;
  if (E <= 0 || E > 65535 || E * N + 256 > kMaxDim || E * ceil_div(N, 128) * ceil_div(K, kGroup) > kMaxDim)
    return FG8_ERR_INVALID_ARG;
  return FG8_OK;
}

LinearWs grouped_ws_layout(int64_t M, int64_t E, int64_t N, int64_t K, int fmt) {
  return linear_ws_layout(M, fmt == FG8_SCALE_UE8M0 ? grouped_sf_rows(E, N) : N, K, fmt);
}

// The few-token kernel (small_m.cu) on fg8_linear's workspace: counters in
// the header (or after the prepare layout for more than kHeaderCounters
// weight tiles), split-K partials after the prepare layout.  fused: x is
// quantized inside the kernel; otherwise the prepare step's codes and
// scales are in the workspace already.
fg8_status launch_small_path(bool fused, const void* x_bf16, int64_t ld_x, int64_t M, int64_t N, int64_t K,
                             const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16, void* y_bf16,
                             int64_t ld_y, int fmt, void* workspace, void* stream) {
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const LinearWs L = linear_ws_layout(M, N, K, fmt);
  const size_t small_off = align_up(L.total, kAlign);
  SmallMArgs a{};
  a.x = x_bf16;
  a.ld_x = ld_x;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.wq = wq_e4m3;
  a.w_scale = w_scale_inv;
  a.bias = bias_bf16;
  a.y = y_bf16;
  a.ld_y = ld_y;
  a.splits = small_m_splits(static_cast<int>(M), static_cast<int>(N), static_cast<int>(K));
  const size_t extra = small_counter_bytes(N);
  a.zero_counters = extra > 0;
  a.counters = reinterpret_cast<uint32_t*>(ws + (extra > 0 ? small_off : kHeaderCounterOffset));
  a.part = reinterpret_cast<float*>(ws + small_off + extra);
  a.preq = !fused;
  if (a.preq) {
    a.xq = ws + L.xq_off;
    a.xs_t = reinterpret_cast<const float*>(ws + L.xs_off);
    a.ld_s = L.ld_s;
    a.sfa = ws + L.xs_off;
    a.sfb = ws + L.wsc_off;
    a.Kq = ceil_div(ceil_div(K, kGroup), 4);
  }
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.test_stall = g_test_stall.load();
  return cuda_status(launch_small_m(a, fmt, static_cast<cudaStream_t>(stream)));
}

namespace fg8 {

// fg8_linear's argument checks (everything but the workspace), in the order
// fg8_linear applies them; FG8_OK for M == 0 with a valid shape.
int check_linear_args_status(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x, const void* wq_e4m3,
                             const void* w_scale_inv, const void* bias_bf16, const void* y_bf16, int64_t ld_y,
                             int fmt) {
  if (fg8_status st = check_gemm_shape(M, N, K, fmt); st != FG8_OK) return st;
  if (ld_x < K || ld_y < N) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (x_bf16 == nullptr || wq_e4m3 == nullptr || w_scale_inv == nullptr || y_bf16 == nullptr)
    return FG8_ERR_INVALID_ARG;
  if (ld_x % 8 != 0 || ld_y % 8 != 0 || !aligned16(x_bf16) || !aligned16(wq_e4m3) || !aligned16(y_bf16) ||
      (bias_bf16 != nullptr && !aligned16(bias_bf16)) || !aligned16(w_scale_inv))
    return FG8_ERR_ALIGNMENT;
  return FG8_OK;
}

}  // namespace fg8

extern "C" {

int fg8_version(void) { return 100; }

const char* fg8_status_string(fg8_status st) {
  switch (st) {
    case FG8_OK: return "ok";
    case FG8_ERR_INVALID_ARG: return "invalid argument (format, size, pointer or leading dimension)";
    case FG8_ERR_ALIGNMENT: return "alignment (K % 16, N % 8, ld % 8 for bf16, 16-byte pointers)";
    case FG8_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0, B200)";
    case FG8_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FG8_ERR_CUDA: return "CUDA launch or runtime error";
    case FG8_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

void fg8_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

void fg8_set_test_stall(int on) { g_test_stall.store(on != 0 ? 1 : 0); }

fg8_status fg8_quantize_weight(const void* w_bf16, int64_t N, int64_t K, int64_t ld_w, void* wq_e4m3,
                               void* w_scale_inv, fg8_scale_fmt fmt, void* stream) {
  if (!fmt_ok(fmt) || N <= 0 || K <= 0 || N > kMaxDim || K > kMaxDim || ld_w < K) return FG8_ERR_INVALID_ARG;
  if (w_bf16 == nullptr || wq_e4m3 == nullptr || w_scale_inv == nullptr) return FG8_ERR_INVALID_ARG;
  if (ceil_div(N, 128) > 65535) return FG8_ERR_INVALID_ARG;
  if (K % 16 != 0 || ld_w % 8 != 0 || !aligned16(w_bf16) || !aligned16(wq_e4m3)) return FG8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  return cuda_status(launch_weight_quant(w_bf16, ld_w, static_cast<int>(N), static_cast<int>(K),
                                         static_cast<uint8_t*>(wq_e4m3), w_scale_inv, fmt,
                                         static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, void* xq_e4m3, void* x_scale,
                            fg8_scale_fmt fmt, void* stream) {
  if (!fmt_ok(fmt) || M < 0 || K <= 0 || M > kMaxDim || K > kMaxDim || ld_x < K) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (x_bf16 == nullptr || xq_e4m3 == nullptr || x_scale == nullptr) return FG8_ERR_INVALID_ARG;
  if (K % 16 != 0 || ld_x % 8 != 0 || !aligned16(x_bf16) || !aligned16(xq_e4m3)) return FG8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  ActQuantArgs a{};
  a.x = x_bf16;
  a.ld_x = ld_x;
  a.M = static_cast<int>(M);
  a.K = static_cast<int>(K);
  a.Kb = ceil_div(K, kGroup);
  a.xq = static_cast<uint8_t*>(xq_e4m3);
  a.xs = x_scale;
  a.layout = kScaleRowMajor;
  return cuda_status(launch_act_quant(a, fmt, dev.sms, static_cast<cudaStream_t>(stream)));
}

size_t fg8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt) {
  if (check_gemm_shape(M, N, K, fmt) != FG8_OK) return 0;
  return linear_workspace_need(M, N, K, fmt);
}

fg8_status fg8_linear_plan(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt, int32_t* plan) {
  if (fg8_status st = check_gemm_shape(M, N, K, fmt); st != FG8_OK) return st;
  if (plan == nullptr) return FG8_ERR_INVALID_ARG;
  if (M > 0 && use_small_m(M, N)) {
    plan[0] = use_fused_small_m(M, fmt) ? 2 : 1;
    plan[1] = 0;
    plan[2] = 0;
    plan[3] = 1;
    return FG8_OK;
  }
  const int sms = sizing_sms();
  const int Kb = ceil_div(K, kGroup), align = fmt == FG8_SCALE_UE8M0 ? 4 : 1;
  const int bn = choose_block_n(static_cast<int>(M), static_cast<int>(N), Kb, align, sms, true);
  const int64_t tiles64 = static_cast<int64_t>(ceil_div(M, 128)) * ceil_div(N, bn);
  const int tiles = static_cast<int>(tiles64 < (int64_t(1) << 30) ? tiles64 : (int64_t(1) << 30));
  const SplitPlan pl = split_plan(tiles, ceil_div(M, 128), Kb, align, sms);
  const bool split = pl.from < tiles && tiles - pl.from <= kHeaderCounters;
  plan[0] = 0;
  plan[1] = bn;
  plan[2] = split ? tiles - pl.from : 0;
  plan[3] = split ? pl.s : 1;
  return FG8_OK;
}

size_t fg8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt) {
  if (check_gemm_shape(M, N, K, fmt) != FG8_OK) return 0;
  return gemm_workspace_need(M, N, K, fmt);
}

size_t fg8_grouped_linear_workspace_bytes(int64_t M, int64_t E, int64_t N, int64_t K, fg8_scale_fmt fmt) {
  if (check_grouped_shape(M, E, N, K, fmt) != FG8_OK) return 0;
  return grouped_ws_layout(M, E, N, K, fmt).total;
}

fg8_status fg8_grouped_row_expert(const int32_t* counts, int64_t E, int64_t cap, int32_t* row_expert,
                                  void* stream) {
  if (E <= 0 || E > 65535 || cap < 0 || E * cap > kMaxDim) return FG8_ERR_INVALID_ARG;
  if (cap == 0) return FG8_OK;
  if (counts == nullptr || row_expert == nullptr) return FG8_ERR_INVALID_ARG;
  if (cap % 128 != 0 || (reinterpret_cast<uintptr_t>(counts) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(row_expert) & 3u) != 0)
    return FG8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  return cuda_status(launch_row_expert(counts, static_cast<int>(E), static_cast<int>(cap), row_expert, dev.sms,
                                       static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_grouped_linear_prepare(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, int64_t E, int64_t N,
                                      const void* w_scale_inv, fg8_scale_fmt fmt, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (fg8_status st = check_grouped_shape(M, E, N, K, fmt); st != FG8_OK) return st;
  if (ld_x < K) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (x_bf16 == nullptr || w_scale_inv == nullptr) return FG8_ERR_INVALID_ARG;
  if (ld_x % 8 != 0 || !aligned16(x_bf16) || !aligned16(w_scale_inv)) return FG8_ERR_ALIGNMENT;
  const LinearWs L = grouped_ws_layout(M, E, N, K, fmt);
  if (fg8_status st = check_workspace(workspace, workspace_bytes, L.total); st != FG8_OK) return st;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (fg8_status st = prepare_act(x_bf16, M, K, ld_x, fmt, ws, L, dev, s); st != FG8_OK) return st;
  if (fmt == FG8_SCALE_UE8M0)  // every expert's [Nb][Kb] bytes as one stack of 128-row tiles
    return cuda_status(launch_sf_pack(static_cast<const uint8_t*>(w_scale_inv),
                                      static_cast<int>(E * ceil_div(N, 128) * 128), sfb_rows(grouped_sf_rows(E, N)),
                                      128, ceil_div(K, kGroup), 1, ws + L.wsc_off, s));
  return FG8_OK;
}

fg8_status fg8_grouped_linear_run(const int32_t* row_expert, int64_t E, const void* wq_e4m3, const void* w_scale_inv,
                                  const void* bias_bf16, void* y_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_y,
                                  fg8_scale_fmt fmt, void* workspace, size_t workspace_bytes, void* stream) {
  if (fg8_status st = check_grouped_shape(M, E, N, K, fmt); st != FG8_OK) return st;
  if (ld_y < N) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (row_expert == nullptr || wq_e4m3 == nullptr || w_scale_inv == nullptr || y_bf16 == nullptr)
    return FG8_ERR_INVALID_ARG;
  if (ld_y % 8 != 0 || !aligned16(wq_e4m3) || !aligned16(y_bf16) || (bias_bf16 != nullptr && !aligned16(bias_bf16)) ||
      !aligned16(w_scale_inv) || (reinterpret_cast<uintptr_t>(row_expert) & 3u) != 0)
    return FG8_ERR_ALIGNMENT;
  const LinearWs L = grouped_ws_layout(M, E, N, K, fmt);
  if (fg8_status st = check_workspace(workspace, workspace_bytes, L.total); st != FG8_OK) return st;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int Kb = ceil_div(K, kGroup);
  GemmArgs g{};
  g.xq = ws + L.xq_off;
  g.wq = wq_e4m3;
  g.y = y_bf16;
  g.ld_y = ld_y;
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.Kb = Kb;
  g.Kq = ceil_div(Kb, 4);
  g.bias = bias_bf16;
  g.status = reinterpret_cast<uint32_t*>(ws);
  g.wait_limit_ns = g_wait_limit_ns.load();
  g.test_stall = g_test_stall.load();
  if (fmt == FG8_SCALE_FLOAT) {
    g.xs_t = reinterpret_cast<const float*>(ws + L.xs_off);
    g.ld_s = L.ld_s;
    g.w_scale = static_cast<const float*>(w_scale_inv);
  } else {
    g.sfa = ws + L.xs_off;
    g.sfb = ws + L.wsc_off;
  }
  g.row_expert = row_expert;
  g.E = static_cast<int>(E);
  g.sfb_tiles = ceil_div(N, 128);
  return cuda_status(launch_gemm(g, fmt, dev.sms, static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_grouped_linear(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, const int32_t* row_expert,
                              int64_t E, int64_t N, const void* wq_e4m3, const void* w_scale_inv,
                              const void* bias_bf16, void* y_bf16, int64_t ld_y, fg8_scale_fmt fmt, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (fg8_status st = check_grouped_shape(M, E, N, K, fmt); st != FG8_OK) return st;
  if (ld_x < K || ld_y < N) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (x_bf16 == nullptr || row_expert == nullptr || wq_e4m3 == nullptr || w_scale_inv == nullptr || y_bf16 == nullptr)
    return FG8_ERR_INVALID_ARG;
  if (ld_x % 8 != 0 || ld_y % 8 != 0 || !aligned16(x_bf16) || !aligned16(wq_e4m3) || !aligned16(y_bf16) ||
      (bias_bf16 != nullptr && !aligned16(bias_bf16)) || !aligned16(w_scale_inv) ||
      (reinterpret_cast<uintptr_t>(row_expert) & 3u) != 0)
    return FG8_ERR_ALIGNMENT;
  if (fg8_status st = fg8_grouped_linear_prepare(x_bf16, M, K, ld_x, E, N, w_scale_inv, fmt, workspace,
                                                 workspace_bytes, stream);
      st != FG8_OK)
    return st;
  return fg8_grouped_linear_run(row_expert, E, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt, workspace,
                                workspace_bytes, stream);
}

// ---- non-default block sizes: weight_block_size = (32, 32) or (64, 64) ([zh] §八) ----
// 1 x b activation groups and b x b weight blocks.  UE8M0: the block-scaled
// MMA applies one scale per 32 K per row (a 64-block's scale on both of its
// steps); float: the GEMM promotes every b-wide slice of K in registers.
bool small_block(int block) { return block == 32 || block == 64; }

fg8_status fg8_quantize_act_block(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, void* xq_e4m3,
                                  void* x_scale, fg8_scale_fmt fmt, int block, void* stream) {
  if (block == 128) return fg8_quantize_act(x_bf16, M, K, ld_x, xq_e4m3, x_scale, fmt, stream);
  if (!small_block(block) || !fmt_ok(fmt) || M < 0 || K <= 0 || M > kMaxDim || K > kMaxDim || ld_x < K)
    return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (x_bf16 == nullptr || xq_e4m3 == nullptr || x_scale == nullptr) return FG8_ERR_INVALID_ARG;
  if (K % 16 != 0 || ld_x % 8 != 0 || !aligned16(x_bf16) || !aligned16(xq_e4m3)) return FG8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  ActQuantArgs a{};
  a.x = x_bf16;
  a.ld_x = ld_x;
  a.M = static_cast<int>(M);
  a.K = static_cast<int>(K);
  a.Kb = ceil_div(K, block);
  a.group = block;
  a.xq = static_cast<uint8_t*>(xq_e4m3);
  a.xs = x_scale;
  a.layout = kScaleRowMajor;
  return cuda_status(launch_act_quant(a, fmt, dev.sms, static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_quantize_weight_block(const void* w_bf16, int64_t N, int64_t K, int64_t ld_w, void* wq_e4m3,
                                     void* w_scale_inv, fg8_scale_fmt fmt, int block, void* stream) {
  if (block == 128) return fg8_quantize_weight(w_bf16, N, K, ld_w, wq_e4m3, w_scale_inv, fmt, stream);
  if (!small_block(block) || !fmt_ok(fmt) || N <= 0 || K <= 0 || N > kMaxDim || K > kMaxDim || ld_w < K)
    return FG8_ERR_INVALID_ARG;
  if (w_bf16 == nullptr || wq_e4m3 == nullptr || w_scale_inv == nullptr) return FG8_ERR_INVALID_ARG;
  if (ceil_div(N, block) * static_cast<int64_t>(ceil_div(K, block)) > kMaxDim / 8) return FG8_ERR_INVALID_ARG;
  if (K % 16 != 0 || ld_w % 8 != 0 || !aligned16(w_bf16) || !aligned16(wq_e4m3)) return FG8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  return cuda_status(launch_weight_quant_small(w_bf16, ld_w, static_cast<int>(N), static_cast<int>(K), block,
                                               static_cast<uint8_t*>(wq_e4m3), w_scale_inv, fmt,
                                               static_cast<cudaStream_t>(stream)));
}

// Workspace of the small-block layer: [header | xq | x scales | W scales]
//   UE8M0: x and W scale-factor tiles, one 512-byte chunk per 128 rows and
//          K-block of 128 (its four bytes per row are the four 32-K steps' scales)
//   float: x scales K-major [ceil(K/b)][ld_s] float32 (W scales read as given)
struct SmallBlockWs {
  size_t xq_off, sfa_off, sfb_off, total;
  int64_t ld_s;
};

SmallBlockWs small_block_ws_layout(int64_t M, int64_t N, int64_t K, int fmt, int block) {
  SmallBlockWs w;
  const int Kb = ceil_div(K, kGroup);
  w.xq_off = kHeaderBytes;
  w.sfa_off = align_up(w.xq_off + static_cast<size_t>(M) * K, kAlign);
  w.ld_s = kmajor_ld(M);
  if (fmt == FG8_SCALE_FLOAT) {
    w.sfb_off = align_up(w.sfa_off + static_cast<size_t>(ceil_div(K, block)) * w.ld_s * sizeof(float), kAlign);
    w.total = w.sfb_off;
  } else {
    w.sfb_off = align_up(w.sfa_off + static_cast<size_t>(ceil_div(M, 128)) * Kb * kSfChunkBytes, kAlign);
    w.total = align_up(w.sfb_off + static_cast<size_t>(sfb_rows(N) / 128) * Kb * kSfChunkBytes, kAlign);
  }
  return w;
}

size_t fg8_linear_block_workspace_bytes(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt, int block) {
  if (block == 128) return fg8_linear_workspace_bytes(M, N, K, fmt);
  if (!small_block(block) || check_gemm_shape(M, N, K, fmt) != FG8_OK) return 0;
  return small_block_ws_layout(M, N, K, fmt, block).total;
}

fg8_status fg8_linear_block(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x, const void* wq_e4m3,
                            const void* w_scale_inv, const void* bias_bf16, void* y_bf16, int64_t ld_y,
                            fg8_scale_fmt fmt, int block, void* workspace, size_t workspace_bytes, void* stream) {
  if (block == 128)
    return fg8_linear(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt, workspace,
                      workspace_bytes, stream);
  if (!small_block(block)) return FG8_ERR_INVALID_ARG;
  if (const int st = fg8::check_linear_args_status(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16,
                                                  ld_y, fmt);
      st != FG8_OK)
    return static_cast<fg8_status>(st);
  if (M == 0) return FG8_OK;
  if (ceil_div(N, block) * static_cast<int64_t>(ceil_div(K, block)) > kMaxDim / 8) return FG8_ERR_INVALID_ARG;
  const SmallBlockWs L = small_block_ws_layout(M, N, K, fmt, block);
  if (fg8_status st = check_workspace(workspace, workspace_bytes, L.total); st != FG8_OK) return st;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int Kb = ceil_div(K, kGroup);
  ActQuantArgs a{};
  a.x = x_bf16;
  a.ld_x = ld_x;
  a.M = static_cast<int>(M);
  a.K = static_cast<int>(K);
  a.Kb = ceil_div(K, block);
  a.group = block;
  a.xq = ws + L.xq_off;
  a.xs = ws + L.sfa_off;
  GemmArgs g{};
  if (fmt == FG8_SCALE_FLOAT) {
    a.layout = kScaleKMajor;
    a.ld_s = L.ld_s;
    if (fg8_status st = cuda_status(launch_act_quant(a, fmt, dev.sms, s)); st != FG8_OK) return st;
    g.xs_t = reinterpret_cast<const float*>(ws + L.sfa_off);
    g.ld_s = L.ld_s;
    g.w_scale = static_cast<const float*>(w_scale_inv);
    g.wblk = block;
  } else {
    a.layout = kScaleSfTiles;
    a.Kq = Kb;  // one chunk per K-block of 128: its four bytes are the four 32-K steps' scales
    a.M_pad = ceil_div(M, 128) * 128;
    if (fg8_status st = cuda_status(launch_act_quant(a, fmt, dev.sms, s)); st != FG8_OK) return st;
    if (fg8_status st = cuda_status(launch_sf_pack(static_cast<const uint8_t*>(w_scale_inv), static_cast<int>(N),
                                                   sfb_rows(N), block, ceil_div(K, block), block / 32,
                                                   ws + L.sfb_off, s));
        st != FG8_OK)
      return st;
    g.sfa = ws + L.sfa_off;
    g.sfb = ws + L.sfb_off;
    g.sf32 = true;
  }
  g.xq = ws + L.xq_off;
  g.wq = wq_e4m3;
  g.y = y_bf16;
  g.ld_y = ld_y;
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.Kb = Kb;
  g.Kq = Kb;
  g.bias = bias_bf16;
  g.status = reinterpret_cast<uint32_t*>(ws);
  g.wait_limit_ns = g_wait_limit_ns.load();
  g.test_stall = g_test_stall.load();
  return cuda_status(launch_gemm(g, fmt, dev.sms, s));
}

fg8_status fg8_linear_prepare(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x,
                              const void* w_scale_inv, fg8_scale_fmt fmt, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (fg8_status st = check_gemm_shape(M, N, K, fmt); st != FG8_OK) return st;
  if (ld_x < K) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (x_bf16 == nullptr || w_scale_inv == nullptr) return FG8_ERR_INVALID_ARG;
  if (ld_x % 8 != 0 || !aligned16(x_bf16)) return FG8_ERR_ALIGNMENT;
  const LinearWs L = linear_ws_layout(M, N, K, fmt);
  if (fg8_status st = check_workspace(workspace, workspace_bytes, L.total); st != FG8_OK) return st;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (fg8_status st = prepare_act(x_bf16, M, K, ld_x, fmt, ws, L, dev, s); st != FG8_OK) return st;
  if (fmt == FG8_SCALE_UE8M0)
    return cuda_status(launch_sf_pack(static_cast<const uint8_t*>(w_scale_inv), static_cast<int>(N), sfb_rows(N),
                                      128, ceil_div(K, kGroup), 1, ws + L.wsc_off, s));
  return FG8_OK;
}

fg8_status fg8_linear_run(const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16, void* y_bf16,
                          int64_t M, int64_t N, int64_t K, int64_t ld_y, fg8_scale_fmt fmt, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (fg8_status st = check_gemm_shape(M, N, K, fmt); st != FG8_OK) return st;
  if (ld_y < N) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (wq_e4m3 == nullptr || w_scale_inv == nullptr || y_bf16 == nullptr) return FG8_ERR_INVALID_ARG;
  if (ld_y % 8 != 0 || !aligned16(wq_e4m3) || !aligned16(y_bf16) || (bias_bf16 != nullptr && !aligned16(bias_bf16)) ||
      !aligned16(w_scale_inv))
    return FG8_ERR_ALIGNMENT;
  if (use_small_m(M, N)) {  // few tokens: the swap-AB split-K kernel streaming the weights
    if (fg8_status st = check_workspace(workspace, workspace_bytes, linear_workspace_need(M, N, K, fmt)); st != FG8_OK)
      return st;
    return launch_small_path(false, nullptr, 0, M, N, K, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt,
                             workspace, stream);
  }
  const LinearWs L = linear_ws_layout(M, N, K, fmt);
  if (fg8_status st = check_workspace(workspace, workspace_bytes, linear_workspace_need(M, N, K, fmt)); st != FG8_OK)
    return st;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int Kb = ceil_div(K, kGroup), Kq = ceil_div(Kb, 4);
  GemmArgs g{};
  g.xq = ws + L.xq_off;
  g.wq = wq_e4m3;
  g.y = y_bf16;
  g.ld_y = ld_y;
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.Kb = Kb;
  g.Kq = Kq;
  g.bias = bias_bf16;
  g.status = reinterpret_cast<uint32_t*>(ws);
  g.wait_limit_ns = g_wait_limit_ns.load();
  g.test_stall = g_test_stall.load();
  set_split_area(g, workspace, workspace_bytes, L.total);
  if (fmt == FG8_SCALE_FLOAT) {
    g.xs_t = reinterpret_cast<const float*>(ws + L.xs_off);
    g.ld_s = L.ld_s;
    g.w_scale = static_cast<const float*>(w_scale_inv);
  } else {
    g.sfa = ws + L.xs_off;
    g.sfb = ws + L.wsc_off;
  }
  return cuda_status(launch_gemm(g, fmt, dev.sms, static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_linear_run_chain(const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16, void* y_bf16,
                                int64_t M, int64_t N, int64_t K, int64_t ld_y, fg8_scale_fmt fmt, void* workspace,
                                size_t workspace_bytes, int64_t next_N, const void* next_w_scale_inv,
                                void* next_workspace, size_t next_workspace_bytes, void* stream) {
  if (fg8_status st = check_gemm_shape(M, N, K, fmt); st != FG8_OK) return st;
  // the next layer: K = N (its activation is this layer's output), next_N outputs
  if (fg8_status st = check_gemm_shape(M, next_N, N, fmt); st != FG8_OK) return st;
  if (ld_y < N) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (wq_e4m3 == nullptr || w_scale_inv == nullptr || y_bf16 == nullptr || next_w_scale_inv == nullptr)
    return FG8_ERR_INVALID_ARG;
  if (ld_y % 8 != 0 || !aligned16(wq_e4m3) || !aligned16(y_bf16) || (bias_bf16 != nullptr && !aligned16(bias_bf16)) ||
      !aligned16(w_scale_inv) || !aligned16(next_w_scale_inv))
    return FG8_ERR_ALIGNMENT;
  const LinearWs L = linear_ws_layout(M, N, K, fmt);
  const LinearWs Ln = linear_ws_layout(M, next_N, N, fmt);
  if (fg8_status st = check_workspace(workspace, workspace_bytes, linear_workspace_need(M, N, K, fmt)); st != FG8_OK)
    return st;
  if (fg8_status st = check_workspace(next_workspace, next_workspace_bytes, Ln.total); st != FG8_OK) return st;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* wn = static_cast<uint8_t*>(next_workspace);
  const int Kb = ceil_div(K, kGroup), Kq = ceil_div(Kb, 4);
  GemmArgs g{};
  g.xq = ws + L.xq_off;
  g.wq = wq_e4m3;
  g.y = y_bf16;
  g.ld_y = ld_y;
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.Kb = Kb;
  g.Kq = Kq;
  g.bias = bias_bf16;
  g.status = reinterpret_cast<uint32_t*>(ws);
  g.wait_limit_ns = g_wait_limit_ns.load();
  g.test_stall = g_test_stall.load();
  if (fmt == FG8_SCALE_FLOAT) {
    g.xs_t = reinterpret_cast<const float*>(ws + L.xs_off);
    g.ld_s = L.ld_s;
    g.w_scale = static_cast<const float*>(w_scale_inv);
  } else {
    g.sfa = ws + L.xs_off;
    g.sfb = ws + L.wsc_off;
  }
  g.nx_xq = wn + Ln.xq_off;
  g.nx_xs = wn + Ln.xs_off;
  g.nx_ld_s = Ln.ld_s;
  g.nx_Kq = ceil_div(ceil_div(N, kGroup), 4);
  g.nx_w_scale = next_w_scale_inv;
  g.nx_w_prep = wn + Ln.wsc_off;
  g.nx_N = static_cast<int>(next_N);
  set_split_area(g, workspace, workspace_bytes, L.total);
  return cuda_status(launch_gemm(g, fmt, dev.sms, static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_linear(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x, const void* wq_e4m3,
                      const void* w_scale_inv, const void* bias_bf16, void* y_bf16, int64_t ld_y, fg8_scale_fmt fmt,
                      void* workspace, size_t workspace_bytes, void* stream) {
  if (const int st = fg8::check_linear_args_status(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16,
                                                  ld_y, fmt);
      st != FG8_OK)
    return static_cast<fg8_status>(st);
  if (M == 0) return FG8_OK;
  if (fg8_status st = check_workspace(workspace, workspace_bytes, linear_workspace_need(M, N, K, fmt)); st != FG8_OK)
    return st;
  if (use_small_m(M, N) && use_fused_small_m(M, fmt))  // one kernel: quantize, GEMM, reduce
    return launch_small_path(true, x_bf16, ld_x, M, N, K, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt,
                             workspace, stream);
  if (fg8_status st = fg8_linear_prepare(x_bf16, M, N, K, ld_x, w_scale_inv, fmt, workspace, workspace_bytes, stream);
      st != FG8_OK)
    return st;
  return fg8_linear_run(wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt, workspace, workspace_bytes,
                        stream);
}

// ---- the activation quantization inside the tiled GEMM (fg8_linear_fused) ----
// Layout: fg8_linear's workspace, then one 32-bit flag per 128-row x 128-channel
// unit of x (ceil(M/128) * ceil(K/128)); the header's words at byte 8 hold
// the call epoch and the kernel's counters.
size_t fused_flags_off(int64_t M, int64_t N, int64_t K, int fmt) {
  return align_up(linear_workspace_need(M, N, K, fmt), kAlign);
}
size_t fused_need(int64_t M, int64_t N, int64_t K, int fmt) {
  return fused_flags_off(M, N, K, fmt) +
         align_up(static_cast<size_t>(ceil_div(M, 128)) * ceil_div(K, kGroup) * sizeof(uint32_t), kAlign);
}
// The in-kernel quantization pays off where a separate act-quant launch is
// latency-bound: short K (up to 32 K-blocks, the short-K tile configuration)
// and enough tokens for the tiled GEMM.
bool can_quantize_in_gemm(int64_t M, int64_t N, int64_t K) {
  return !use_small_m(M, N) && ceil_div(K, kGroup) <= 32;
}

size_t fg8_linear_fused_workspace_bytes(int64_t M, int64_t N, int64_t K, fg8_scale_fmt fmt) {
  if (check_gemm_shape(M, N, K, fmt) != FG8_OK) return 0;
  return fused_need(M, N, K, fmt);
}

fg8_status fg8_linear_fused(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x, const void* wq_e4m3,
                            const void* w_scale_inv, const void* bias_bf16, void* y_bf16, int64_t ld_y,
                            fg8_scale_fmt fmt, void* workspace, size_t workspace_bytes, int64_t next_N,
                            const void* next_w_scale_inv, void* next_workspace, size_t next_workspace_bytes,
                            void* stream) {
  if (const int st = fg8::check_linear_args_status(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16,
                                                  ld_y, fmt);
      st != FG8_OK)
    return static_cast<fg8_status>(st);
  const bool chain = next_w_scale_inv != nullptr;
  if (chain) {  // the next layer: K = N, next_N outputs
    if (fg8_status st = check_gemm_shape(M, next_N, N, fmt); st != FG8_OK) return st;
    if (!aligned16(next_w_scale_inv)) return FG8_ERR_ALIGNMENT;
  }
  if (M == 0) return FG8_OK;
  if (fg8_status st = check_workspace(workspace, workspace_bytes, fused_need(M, N, K, fmt)); st != FG8_OK) return st;
  const LinearWs Ln = linear_ws_layout(M, chain ? next_N : 8, N, fmt);
  if (chain)
    if (fg8_status st = check_workspace(next_workspace, next_workspace_bytes, Ln.total); st != FG8_OK) return st;
  if (!chain && use_small_m(M, N) && M <= kFusedMMax)  // few tokens: the few-token kernel quantizes x itself
    return launch_small_path(true, x_bf16, ld_x, M, N, K, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt,
                             workspace, stream);
  if (!can_quantize_in_gemm(M, N, K)) {  // long K, or 17 to 128 tokens: the separate prepare step
    if (!chain)
      return fg8_linear(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt, workspace,
                        workspace_bytes, stream);
    if (fg8_status st = fg8_linear_prepare(x_bf16, M, N, K, ld_x, w_scale_inv, fmt, workspace, workspace_bytes,
                                           stream);
        st != FG8_OK)
      return st;
    return fg8_linear_run_chain(wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt, workspace,
                                workspace_bytes, next_N, next_w_scale_inv, next_workspace, next_workspace_bytes,
                                stream);
  }
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const LinearWs L = linear_ws_layout(M, N, K, fmt);
  const int Kb = ceil_div(K, kGroup), Kq = ceil_div(Kb, 4);
  GemmArgs g{};
  g.xq = ws + L.xq_off;
  g.wq = wq_e4m3;
  g.y = y_bf16;
  g.ld_y = ld_y;
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.Kb = Kb;
  g.Kq = Kq;
  g.bias = bias_bf16;
  g.status = reinterpret_cast<uint32_t*>(ws);
  g.wait_limit_ns = g_wait_limit_ns.load();
  g.test_stall = g_test_stall.load();
  if (fmt == FG8_SCALE_FLOAT) {
    g.xs_t = reinterpret_cast<const float*>(ws + L.xs_off);
    g.ld_s = L.ld_s;
    g.w_scale = static_cast<const float*>(w_scale_inv);
  } else {
    g.sfa = ws + L.xs_off;
    g.sfb = ws + L.wsc_off;
    g.qwsc = w_scale_inv;
  }
  g.qx = x_bf16;
  g.ld_qx = ld_x;
  g.qflags = reinterpret_cast<uint32_t*>(ws + fused_flags_off(M, N, K, fmt));
  // (no split-K tail: these short-K shapes never split, in fg8_linear either)
  g.qepoch = reinterpret_cast<uint32_t*>(ws + kHeaderEpochOffset);
  if (chain) {
    uint8_t* wn = static_cast<uint8_t*>(next_workspace);
    g.nx_xq = wn + Ln.xq_off;
    g.nx_xs = wn + Ln.xs_off;
    g.nx_ld_s = Ln.ld_s;
    g.nx_Kq = ceil_div(ceil_div(N, kGroup), 4);
    g.nx_w_scale = next_w_scale_inv;
    g.nx_w_prep = wn + Ln.wsc_off;
    g.nx_N = static_cast<int>(next_N);
  }
  return cuda_status(launch_gemm(g, fmt, dev.sms, static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_gemm_prequant(const void* xq_e4m3, const void* x_scale, const void* wq_e4m3, const void* w_scale_inv,
                             const void* bias_bf16, void* y_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_y,
                             fg8_scale_fmt fmt, void* workspace, size_t workspace_bytes, void* stream) {
  if (fg8_status st = check_gemm_shape(M, N, K, fmt); st != FG8_OK) return st;
  if (ld_y < N) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (xq_e4m3 == nullptr || x_scale == nullptr || wq_e4m3 == nullptr || w_scale_inv == nullptr || y_bf16 == nullptr)
    return FG8_ERR_INVALID_ARG;
  if (ld_y % 8 != 0 || !aligned16(xq_e4m3) || !aligned16(wq_e4m3) || !aligned16(y_bf16) ||
      (bias_bf16 != nullptr && !aligned16(bias_bf16)))
    return FG8_ERR_ALIGNMENT;
  const GemmWs L = gemm_ws_layout(M, N, K, fmt);
  if (fg8_status st = check_workspace(workspace, workspace_bytes, gemm_workspace_need(M, N, K, fmt)); st != FG8_OK)
    return st;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int Kb = ceil_div(K, kGroup), Kq = ceil_div(Kb, 4);

  GemmArgs g{};
  g.xq = xq_e4m3;
  g.wq = wq_e4m3;
  g.y = y_bf16;
  g.ld_y = ld_y;
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.Kb = Kb;
  g.Kq = Kq;
  g.bias = bias_bf16;
  g.status = reinterpret_cast<uint32_t*>(ws);
  g.wait_limit_ns = g_wait_limit_ns.load();
  g.test_stall = g_test_stall.load();
  set_split_area(g, workspace, workspace_bytes, L.total);
  if (fmt == FG8_SCALE_FLOAT) {
    if (fg8_status st = cuda_status(launch_xs_transpose(static_cast<const float*>(x_scale), static_cast<int>(M), Kb,
                                                        L.ld_s, reinterpret_cast<float*>(ws + L.xs_off), s));
        st != FG8_OK)
      return st;
    g.xs_t = reinterpret_cast<const float*>(ws + L.xs_off);
    g.ld_s = L.ld_s;
    g.w_scale = static_cast<const float*>(w_scale_inv);
  } else {
    if (fg8_status st = cuda_status(launch_sf_pack(static_cast<const uint8_t*>(x_scale), static_cast<int>(M),
                                                   (M + 127) / 128 * 128, 1, Kb, 1, ws + L.xs_off, s));
        st != FG8_OK)
      return st;
    if (fg8_status st = cuda_status(launch_sf_pack(static_cast<const uint8_t*>(w_scale_inv), static_cast<int>(N),
                                                   sfb_rows(N), 128, Kb, 1, ws + L.wsc_off, s));
        st != FG8_OK)
      return st;
    g.sfa = ws + L.xs_off;
    g.sfb = ws + L.wsc_off;
  }
  return cuda_status(launch_gemm(g, fmt, dev.sms, s));
}

fg8_status fg8_quantize_act_static(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, const float* act_scale,
                                   void* xq_e4m3, void* x_scale, void* stream) {
  if (M < 0 || K <= 0 || M > kMaxDim || K > kMaxDim || ld_x < K) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (x_bf16 == nullptr || act_scale == nullptr || xq_e4m3 == nullptr || x_scale == nullptr) return FG8_ERR_INVALID_ARG;
  if (K % 16 != 0 || ld_x % 8 != 0 || !aligned16(x_bf16) || !aligned16(xq_e4m3) ||
      (reinterpret_cast<uintptr_t>(act_scale) & 3u) != 0)
    return FG8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  ActQuantArgs a{};
  a.x = x_bf16;
  a.ld_x = ld_x;
  a.M = static_cast<int>(M);
  a.K = static_cast<int>(K);
  a.Kb = ceil_div(K, kGroup);
  a.xq = static_cast<uint8_t*>(xq_e4m3);
  a.xs = x_scale;
  a.layout = kScaleRowMajor;
  a.static_scale = act_scale;
  return cuda_status(launch_act_quant(a, FG8_SCALE_FLOAT, dev.sms, static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_linear_static(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x, const float* act_scale,
                             const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16, void* y_bf16,
                             int64_t ld_y, void* workspace, size_t workspace_bytes, void* stream) {
  const fg8_scale_fmt fmt = FG8_SCALE_FLOAT;
  if (fg8_status st = check_gemm_shape(M, N, K, fmt); st != FG8_OK) return st;
  if (ld_x < K || ld_y < N) return FG8_ERR_INVALID_ARG;
  if (M == 0) return FG8_OK;
  if (x_bf16 == nullptr || act_scale == nullptr || wq_e4m3 == nullptr || w_scale_inv == nullptr || y_bf16 == nullptr)
    return FG8_ERR_INVALID_ARG;
  if (ld_x % 8 != 0 || ld_y % 8 != 0 || !aligned16(x_bf16) || !aligned16(wq_e4m3) || !aligned16(y_bf16) ||
      (bias_bf16 != nullptr && !aligned16(bias_bf16)) || !aligned16(w_scale_inv) ||
      (reinterpret_cast<uintptr_t>(act_scale) & 3u) != 0)
    return FG8_ERR_ALIGNMENT;
  const LinearWs L = linear_ws_layout(M, N, K, fmt);
  // the whole workspace the GEMM step needs (few tokens: split-K partials
  // too), checked before the quantization is enqueued
  if (fg8_status st = check_workspace(workspace, workspace_bytes, linear_workspace_need(M, N, K, fmt)); st != FG8_OK)
    return st;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  ActQuantArgs a{};
  a.x = x_bf16;
  a.ld_x = ld_x;
  a.M = static_cast<int>(M);
  a.K = static_cast<int>(K);
  a.Kb = ceil_div(K, kGroup);
  a.xq = ws + L.xq_off;
  a.xs = ws + L.xs_off;
  a.layout = kScaleKMajor;
  a.ld_s = L.ld_s;
  a.static_scale = act_scale;
  if (fg8_status st = cuda_status(launch_act_quant(a, fmt, dev.sms, static_cast<cudaStream_t>(stream))); st != FG8_OK)
    return st;
  return fg8_linear_run(wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt, workspace, workspace_bytes,
                        stream);
}

fg8_status fg8_dequantize_weight(const void* wq_e4m3, int64_t N, int64_t K, const void* w_scale_inv,
                                 fg8_scale_fmt fmt, void* w_bf16, int64_t ld_w, void* stream) {
  if (!fmt_ok(fmt) || N <= 0 || K <= 0 || N > kMaxDim || K > kMaxDim || ld_w < K) return FG8_ERR_INVALID_ARG;
  if (N * K > (int64_t(1) << 40)) return FG8_ERR_INVALID_ARG;
  if (wq_e4m3 == nullptr || w_scale_inv == nullptr || w_bf16 == nullptr) return FG8_ERR_INVALID_ARG;
  if (K % 16 != 0 || ld_w % 8 != 0 || !aligned16(wq_e4m3) || !aligned16(w_bf16)) return FG8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  return cuda_status(launch_dequant_weight(static_cast<const uint8_t*>(wq_e4m3), static_cast<int>(N),
                                           static_cast<int>(K), w_scale_inv, fmt, static_cast<uint16_t*>(w_bf16),
                                           ld_w, dev.sms, static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_scale_to_ue8m0(const void* scale_f32, int64_t n, void* scale_e8m0, uint32_t* invalid_count,
                              void* stream) {
  if (n < 0) return FG8_ERR_INVALID_ARG;
  if (n == 0) return FG8_OK;
  if (scale_f32 == nullptr || scale_e8m0 == nullptr) return FG8_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scale_f32) & 3u) != 0 || (reinterpret_cast<uintptr_t>(invalid_count) & 3u) != 0)
    return FG8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (fg8_status st = current_device(&dev); st != FG8_OK) return st;
  return cuda_status(launch_scale_to_e8m0(static_cast<const float*>(scale_f32), n, static_cast<uint8_t*>(scale_e8m0),
                                          invalid_count, dev.sms, static_cast<cudaStream_t>(stream)));
}

fg8_status fg8_check_device_status(void* workspace, void* stream) {
  if (workspace == nullptr) return FG8_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return FG8_ERR_CUDA;
  }
  if (word != 0) {
    // a kernel gave up mid-way: its split-K counters may be left counting,
    // so the header starts from zero again -- all but the epoch word of the
    // in-GEMM quantization, which only ever advances
    uint8_t* h = static_cast<uint8_t*>(workspace);
    if (cudaMemsetAsync(h + kHeaderEpochOffset + 4, 0, kHeaderBytes - kHeaderEpochOffset - 4, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
      cudaGetLastError();
      return FG8_ERR_CUDA;
    }
  }
  return word == 0 ? FG8_OK : static_cast<fg8_status>(word);
}

}  // extern "C"
