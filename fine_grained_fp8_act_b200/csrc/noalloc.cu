// noalloc.cu -- fg8_linear for callers that cannot allocate device memory.
//
// fg8_linear needs a caller-provided device workspace.  Some callers have no
// way to provide one: a host framework that owns every byte of device memory
// through its own pool and forbids other allocations, or latency-critical code
// that must never call cudaMalloc (which can synchronize the whole device).
// fg8_linear_noalloc serves them with a fixed scratch buffer that lives in
// this library's own device memory: a file-scope __device__ array of
// kNoAllocScratchBytes, created when the module is loaded on a device and
// kept until the process exits.  Nothing here calls cudaMalloc, cudaFree or
// any allocating routine.

#include <cuda_runtime.h>

#include <mutex>

#include "fg8.h"
#include "fg8_internal.h"

namespace {

// 64 MiB: enough for, e.g., 8192 tokens x 7168 input channels, or the ESM-2
// and Llama-3-8B shapes up to 4096 tokens (the workspace is M*K bytes of
// quantized activations plus their scales and the weight scales, and up to
// 148 x 128 KiB of split-K partials for the tiled GEMM's last wave).
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

// The scratch.  In host code this name is only a stand-in for the device
// symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (this may load the module, so it must not run inside a stream
// capture).  Returns nullptr on failure.
void* scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" fg8_status fg8_linear_noalloc(const void* x_bf16, int64_t M, int64_t N, int64_t K, int64_t ld_x,
                                         const void* wq_e4m3, const void* w_scale_inv, const void* bias_bf16,
                                         void* y_bf16, int64_t ld_y, fg8_scale_fmt fmt, void* stream) {
  // fg8_linear's own argument checks come first, so a bad call returns its
  // status without touching the scratch or the device
  if (const int st = fg8::check_linear_args_status(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16,
                                                  ld_y, fmt);
      st != FG8_OK)
    return static_cast<fg8_status>(st);
  if (M == 0) return FG8_OK;
  const size_t need = fg8_linear_workspace_bytes(M, N, K, fmt);
  if (need == 0 || need > kNoAllocScratchBytes) return FG8_ERR_WORKSPACE;  // too large for the fixed scratch
  void* scratch = scratch_for_current_device();
  if (scratch == nullptr) return FG8_ERR_CUDA;
  // The scratch keeps the previous call's bytes; the only part that must
  // start at zero is the header at its head (status word, split-K counters).
  if (cudaMemsetAsync(scratch, 0, fg8::kWorkspaceHeaderBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FG8_ERR_CUDA;
  }
  return fg8_linear(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt, scratch,
                    kNoAllocScratchBytes, stream);
}
