// ba_attention_fwd_noalloc: the whole forward pass with the library's own scratch memory.
//
// Who needs this: some callers cannot give the library a workspace. A plugin called by a
// host framework may receive only its input and output buffers and no allocator handle; a
// serving runtime may plan all device memory at start-up and forbid allocation afterwards,
// because cudaMalloc can synchronize the device and bypasses the host's own allocator. For
// them this entry point runs the same kernels as ba_attention_fwd, with the workspace taken
// from a fixed array in the library's device memory instead of from the caller.
//
// Costs and rules:
//   * Every GPU that loads this library reserves kScratchBytes of device memory for the
//     array, until the process exits.
//   * All calls share the one array. Two calls that may run at the same time on the GPU
//     (different streams without ordering between them) race on it; callers must order them.
//   * The array keeps whatever the last call left in it. Nothing in it has to start at zero:
//     every region is fully written by the first kernels of a call before any kernel reads it.
//   * The first call on each device looks up the array's device address (cudaGetSymbolAddress,
//     with that device current) and caches it; make that first call before any stream capture.
//     The cache assumes the device's primary context lives as long as the process: after a
//     cudaDeviceReset the library's device memory is reloaded elsewhere and the cached address
//     is stale, so a process that resets a device must not call this entry point afterwards.
//   * Problems whose workspace exceeds kScratchBytes are refused with BA_ERR_WORKSPACE before
//     anything is launched. Nothing here calls cudaMalloc, cudaFree or another allocating routine.
#include <cuda_runtime.h>

#include <mutex>

#include "binattn.h"

namespace {

constexpr size_t kScratchBytes = size_t{32} << 20;  // 32 MiB, BA_NOALLOC_SCRATCH_BYTES in binattn.h
static_assert(kScratchBytes == BA_NOALLOC_SCRATCH_BYTES, "header and library disagree on the limit");

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" ba_status ba_attention_fwd_noalloc(const void* q, const void* k, const void* v, ba_dtype dt, int B,
                                              int H, int N, int d, const ba_bias* bias, float softmax_scale,
                                              void* o, ba_dtype o_dt, int32_t* dbg_logits, void* stream) {
  const size_t need = ba_workspace_bytes(B, H, N, d);
  if (need == static_cast<size_t>(-1)) return (B < 0 || H < 0 || N < 0) ? BA_ERR_INVALID_ARG : BA_ERR_UNSUPPORTED;
  if (need > kScratchBytes) return BA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0 && scratch_address(&scratch) != cudaSuccess) return BA_ERR_CUDA;
  return ba_attention_fwd(q, k, v, dt, B, H, N, d, bias, softmax_scale, o, o_dt, scratch, kScratchBytes,
                          dbg_logits, stream);
}
