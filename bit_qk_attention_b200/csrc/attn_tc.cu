// Placeholder of the tcgen05 kernel translation unit (filled in next).
#include "common.cuh"
#include "kernels.h"

namespace binattn {

__device__ int g_device_status = 0;

bool attn_tc_supported(const AttnParams&) { return false; }

cudaError_t launch_attn_tc(const AttnParams&, cudaStream_t) { return cudaErrorNotSupported; }

cudaError_t read_and_clear_device_status(int* value, cudaStream_t s) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(value, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return e;
  const int zero = 0;
  if ((e = cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s)) != cudaSuccess)
    return e;
  return cudaStreamSynchronize(s);
}

}  // namespace binattn
