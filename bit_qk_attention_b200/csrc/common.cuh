// Shared device helpers of the BinaryAttention library (CUDA, sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "binattn.h"

namespace binattn {

constexpr int kSignWords = 4;     // 128 sign bits per token row
constexpr int kKvBlock = 128;     // key block of the online softmax (the P codes depend on it)
constexpr int kPrepTokens = 128;  // tokens per CTA in the streaming kernels

__host__ __device__ inline int v_row_bytes(int d) { return (d + 15) & ~15; }
__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Eight 16-bit floats held in a uint4 -> eight fp32 values (exact widening).
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& u, float f[8]);

template <>
__device__ __forceinline__ void unpack8<__half>(const uint4& u, float f[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h;
    *reinterpret_cast<uint32_t*>(&h) = w[i];
    const float2 p = __half22float2(h);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
  }
}

template <>
__device__ __forceinline__ void unpack8<__nv_bfloat16>(const uint4& u, float f[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // bf16 -> fp32 is a 16-bit left shift of the bit pattern.
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <typename T>
__device__ __forceinline__ float load1(const T* p);
template <>
__device__ __forceinline__ float load1<__half>(const __half* p) { return __half2float(*p); }
template <>
__device__ __forceinline__ float load1<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Programmatic dependent launch. A kernel launched with programmatic stream serialization may
// start while the kernel before it in the stream is still running: grid_dependency_wait()
// returns once that kernel has completed and its writes are visible (at once when there is no
// such kernel). allow_dependents() lets the next kernel start before this one completes.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Output store of one fp32 value in the requested dtype.
__device__ __forceinline__ void store_out(void* o, int64_t idx, float val, int o_dt) {
  if (o_dt == BA_F32) {
    reinterpret_cast<float*>(o)[idx] = val;
  } else if (o_dt == BA_F16) {
    reinterpret_cast<__half*>(o)[idx] = __float2half_rn(val);
  } else {
    reinterpret_cast<__nv_bfloat16*>(o)[idx] = __float2bfloat16_rn(val);
  }
}

// Bias parameters as the kernels see them.
struct BiasParams {
  int kind;
  const float* data;
  int64_t batch_stride;
  int grid_h, grid_w, table_h, table_w, n_prefix;
};

__device__ __forceinline__ float bias_at(const BiasParams& bz, int64_t b, int64_t h, int64_t N,
                                         int64_t i, int64_t j) {
  if (bz.kind == BA_BIAS_DENSE) return __ldg(bz.data + b * bz.batch_stride + (h * N + i) * N + j);
  if (bz.kind == BA_BIAS_RELPOS2D) {
    if (i < bz.n_prefix || j < bz.n_prefix) return 0.0f;
    const int ti = static_cast<int>(i) - bz.n_prefix, tj = static_cast<int>(j) - bz.n_prefix;
    const int yi = ti / bz.grid_w, xi = ti - yi * bz.grid_w;
    const int yj = tj / bz.grid_w, xj = tj - yj * bz.grid_w;
    const int64_t tsize = static_cast<int64_t>(2 * bz.table_h - 1) * (2 * bz.table_w - 1);
    return __ldg(bz.data + h * tsize + static_cast<int64_t>(yi - yj + bz.table_h - 1) * (2 * bz.table_w - 1) +
                 (xi - xj + bz.table_w - 1));
  }
  return 0.0f;
}

// Operands of the fused step.
struct AttnParams {
  const uint32_t* bits_q;
  const uint32_t* bits_k;
  const float* mu_q;
  const float* mu_k;
  const int8_t* vq;
  const float* v_scale;
  int B, H, N, d, dp;
  BiasParams bias;
  float softmax_scale;  // already resolved (> 0)
  void* o;
  int o_dt;
  int32_t* dbg_logits;
  uint8_t* dbg_p;   // debug: the 8-bit codes P_ij [B][H][N][N], or null
  int p_check_all;  // recompute every near-tie code exactly, not only where it could matter
};

}  // namespace binattn
