// Streaming kernels of the BinaryAttention forward pass (sm_100a):
//   prep_kernel     — sign bits + per-chunk sum |x| of q and k, per-chunk channel max |v|;
//   finalize_kernel — mu = sum / (N d) per (b, h); per-channel V scales;
//   quant_kernel    — V -> int8 rows with the per-channel inverse scale.
// Sign binarisation and mu: gist.science/zh technical summary 2.2(1) (s_i = mu_q sign(q_i),
// mu the mean along token and channel axes). Channel-aware 8-bit V: gist.science/zh 2.2(3),
// gist.science/nl Methodologie 2.
//
// All three are HBM-bound: each 128-token chunk of one (b, h) slice is one CTA, read with
// 16-byte non-allocating loads, fully coalesced (consecutive threads read consecutive
// 16-byte pieces of consecutive rows). Reductions are deterministic: fixed-order in-CTA
// trees, then fixed-order sums over chunks.
#include "common.cuh"
#include "kernels.h"

namespace binattn {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxIter = 8;  // ceil(kPrepTokens / rows_per_pass) for d/8 <= 16

// Sum over the CTA in double. Every |x| of a 16-bit input is exact in double and the
// partial sums stay exact while they are below 2^53 units of the smallest input's ulp, so
// the result does not depend on the summation order in practice (the CPU reference sums
// sequentially in double and rounds the mean to fp32 the same way).
__device__ __forceinline__ double block_sum(double v, double* sred) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sred[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0) {
    for (int w = 0; w < kThreads / 32; ++w) t += sred[w];
  }
  return t;  // valid in thread 0
}

// Vector path: d % 8 == 0, so every row is a whole number of 16-byte pieces.
template <typename T>
__device__ void prep_pack_vec(const PrepJob& job, const PrepDims& g, int64_t bh, int chunk) {
  __shared__ __align__(16) uint8_t sbits[kPrepTokens][16];
  __shared__ double sred[kThreads / 32];
  const int tok0 = chunk * kPrepTokens;
  const int ntok = min(kPrepTokens, g.N - tok0);
  const int tpr = g.d >> 3;
  const int rpp = kThreads / tpr;
  const int sub = threadIdx.x % tpr, r0 = threadIdx.x / tpr;
  reinterpret_cast<uint2*>(&sbits[0][0])[threadIdx.x] = make_uint2(0u, 0u);
  __syncthreads();
  const char* base = reinterpret_cast<const char*>(job.src) + ((bh * g.N + tok0) * g.d) * 2;
  uint4 u[kMaxIter];
#pragma unroll
  for (int it = 0; it < kMaxIter; ++it) {
    const int r = r0 + it * rpp;
    if (r0 < rpp && r < ntok) u[it] = ldg_stream(base + (static_cast<int64_t>(r) * g.d + sub * 8) * 2);
  }
  double acc = 0.0;
#pragma unroll
  for (int it = 0; it < kMaxIter; ++it) {
    const int r = r0 + it * rpp;
    if (r0 < rpp && r < ntok) {
      float f[8];
      unpack8<T>(u[it], f);
      uint32_t byte = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        byte |= (f[e] < 0.0f ? 1u : 0u) << e;
        acc += static_cast<double>(fabsf(f[e]));
      }
      sbits[r][sub] = static_cast<uint8_t>(byte);
    }
  }
  __syncthreads();
  if (threadIdx.x < ntok)
    reinterpret_cast<uint4*>(job.bits)[bh * g.N + tok0 + threadIdx.x] =
        reinterpret_cast<const uint4*>(&sbits[0][0])[threadIdx.x];
  const double tot = block_sum(acc, sred);
  if (threadIdx.x == 0) job.part_sum[bh * g.nchunk + chunk] = tot;
}

template <typename T>
__device__ void prep_amax_vec(const PrepJob& job, const PrepDims& g, int64_t bh, int chunk) {
  __shared__ float sred[kThreads * 8];
  const int tok0 = chunk * kPrepTokens;
  const int ntok = min(kPrepTokens, g.N - tok0);
  const int tpr = g.d >> 3;
  const int rpp = kThreads / tpr;
  const int sub = threadIdx.x % tpr, r0 = threadIdx.x / tpr;
  const char* base = reinterpret_cast<const char*>(job.src) + ((bh * g.N + tok0) * g.d) * 2;
  uint4 u[kMaxIter];
#pragma unroll
  for (int it = 0; it < kMaxIter; ++it) {
    const int r = r0 + it * rpp;
    if (r0 < rpp && r < ntok) u[it] = ldg_stream(base + (static_cast<int64_t>(r) * g.d + sub * 8) * 2);
  }
  float mx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = 0.0f;
#pragma unroll
  for (int it = 0; it < kMaxIter; ++it) {
    const int r = r0 + it * rpp;
    if (r0 < rpp && r < ntok) {
      float f[8];
      unpack8<T>(u[it], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], fabsf(f[e]));
    }
  }
  if (r0 < rpp) {
#pragma unroll
    for (int e = 0; e < 8; ++e) sred[r0 * g.d + sub * 8 + e] = mx[e];
  }
  __syncthreads();
  const int rows = min(rpp, ntok);
  for (int c = threadIdx.x; c < g.dp; c += kThreads) {
    float m = 0.0f;
    if (c < g.d)
      for (int rr = 0; rr < rows; ++rr) m = fmaxf(m, sred[rr * g.d + c]);
    job.part[(bh * g.nchunk + chunk) * g.dp + c] = m;
  }
}

// Scalar path for d % 8 != 0 (rows not made of whole 16-byte pieces).
template <typename T>
__device__ void prep_scalar(const PrepJob& job, const PrepDims& g, int64_t bh, int chunk) {
  __shared__ uint32_t swords[kPrepTokens][kSignWords];
  __shared__ int smax[128];
  __shared__ double sred[kThreads / 32];
  const int tok0 = chunk * kPrepTokens;
  const int ntok = min(kPrepTokens, g.N - tok0);
  for (int e = threadIdx.x; e < kPrepTokens * kSignWords; e += kThreads) (&swords[0][0])[e] = 0u;
  if (threadIdx.x < 128) smax[threadIdx.x] = 0;
  __syncthreads();
  const T* base = reinterpret_cast<const T*>(job.src) + (bh * g.N + tok0) * g.d;
  double acc = 0.0;
  for (int e = threadIdx.x; e < ntok * g.d; e += kThreads) {
    const int r = e / g.d, c = e - r * g.d;
    const float f = load1<T>(base + e);
    if (job.kind == kJobPack) {
      if (f < 0.0f) atomicOr(&swords[r][c >> 5], 1u << (c & 31));
      acc += static_cast<double>(fabsf(f));
    } else {
      atomicMax(&smax[c], __float_as_int(fabsf(f)));  // non-negative floats order like ints
    }
  }
  __syncthreads();
  if (job.kind == kJobPack) {
    if (threadIdx.x < ntok)
      reinterpret_cast<uint4*>(job.bits)[bh * g.N + tok0 + threadIdx.x] =
          reinterpret_cast<const uint4*>(&swords[0][0])[threadIdx.x];
    const double tot = block_sum(acc, sred);
    if (threadIdx.x == 0) job.part_sum[bh * g.nchunk + chunk] = tot;
  } else {
    for (int c = threadIdx.x; c < g.dp; c += kThreads)
      job.part[(bh * g.nchunk + chunk) * g.dp + c] = (c < g.d) ? __int_as_float(smax[c]) : 0.0f;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) prep_kernel(PrepParams p) {
  const int64_t cta = blockIdx.x;
  const int64_t bh = cta / p.g.nchunk;
  const int chunk = static_cast<int>(cta - bh * p.g.nchunk);
  const PrepJob job = (blockIdx.y == 0) ? p.job[0] : (blockIdx.y == 1 ? p.job[1] : p.job[2]);
  if ((p.g.d & 7) == 0) {
    if (job.kind == kJobPack)
      prep_pack_vec<T>(job, p.g, bh, chunk);
    else
      prep_amax_vec<T>(job, p.g, bh, chunk);
  } else {
    prep_scalar<T>(job, p.g, bh, chunk);
  }
}

__global__ void __launch_bounds__(128) finalize_kernel(FinalizeParams p) {
  const int64_t bh = blockIdx.x;
  const PrepDims& g = p.g;
  if (threadIdx.x < 32) {
    for (int j = 0; j < p.npack; ++j) {
      // Fixed-order double sum of the chunk partials.
      double s = 0.0;
      for (int c = threadIdx.x; c < g.nchunk; c += 32) s += p.part_mu[j][bh * g.nchunk + c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (threadIdx.x == 0) p.mu[j][bh] = static_cast<float>(s / (static_cast<double>(g.N) * g.d));
    }
  }
  if (p.part_amax != nullptr) {
    for (int c = threadIdx.x; c < g.dp; c += blockDim.x) {
      float m = 0.0f;
      for (int ch = 0; ch < g.nchunk; ++ch) m = fmaxf(m, p.part_amax[(bh * g.nchunk + ch) * g.dp + c]);
      const bool live = (c < g.d) && (m > 0.0f);
      p.inv[bh * g.dp + c] = live ? __fdiv_rn(127.0f, m) : 0.0f;
      if (c < g.d) p.v_scale[bh * g.d + c] = live ? __fdiv_rn(m, 127.0f) : 0.0f;
    }
  }
}

__device__ __forceinline__ uint32_t quant4(const float* f, const float* inv) {
  uint32_t w = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    int q = __float2int_rn(__fmul_rn(f[e], inv[e]));
    q = max(-127, min(127, q));
    w |= (static_cast<uint32_t>(q) & 0xffu) << (8 * e);
  }
  return w;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) quant_kernel(QuantParams p) {
  __shared__ float sinv[128];
  const int64_t cta = blockIdx.x;
  const int64_t bh = cta / p.g.nchunk;
  const int chunk = static_cast<int>(cta - bh * p.g.nchunk);
  const int tok0 = chunk * kPrepTokens;
  const int ntok = min(kPrepTokens, p.g.N - tok0);
  const int d = p.g.d, dp = p.g.dp;
  if (threadIdx.x < dp) sinv[threadIdx.x] = p.inv[bh * dp + threadIdx.x];
  __syncthreads();
  int8_t* out = p.vq + (bh * p.g.N + tok0) * dp;
  if ((d & 7) == 0) {
    const int opr = dp >> 3;  // 8-byte output pieces per row
    const int rpp = kThreads / opr;
    const int sub = threadIdx.x % opr, r0 = threadIdx.x / opr;
    if (r0 >= rpp) return;
    const char* base = reinterpret_cast<const char*>(p.v) + ((bh * p.g.N + tok0) * d) * 2;
    for (int r = r0; r < ntok; r += rpp) {
      uint2 w = make_uint2(0u, 0u);
      if (sub * 8 < d) {
        const uint4 u = ldg_stream(base + (static_cast<int64_t>(r) * d + sub * 8) * 2);
        float f[8];
        unpack8<T>(u, f);
        w.x = quant4(f, &sinv[sub * 8]);
        w.y = quant4(f + 4, &sinv[sub * 8 + 4]);
      }
      *reinterpret_cast<uint2*>(out + static_cast<int64_t>(r) * dp + sub * 8) = w;
    }
  } else {
    const T* base = reinterpret_cast<const T*>(p.v) + (bh * p.g.N + tok0) * d;
    for (int e = threadIdx.x; e < ntok * dp; e += kThreads) {
      const int r = e / dp, c = e - r * dp;
      int q = 0;
      if (c < d) {
        q = __float2int_rn(__fmul_rn(load1<T>(base + static_cast<int64_t>(r) * d + c), sinv[c]));
        q = max(-127, min(127, q));
      }
      out[e] = static_cast<int8_t>(q);
    }
  }
}

}  // namespace

cudaError_t launch_prep(const PrepParams& p, int dt, int njobs, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(p.g.BH * p.g.nchunk), static_cast<unsigned>(njobs));
  if (dt == BA_F16)
    prep_kernel<__half><<<grid, kThreads, 0, s>>>(p);
  else
    prep_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const FinalizeParams& p, cudaStream_t s) {
  finalize_kernel<<<static_cast<unsigned>(p.g.BH), 128, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quant(const QuantParams& p, int dt, cudaStream_t s) {
  const unsigned grid = static_cast<unsigned>(p.g.BH * p.g.nchunk);
  if (dt == BA_F16)
    quant_kernel<__half><<<grid, kThreads, 0, s>>>(p);
  else
    quant_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace binattn
