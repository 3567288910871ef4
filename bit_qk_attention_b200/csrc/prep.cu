// Streaming kernels of the BinaryAttention forward pass (sm_100a):
//   prep_slice_kernel — short slices (d % 8 == 0, d >= 32, many slices): one CTA per (slice,
//                       tensor) writes the sign bits and mu of q and k, or the scales and int8
//                       rows of v, in one launch;
//   prep_warp_kernel  — otherwise, rows of whole 16-byte pieces: one warp per 128-token chunk,
//                       sign bits + per-chunk sum |x| of q and k; one CTA per eight chunks of
//                       v, their channel max |v|;
//   prep_kernel       — d % 8 != 0: a CTA per (tensor, chunk), the same per-chunk partials;
//   quant_kernel      — V -> int8 rows, 128-1024 tokens per CTA; each CTA reduces its slice's
//                       channel-max partials to the inverse scales itself, and a slice's first
//                       CTA writes mu of q and k and the V scales (no separate finalize launch);
//   finalize_kernel   — mu = sum / (N d) per (b, h), for sign packing on its own.
// Sign binarisation and mu: gist.science/zh technical summary 2.2(1) (s_i = mu_q sign(q_i),
// mu averaging |x| over every token and channel of the slice). Channel-aware 8-bit V: gist.science/zh 2.2(3),
// gist.science/nl Methodologie 2.
//
// All are HBM-bound: 16-byte loads, fully coalesced (consecutive threads read consecutive
// 16-byte pieces of consecutive rows), many in flight per thread. The |x| sums are taken in
// double, where every partial sum of 16-bit magnitudes is exact, so they do not depend on the
// summation order.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace binattn {

namespace {

constexpr int kThreads = 256;

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
  prep_scalar<T>(job, p.g, bh, chunk);
}

// A channel gets codes when its maximum is nonzero and 127 / amax is a finite float. A bf16
// channel with amax below 127 / FLT_MAX (about 3.7e-37) would get inv = +inf, codes of inf and
// NaN: it is treated as a zero channel instead (codes 0, scale 0), as the definition reads.
__device__ __forceinline__ bool channel_live(float amax, float inv) {
  return amax > 0.0f && inv <= 3.402823466e38f;
}

__global__ void __launch_bounds__(32) finalize_kernel(FinalizeParams p) {
  const int64_t bh = blockIdx.x;
  const PrepDims& g = p.g;
  for (int j = 0; j < p.npack; ++j) {
    double s = 0.0;
    for (int c = threadIdx.x; c < g.nchunk; c += 32) s += p.part_mu[j][bh * g.nchunk + c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) p.mu[j][bh] = static_cast<float>(s / (static_cast<double>(g.N) * g.d));
  }
}

// Four int8 codes rne(v * inv), packed. The product is rounded to fp32 first (as the definition
// states), then to the nearest integer, ties to even, by adding 1.5 * 2^23: the integer lands in
// the low mantissa bits, whose low byte is its two's-complement byte. The clamp to [-127, 127]
// never acts on finite inputs: inv = rn(127 / amax) is finite (channel_live) and |v| <= amax
// give |rn(v * inv)| <= 127 (1 + 2^-24)^2 < 127.5; a dead channel has inv = 0 and codes 0.
__device__ __forceinline__ uint32_t quant4(const float* f, const float* inv) {
  uint32_t y[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) y[e] = __float_as_uint(__fadd_rn(__fmul_rn(f[e], inv[e]), 12582912.0f));
  return __byte_perm(__byte_perm(y[0], y[1], 0x0040), __byte_perm(y[2], y[3], 0x0040), 0x5410);
}

constexpr int kQuantBatch = 8;  // passes of the quantiser whose loads are in flight together

// Loads of one batch of V pieces: row r0 + j rpp + rp, piece sub, for j < kQuantBatch.
__device__ __forceinline__ void quant_load(uint4 (&u)[kQuantBatch], const char* base, int r0, int ntok, int d,
                                           int rpp, int rp, int sub, bool on) {
#pragma unroll
  for (int j = 0; j < kQuantBatch; ++j) {
    const int r = r0 + j * rpp + rp;
    if (on && r < ntok) u[j] = ldg_stream(base + (static_cast<int64_t>(r) * d + sub * 8) * 2);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) quant_kernel(QuantParams p) {
  allow_dependents();  // the attention kernel may start early; it waits for this grid
  __shared__ float4 sred[kThreads];
  __shared__ float sinv[128];
  const PrepDims& g = p.g;
  const int d = g.d, dp = g.dp;
  const int ngrp = (g.N + p.tpc - 1) / p.tpc;
  // Last slice first: the streaming kernel before this one reads V in slice order, so the
  // slices it read last are the likeliest to be still in L2.
  const int64_t cta = static_cast<int64_t>(gridDim.x) - 1 - blockIdx.x;
  const int64_t bh = cta / ngrp;
  const int grp = static_cast<int>(cta - bh * ngrp);
  const int tok0 = grp * p.tpc;
  const int ntok = min(p.tpc, g.N - tok0);
  const bool vec = (d & 7) == 0;
  // Vector path: thread (rp, sub) writes the 8-byte piece sub of rows rp + rpp t; pieces at or
  // past d are the zero padding of the row.
  const int opr = dp >> 3;
  const int rpp = kThreads / opr;
  const int sub = threadIdx.x % opr, rp = threadIdx.x / opr;
  const bool on_row = vec && rp < rpp;
  const bool on = on_row && sub * 8 < d;
  const char* base = reinterpret_cast<const char*>(p.v) + ((bh * g.N + tok0) * d) * 2;
  // The first batch reads only the caller's V: it is in flight while this CTA waits for the
  // streaming kernel's partials.
  uint4 u[kQuantBatch];
  quant_load(u, base, 0, ntok, d, rpp, rp, sub, on);
  grid_dependency_wait();

  // Channel maxima of the slice: the max over its npart partial rows, read as float4 columns by
  // rstride row lanes each, then over the row lanes in shared memory.
  const int nc4 = dp >> 2;
  const int rstride = kThreads / nc4;
  {
    const int col = threadIdx.x % nc4, r0 = threadIdx.x / nc4;
    float4 m = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (r0 < rstride) {
      const float4* src = reinterpret_cast<const float4*>(p.part_amax + bh * p.npart * dp) + col;
#pragma unroll 4
      for (int r = r0; r < p.npart; r += rstride) {
        const float4 x = __ldcg(src + static_cast<int64_t>(r) * nc4);
        m.x = fmaxf(m.x, x.x);
        m.y = fmaxf(m.y, x.y);
        m.z = fmaxf(m.z, x.z);
        m.w = fmaxf(m.w, x.w);
      }
    }
    sred[threadIdx.x] = m;
  }
  __syncthreads();
  if (threadIdx.x < dp) {
    const int c = threadIdx.x;
    const float* sr = reinterpret_cast<const float*>(sred);
    float m = 0.0f;
    for (int rr = 0; rr < rstride; ++rr) m = fmaxf(m, sr[rr * dp + c]);
    const float inv = __fdiv_rn(127.0f, m);
    const bool live = (c < d) && channel_live(m, inv);
    sinv[c] = live ? inv : 0.0f;
    if (grp == 0 && c < d) p.v_scale[bh * d + c] = live ? __fdiv_rn(m, 127.0f) : 0.0f;
  }
  // mu of the packed tensors (one warp each, on the slice's first CTA): the sum of the chunk
  // partials, exact in double in any order, over N d.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (grp == 0 && warp < p.npack) {
    const double* src = (warp == 0 ? p.part_mu[0] : p.part_mu[1]) + bh * g.nchunk;
    double s = 0.0;
    for (int c = lane; c < g.nchunk; c += 32) s += __ldcg(src + c);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) (warp == 0 ? p.mu[0] : p.mu[1])[bh] = static_cast<float>(s / (static_cast<double>(g.N) * d));
  }
  __syncthreads();

  int8_t* out = p.vq + (bh * g.N + tok0) * dp;
  if (vec) {
    float inv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) inv[e] = sinv[sub * 8 + e];
    const int rows_per_batch = kQuantBatch * rpp;
    for (int r0 = 0; r0 < ntok; r0 += rows_per_batch) {
      if (r0 > 0) quant_load(u, base, r0, ntok, d, rpp, rp, sub, on);
#pragma unroll
      for (int j = 0; j < kQuantBatch; ++j) {
        const int r = r0 + j * rpp + rp;
        if (on_row && r < ntok) {
          uint2 w = make_uint2(0u, 0u);
          if (on) {
            float f[8];
            unpack8<T>(u[j], f);
            w.x = quant4(f, inv);
            w.y = quant4(f + 4, inv + 4);
          }
          *reinterpret_cast<uint2*>(out + static_cast<int64_t>(r) * dp + sub * 8) = w;
        }
      }
    }
  } else {
    const T* vb = reinterpret_cast<const T*>(p.v) + (bh * g.N + tok0) * d;
    for (int e = threadIdx.x; e < ntok * dp; e += kThreads) {
      const int r = e / dp, c = e - r * dp;
      int q = 0;
      if (c < d) {
        q = __float2int_rn(__fmul_rn(load1<T>(vb + static_cast<int64_t>(r) * d + c), sinv[c]));
        q = max(-127, min(127, q));
      }
      out[e] = static_cast<int8_t>(q);
    }
  }
}

// 16-byte pieces of eight 16-bit values: the sign byte (bit e = x_e < 0 by IEEE compare: -0.0 and
// NaN give 0) and the double sum of |x| (each magnitude exact in double; every partial sum
// exact, so the order is free). fp16 works on the packed halves: a half2 compare gives a lane
// mask per word, and each magnitude is read as a double by bit placement alone (f16_scaled).
//
// An fp16 magnitude with exponent field e and fraction m, placed at bit 52 - 10 of a double
// (fraction) and bit 52 (exponent field), is the double with exponent field e and fraction m:
// (1 + m/2^10) 2^(e - 1023) for e >= 1 and m 2^-1032 for e = 0 (a subnormal double), i.e.
// exactly |x| 2^-1008 in both cases. Sums of these scaled values round exactly as the sums of
// |x| do (a power-of-two scale; below 2^-1022 every sum of multiples of 2^-1032 is exact), and
// one multiply by 2^1008 at the end restores the scale.
constexpr double kF16Unscale = 0x1p1008;
__device__ __forceinline__ double f16_scaled(uint32_t hi_word) {
  return __hiloint2double(static_cast<int>(hi_word), 0);
}

template <typename T>
__device__ __forceinline__ uint32_t piece_sign_abs(const uint4& u, double& acc) {
  if constexpr (std::is_same<T, __half>::value) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t x = 0;
    double a8[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h2;
      *reinterpret_cast<uint32_t*>(&h2) = w[i];
      const uint32_t m = __hlt2_mask(h2, __float2half2_rn(0.0f));  // 0xFFFF per lane below zero
      x |= (m & 0x00010001u) << (2 * i);  // element 2i at bit 2i, element 2i + 1 at bit 16 + 2i
      const uint32_t a = w[i] & 0x7FFF7FFFu;
      a8[2 * i] = f16_scaled((a << 10) & 0x01FFFC00u);
      a8[2 * i + 1] = f16_scaled((a >> 6) & 0x01FFFC00u);
    }
    acc += ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
    return (x | (x >> 15)) & 0xFFu;
  } else {
    float f[8];
    unpack8<T>(u, f);
    uint32_t byte = 0;
    double a8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      byte |= (f[e] < 0.0f ? 1u : 0u) << e;
      a8[e] = static_cast<double>(fabsf(f[e]));
    }
    acc += ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
    return byte;
  }
}

// ---------------------------------------------------------------------------------------
// Warp-granular streaming for rows of whole 16-byte pieces (d % 8 == 0). A warp covers
// rpp = 32 / (d/8) rows per pass, lane (row-in-pass, piece) reading one 16-byte piece, so a
// pass reads rpp consecutive rows as one coalesced span; kBatch passes are loaded before any
// is used. Warps never wait for each other: reductions are warp shuffles, and the sign bytes
// of a chunk are assembled in the warp's own shared-memory rows.
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 8;

struct Lanes {
  int tpr, rpp, sub, rp;
  bool on;
};

__device__ __forceinline__ Lanes lanes_for(int d) {
  Lanes L;
  const int lane = threadIdx.x & 31;
  L.tpr = d >> 3;
  L.rpp = 32 / L.tpr;
  L.sub = lane % L.tpr;
  L.rp = lane / L.tpr;
  L.on = L.rp < L.rpp;
  return L;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Max over the lanes that hold the same 8 channels (lanes sub + tpr * t); every lane of the
// group gets the result.
__device__ __forceinline__ void group_max(float (&mx)[8], const Lanes& L) {
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = __shfl_sync(0xffffffffu, mx[e], L.sub);
  for (int t = 1; t < L.rpp; ++t) {
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], __shfl_sync(0xffffffffu, mx[e], L.sub + L.tpr * t));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = m[e];
}

// Sign bytes and sum |x| of one chunk (rows [0, ntok) at `rows`, row stride d). The chunk's
// 16-byte sign rows go to `bits` through the warp's staging rows `sb` (bytes past d/8 are
// zero). Returns this lane's part of the sum.
template <typename T>
__device__ __forceinline__ double pack_chunk(const char* rows, int ntok, int d, const Lanes& L, uint8_t (*sb)[16],
                                             uint4* bits) {
  double acc = 0.0;
  const int npass = (ntok + L.rpp - 1) / L.rpp;
  for (int p0 = 0; p0 < npass; p0 += kBatch) {
    uint4 u[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int r = (p0 + j) * L.rpp + L.rp;
      if (L.on && r < ntok) u[j] = ldg_stream(rows + (static_cast<int64_t>(r) * d + L.sub * 8) * 2);
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int r = (p0 + j) * L.rpp + L.rp;
      if (L.on && r < ntok) {
        float f[8];
        unpack8<T>(u[j], f);
        uint32_t byte = 0;
        double a8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          byte |= (f[e] < 0.0f ? 1u : 0u) << e;
          a8[e] = static_cast<double>(fabsf(f[e]));
        }
        // Every partial sum of 16-bit magnitudes is exact in double: the order is free.
        acc += ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
        sb[r][L.sub] = static_cast<uint8_t>(byte);
      }
    }
  }
  __syncwarp();
  for (int r = threadIdx.x & 31; r < ntok; r += 32) bits[r] = *reinterpret_cast<const uint4*>(sb[r]);
  __syncwarp();
  return acc;
}

// Channel maxima |v| of one chunk into this lane's 8 channels (8 * sub ...).
template <typename T>
__device__ __forceinline__ void amax_chunk(const char* rows, int ntok, int d, const Lanes& L, float (&mx)[8]) {
  const int npass = (ntok + L.rpp - 1) / L.rpp;
  for (int p0 = 0; p0 < npass; p0 += kBatch) {
    uint4 u[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int r = (p0 + j) * L.rpp + L.rp;
      if (L.on && r < ntok) u[j] = __ldg(reinterpret_cast<const uint4*>(rows + (static_cast<int64_t>(r) * d + L.sub * 8) * 2));
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int r = (p0 + j) * L.rpp + L.rp;
      if (L.on && r < ntok) {
        float f[8];
        unpack8<T>(u[j], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], fabsf(f[e]));
      }
    }
  }
}

__device__ __forceinline__ uint8_t (*warp_bits_rows())[16] {
  __shared__ __align__(16) uint8_t sbits[kWarps][kPrepTokens][16];
  uint8_t (*sb)[16] = sbits[threadIdx.x >> 5];
  // Bytes past d/8 of a sign row are never written: zero this warp's rows once.
  for (int e = threadIdx.x & 31; e < kPrepTokens; e += 32) *reinterpret_cast<uint4*>(sb[e]) = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
  return sb;
}

// Chunk mode. CTAs [0, pack_ctas): one warp per (packing job, slice, 128-token chunk), its sign
// rows and partial sum |x|. The CTAs after them (when there is a channel-max job): one per
// (slice, group of kWarps chunks), a warp per chunk, the group's channel maxima reduced in
// shared memory to one partial row. The V CTAs come last in the grid, so V is the tensor read
// most recently when the quantiser reads it again.
template <typename T>
__global__ void __launch_bounds__(kThreads, 3) prep_warp_kernel(PrepParams p, int npack, unsigned pack_ctas) {
  allow_dependents();  // the quantiser may start early; it waits for this grid
  const PrepDims& g = p.g;
  const Lanes L = lanes_for(g.d);
  const int warp = threadIdx.x >> 5;
  if (blockIdx.x < pack_ctas) {
    const int64_t per_job = g.BH * g.nchunk;
    const int64_t unit = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
    uint8_t (*sb)[16] = warp_bits_rows();
    if (unit >= npack * per_job) return;
    const int j = static_cast<int>(unit / per_job);
    const PrepJob job = j == 0 ? p.job[0] : p.job[1];
    const int64_t rest = unit - j * per_job;
    const int64_t bh = rest / g.nchunk;
    const int chunk = static_cast<int>(rest - bh * g.nchunk);
    const int tok0 = chunk * kPrepTokens;
    const int ntok = min(kPrepTokens, g.N - tok0);
    const char* rows = reinterpret_cast<const char*>(job.src) + ((bh * g.N + tok0) * g.d) * 2;
    const double tot = warp_sum(pack_chunk<T>(rows, ntok, g.d, L, sb, reinterpret_cast<uint4*>(job.bits) + bh * g.N + tok0));
    if ((threadIdx.x & 31) == 0) job.part_sum[bh * g.nchunk + chunk] = tot;
    return;
  }
  __shared__ float smax[kWarps][128];
  const PrepJob job = npack == 0 ? p.job[0] : (npack == 1 ? p.job[1] : p.job[2]);
  const int ngrp = (g.nchunk + kWarps - 1) / kWarps;
  const int64_t c = blockIdx.x - pack_ctas;
  const int64_t bh = c / ngrp;
  const int grp = static_cast<int>(c - bh * ngrp);
  const int chunk = grp * kWarps + warp;
  float mx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = 0.0f;
  if (chunk < g.nchunk) {
    const int tok0 = chunk * kPrepTokens;
    const int ntok = min(kPrepTokens, g.N - tok0);
    amax_chunk<T>(reinterpret_cast<const char*>(job.src) + ((bh * g.N + tok0) * g.d) * 2, ntok, g.d, L, mx);
  }
  group_max(mx, L);
  if (L.on && L.rp == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) smax[warp][L.sub * 8 + e] = mx[e];
  }
  __syncthreads();
  for (int ch = threadIdx.x; ch < g.dp; ch += kThreads) {
    float m = 0.0f;
    if (ch < g.d)
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, smax[w][ch]);
    job.part[(bh * ngrp + grp) * g.dp + ch] = m;
  }
}

// Whole-slice mode (d >= 32): one CTA per (slice, tensor) loads the slice in batches of kSliceBatch
// passes of rpp = 256 / (d/8) rows (a slice of up to kSliceBatch * rpp rows in one batch, all of
// its loads in flight at once), then reduces once: mu for q and k; for v the channel maxima, the
// scales, and a second batch of loads (L2) that quantises. Sign bytes are assembled per batch
// in shared memory and written as 16-byte rows. Two batch depths: 7 passes when they hold the
// slice in one batch (a DeiT-B slice, 197 rows of 64), which keeps the kernel within 64
// registers so that four CTAs share an SM and more of one CTA's loads overlap another's
// arithmetic; otherwise 10 passes at three CTAs per SM (the load slots past the slice's rows
// cost issue slots, so the shallower batch is taken whenever it suffices).
constexpr int kSliceBatchShort = 7;
constexpr int kSliceBatch = 10;

template <typename T, int kSliceBatch>
__global__ void __launch_bounds__(kThreads, kSliceBatch <= kSliceBatchShort ? 4 : 3) prep_slice_kernel(SliceParams p) {
  // The attention kernel that follows may start on SMs this grid frees once every CTA of it
  // is running; it waits for this grid's completion before it reads what this grid writes.
  allow_dependents();
  __shared__ __align__(16) uint8_t sbits[kSliceBatch * kThreads / 4][16];  // d >= 32: at most 64 rows per pass
  __shared__ float smax[kThreads * 8];
  __shared__ double sred[kThreads / 32];
  const PrepDims& g = p.g;
  const int64_t bh = blockIdx.x;
  // 0: q, 1: k, 2: v. The v CTAs (two passes over their slice) are the longest: they take the
  // first grid row, so they are scheduled first and the q and k CTAs fill in behind them.
  const int job = (static_cast<int>(blockIdx.y) + 2) % 3;
  const int d = g.d, dp = g.dp;
  const int tpr = d >> 3;
  const int rpp = kThreads / tpr;
  const int sub = threadIdx.x % tpr, rp = threadIdx.x / tpr;
  const bool on = rp < rpp;
  const int rows_per_batch = kSliceBatch * rpp;
  const char* src = reinterpret_cast<const char*>(job == 0 ? p.q : (job == 1 ? p.k : p.v)) + (bh * g.N * d) * 2;
  if (job < 2) {
    // Bytes past d/8 of a sign row are never written.
    for (int e = threadIdx.x; e < rows_per_batch; e += kThreads)
      *reinterpret_cast<uint4*>(sbits[e]) = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    uint4* bits = reinterpret_cast<uint4*>(job == 0 ? p.bits_q : p.bits_k) + bh * g.N;
    double acc = 0.0;
    for (int r0 = 0; r0 < g.N; r0 += rows_per_batch) {
      const int nrow = min(rows_per_batch, g.N - r0);
      uint4 u[kSliceBatch];
#pragma unroll
      for (int j = 0; j < kSliceBatch; ++j) {
        const int r = j * rpp + rp;
        if (on && r < nrow) u[j] = ldg_stream(src + (static_cast<int64_t>(r0 + r) * d + sub * 8) * 2);
      }
#pragma unroll
      for (int j = 0; j < kSliceBatch; ++j) {
        const int r = j * rpp + rp;
        if (on && r < nrow) sbits[r][sub] = static_cast<uint8_t>(piece_sign_abs<T>(u[j], acc));
      }
      __syncthreads();
      for (int r = threadIdx.x; r < nrow; r += kThreads) bits[r0 + r] = *reinterpret_cast<const uint4*>(sbits[r]);
      __syncthreads();
    }
    double tot = block_sum(acc, sred);
    if constexpr (std::is_same<T, __half>::value) tot *= kF16Unscale;  // exact (see f16_scaled)
    if (threadIdx.x == 0) (job == 0 ? p.mu_q : p.mu_k)[bh] = static_cast<float>(tot / (static_cast<double>(g.N) * d));
    return;
  }
  // v: channel maxima over the slice (fp16: packed half2 maxima of the magnitudes, exact).
  float mx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = 0.0f;
  uint32_t hm[4] = {0u, 0u, 0u, 0u};  // fp16: |v| maxima as half2 bit patterns (0 = +0.0)
  for (int r0 = 0; r0 < g.N; r0 += rows_per_batch) {
    const int nrow = min(rows_per_batch, g.N - r0);
    uint4 u[kSliceBatch];
#pragma unroll
    for (int j = 0; j < kSliceBatch; ++j) {
      const int r = j * rpp + rp;
      if (on && r < nrow) u[j] = __ldg(reinterpret_cast<const uint4*>(src + (static_cast<int64_t>(r0 + r) * d + sub * 8) * 2));
    }
#pragma unroll
    for (int j = 0; j < kSliceBatch; ++j) {
      const int r = j * rpp + rp;
      if (on && r < nrow) {
        if constexpr (std::is_same<T, __half>::value) {
          const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            __half2 a, b;
            *reinterpret_cast<uint32_t*>(&a) = w[i] & 0x7FFF7FFFu;
            *reinterpret_cast<uint32_t*>(&b) = hm[i];
            const __half2 c = __hmax2(a, b);
            hm[i] = *reinterpret_cast<const uint32_t*>(&c);
          }
        } else {
          float f[8];
          unpack8<T>(u[j], f);
#pragma unroll
          for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], fabsf(f[e]));
        }
      }
    }
  }
  if constexpr (std::is_same<T, __half>::value) {
    const uint4 hv = make_uint4(hm[0], hm[1], hm[2], hm[3]);
    unpack8<T>(hv, mx);
  }
  __shared__ float sinv[128];
  if (on) {
#pragma unroll
    for (int e = 0; e < 8; ++e) smax[rp * d + sub * 8 + e] = mx[e];
  }
  __syncthreads();
  const int rows = min(rpp, g.N);
  for (int c = threadIdx.x; c < dp; c += kThreads) {
    float m = 0.0f;
    if (c < d)
      for (int rr = 0; rr < rows; ++rr) m = fmaxf(m, smax[rr * d + c]);
    const float inv = __fdiv_rn(127.0f, m);
    const bool live = (c < d) && channel_live(m, inv);
    sinv[c] = live ? inv : 0.0f;
    if (c < d) p.v_scale[bh * d + c] = live ? __fdiv_rn(m, 127.0f) : 0.0f;
  }
  __syncthreads();
  float inv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) inv[e] = sinv[sub * 8 + e];
  const bool pad = (d & 15) == 8 && sub == tpr - 1;
  int8_t* vq = p.vq + bh * g.N * dp;
  for (int r0 = 0; r0 < g.N; r0 += rows_per_batch) {
    const int nrow = min(rows_per_batch, g.N - r0);
    uint4 u[kSliceBatch];
#pragma unroll
    for (int j = 0; j < kSliceBatch; ++j) {
      const int r = j * rpp + rp;
      if (on && r < nrow) u[j] = ldg_stream(src + (static_cast<int64_t>(r0 + r) * d + sub * 8) * 2);
    }
#pragma unroll
    for (int j = 0; j < kSliceBatch; ++j) {
      const int r = j * rpp + rp;
      if (on && r < nrow) {
        float f[8];
        unpack8<T>(u[j], f);
        const uint2 w = make_uint2(quant4(f, inv), quant4(f + 4, inv + 4));
        int8_t* o = vq + static_cast<int64_t>(r0 + r) * dp + sub * 8;
        if (pad)
          *reinterpret_cast<uint4*>(o) = make_uint4(w.x, w.y, 0u, 0u);
        else
          *reinterpret_cast<uint2*>(o) = w;
      }
    }
  }
}

}  // namespace

unsigned warp_grid(int64_t units) { return static_cast<unsigned>(ceil_div(units, kWarps)); }

int amax_parts(const PrepDims& g) { return (g.d & 7) == 0 ? static_cast<int>(ceil_div(g.nchunk, kWarps)) : g.nchunk; }

cudaError_t launch_prep(const PrepParams& p, int dt, int njobs, cudaStream_t s) {
  if ((p.g.d & 7) == 0) {
    int npack = 0;
    while (npack < njobs && p.job[npack].kind == kJobPack) ++npack;
    const unsigned pack_ctas = warp_grid(npack * p.g.BH * p.g.nchunk);
    const unsigned grid = pack_ctas + (npack < njobs ? static_cast<unsigned>(p.g.BH * amax_parts(p.g)) : 0u);
    if (dt == BA_F16)
      prep_warp_kernel<__half><<<grid, kThreads, 0, s>>>(p, npack, pack_ctas);
    else
      prep_warp_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(p, npack, pack_ctas);
    return cudaGetLastError();
  }
  const dim3 grid(static_cast<unsigned>(p.g.BH * p.g.nchunk), static_cast<unsigned>(njobs));
  if (dt == BA_F16)
    prep_kernel<__half><<<grid, kThreads, 0, s>>>(p);
  else
    prep_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const FinalizeParams& p, cudaStream_t s) {
  finalize_kernel<<<static_cast<unsigned>(p.g.BH), 32, 0, s>>>(p);
  return cudaGetLastError();
}

// The whole-slice kernel gives each CTA a whole (slice, tensor): it needs enough slices to fill
// the GPU and short slices (at most two load batches each; longer ones stream better as
// 128-token chunks spread over many CTAs), and rows of whole 16-byte pieces.
bool use_slice_prep(const PrepDims& g) {
  if ((g.d & 7) != 0 || g.d < 32) return false;
  const int rows_per_batch = kSliceBatch * (kThreads / (g.d >> 3));
  return 3 * g.BH >= 384 && g.N <= 2 * rows_per_batch;
}

cudaError_t launch_prep_slices(const SliceParams& p, int dt, cudaStream_t s) {
  if ((p.g.d & 7) != 0 || p.g.d < 32) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(p.g.BH), 3);
  const bool shallow = p.g.N <= kSliceBatchShort * (kThreads / (p.g.d >> 3));
  if (dt == BA_F16) {
    if (shallow)
      prep_slice_kernel<__half, kSliceBatchShort><<<grid, kThreads, 0, s>>>(p);
    else
      prep_slice_kernel<__half, kSliceBatch><<<grid, kThreads, 0, s>>>(p);
  } else {
    if (shallow)
      prep_slice_kernel<__nv_bfloat16, kSliceBatchShort><<<grid, kThreads, 0, s>>>(p);
    else
      prep_slice_kernel<__nv_bfloat16, kSliceBatch><<<grid, kThreads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

// Tokens per quantiser CTA: 1024, halved (down to 128) while the grid would hold fewer than 512
// CTAs, so that short slices still spread over every SM.
int quant_tokens_per_cta(const PrepDims& g) {
  int tpc = kQuantTokens;
  while (tpc > kPrepTokens && g.BH * ceil_div(g.N, tpc) < 512) tpc /= 2;
  return tpc;
}

// A programmatic dependent of the streaming kernel: its CTAs may be resident, with their first
// V loads in flight, before that grid completes.
cudaError_t launch_quant(const QuantParams& p, int dt, cudaStream_t s) {
  if (p.tpc < 1) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(p.g.BH * ceil_div(p.g.N, p.tpc)));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dt == BA_F16) return cudaLaunchKernelEx(&cfg, quant_kernel<__half>, p);
  return cudaLaunchKernelEx(&cfg, quant_kernel<__nv_bfloat16>, p);
}

}  // namespace binattn
