// Fused BinaryAttention forward on CUDA cores (sm_100a): the straightforward kernel.
//
// One CTA = 64 query rows of one (b, h); 4 threads per row, each owning every fourth key
// of a 128-key block and a quarter of the output channels. Per key block:
//   x_ij = d - 2 popc(q bits XOR k bits)            (gist.science/zh 2.1 and 2.2(1))
//   s_ij = fmaf(alpha, x_ij, b_ij)                   (bias: gist.science/zh 2.2(2))
//   m_t = max(m_{t-1}, max_j s_ij), c_t = exp(m_{t-1} - m_t), P~ = exp(s - m_t), l = l c_t + sum P~
//   P = rne(255 P~) as uint8                         (gist.science/zh 2.2(3))
//   acc = sum_j P_ij vq_jc with dp4a (u8 x s8 -> s32; the instruction class named on
//         every page for P.V), O~ = O~ c_t + acc
// and at the end O = O~ * v_scale / (255 l). The online softmax over ascending key blocks
// is FlashAttention-2's (gist.science/zh 2.3).
//
// This kernel is the reference for the tcgen05 kernel and covers every supported shape.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"

namespace binattn {

namespace {

constexpr int kRows = 64;
constexpr int kThreads = 256;
constexpr int kRowWords = kKvBlock / 4 + 1;  // 128 bytes of codes per row + 4 pad bytes

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnParams p) {
  __shared__ uint4 skb[kKvBlock];
  __shared__ uint32_t svt[128 * kRowWords];  // V block transposed: [channel][key bytes]
  __shared__ uint32_t sp[kRows * kRowWords];  // P codes: [row][key bytes]

  const int N = p.N, d = p.d, dp = p.dp;
  const int qtiles = static_cast<int>(ceil_div(N, kRows));
  const int64_t bh = blockIdx.x / qtiles;
  const int qt = static_cast<int>(blockIdx.x - bh * qtiles);
  const int64_t b = bh / p.H, h = bh - b * p.H;
  const int tid = threadIdx.x;
  const int r = tid >> 2, quad = tid & 3;
  const int i = qt * kRows + r;
  const bool row_ok = i < N;
  const int cpt = dp >> 2;  // output channels per thread (dp is a multiple of 16)

  uint4 qb = make_uint4(0u, 0u, 0u, 0u);
  if (row_ok) qb = reinterpret_cast<const uint4*>(p.bits_q)[bh * N + i];
  const float alpha = __fmul_rn(__fmul_rn(p.softmax_scale, p.mu_q[bh]), p.mu_k[bh]);

  float m = -CUDART_INF_F, l = 0.0f;
  float of[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) of[c] = 0.0f;

  uint8_t* svt_b = reinterpret_cast<uint8_t*>(svt);
  uint8_t* sp_b = reinterpret_cast<uint8_t*>(sp);
  const uint32_t* vq32 = reinterpret_cast<const uint32_t*>(p.vq);
  const int wpk = dp >> 2;  // V words per key

  for (int t0 = 0; t0 < N; t0 += kKvBlock) {
    const int nk = min(kKvBlock, N - t0);
    __syncthreads();
    if (tid < kKvBlock)
      skb[tid] = (tid < nk) ? reinterpret_cast<const uint4*>(p.bits_k)[bh * N + t0 + tid]
                            : make_uint4(0u, 0u, 0u, 0u);
    for (int idx = tid; idx < kKvBlock * wpk; idx += kThreads) {
      const int j = idx / wpk, cw = idx - j * wpk;
      const uint32_t w = (j < nk) ? __ldg(vq32 + (bh * N + t0 + j) * wpk + cw) : 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) svt_b[(4 * cw + e) * (kRowWords * 4) + j] = static_cast<uint8_t>(w >> (8 * e));
    }
    __syncthreads();

    float s[32];
    float tmax = -CUDART_INF_F;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int j = quad + 4 * u;
      s[u] = -CUDART_INF_F;
      if (row_ok && j < nk) {
        const uint4 kb = skb[j];
        const int diff = __popc(qb.x ^ kb.x) + __popc(qb.y ^ kb.y) + __popc(qb.z ^ kb.z) + __popc(qb.w ^ kb.w);
        const int x = d - 2 * diff;
        const float bias = bias_at(p.bias, b, h, N, i, t0 + j);
        s[u] = __fmaf_rn(alpha, static_cast<float>(x), bias);
        if (p.dbg_logits != nullptr) p.dbg_logits[(bh * N + i) * N + t0 + j] = x;
        tmax = fmaxf(tmax, s[u]);
      }
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float m_new = fmaxf(m, tmax);
    // exp(m_old - m_new) and exp(s - m) in double, rounded to fp32: the 8-bit code is then
    // decided on the same correctly rounded fp32 value the CPU reference uses.
    const float c = (m == -CUDART_INF_F) ? 0.0f : static_cast<float>(exp(static_cast<double>(m) - m_new));
    float lsum = 0.0f;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int j = quad + 4 * u;
      int code = 0;
      if (s[u] != -CUDART_INF_F) {
        const float pf = static_cast<float>(exp(static_cast<double>(s[u]) - static_cast<double>(m_new)));
        lsum += pf;
        code = min(255, max(0, __float2int_rn(__fmul_rn(255.0f, pf))));
      }
      sp_b[r * (kRowWords * 4) + j] = static_cast<uint8_t>(code);
      if (p.dbg_p != nullptr && row_ok && j < nk) p.dbg_p[(bh * N + i) * N + t0 + j] = static_cast<uint8_t>(code);
    }
    if (row_ok) {
      l = l * c + lsum;
      m = m_new;
    }
    __syncthreads();

#pragma unroll
    for (int cc = 0; cc < 32; ++cc) {
      if (cc < cpt) {
        const int ch = quad * cpt + cc;
        int acc = 0;
#pragma unroll 8
        for (int w = 0; w < kKvBlock / 4; ++w) acc = dp4a_us(sp[r * kRowWords + w], svt[ch * kRowWords + w], acc);
        of[cc] = __fmaf_rn(of[cc], c, static_cast<float>(acc));
      }
    }
  }

  float lt = l;
  lt += __shfl_xor_sync(0xffffffffu, lt, 1);
  lt += __shfl_xor_sync(0xffffffffu, lt, 2);
  if (!row_ok) return;
  const float inv_l = 1.0f / (255.0f * lt);
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const int ch = quad * cpt + k;
    if (k < cpt && ch < d) {
      const float val = of[k] * p.v_scale[bh * d + ch] * inv_l;
      store_out(p.o, (bh * N + i) * d + ch, val, p.o_dt);
    }
  }
}

}  // namespace

cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t s) {
  const int64_t qtiles = ceil_div(p.N, kRows);
  const int64_t grid = static_cast<int64_t>(p.B) * p.H * qtiles;
  attn_simt_kernel<<<static_cast<unsigned>(grid), kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace binattn
