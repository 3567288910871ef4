// Fused BinaryAttention forward on 5th-generation tensor cores (sm_100a: tcgen05 + TMEM + TMA).
//
// What it computes is the blockwise forward of the CUDA-core kernel (attn_simt.cu) and of the
// CPU reference: binary QK (gist.science/zh technical summary 2.1-2.2(1)), bias b_ij (2.2(2)),
// FlashAttention-2-style online softmax over ascending 128-key blocks (2.3), 8-bit P on [0,1]
// (2.2(3)), per-channel int8 V and an integer P.V (the u8 x s8 -> s32 instruction class named
// on every page).
//
// How, on B200:
//   * One CTA per SM; each CTA owns NQ query tiles of 128 rows of one (b, h).
//   * Warp 0 (producer) expands the 1-bit sign rows of Q (once) and of each K block into fp8
//     +-1 operands in shared memory (channels >= d become 0), and TMA-loads the int8 V block
//     (a 4-D tensor map that lands it in the MN-major core-matrix layout the MMA reads).
//   * Warp 1 issues the MMAs from one thread:
//       S  = Q . K^T   tcgen05.mma kind::f8f6f4 (e4m3 +-1, fp32 accumulate: exact integers)
//       O += P . V     tcgen05.mma kind::i8, A = the uint8 codes read from TMEM, B = int8 V
//     both accumulators live in tensor memory.
//   * Warpgroup 1+q (one thread per query row) runs the softmax of query tile q: it reads its
//     row of S from TMEM, forms s = fmaf(alpha, x, b), the running max, P~ = 2^((s-m) log2 e),
//     the row sum, and writes the 8-bit codes back to TMEM as the A operand of P.V.
//   * The int32 P.V accumulator keeps accumulating across key blocks while a row's running max
//     is unchanged (the rescale factor is exactly 1 then); when a row's max rises the thread
//     folds the accumulator into its fp32 running output, O~ = (O~ + acc) * exp(m_old - m_new),
//     and zeroes the accumulator row. This is the same arithmetic as rescaling every block.
//   * Every wait is bounded (1 s): on expiry the kernel records BA_ERR_TIMEOUT in a device
//     status word, every role leaves its loop, and the CTA frees its tensor memory.
#include <cuda.h>
#include <math_constants.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace binattn {

__device__ int g_device_status = 0;

namespace {

using namespace ptx;

constexpr int BM = 128;        // query rows per tile = MMA M
constexpr int BN = kKvBlock;   // keys per block = MMA N of QK, K of P.V
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

template <int DP>
struct Cfg {
  static constexpr int DQ = (DP + 31) / 32 * 32;   // QK contraction width: fp8 K-steps of 32
  static constexpr int NQ = (DP <= 64) ? 2 : 1;     // query tiles per CTA
  static constexpr int kThreads = 128 + 128 * NQ;   // 4 service warps + NQ softmax warpgroups
  static constexpr int kQBytes = BM * DQ;
  static constexpr int kKBytes = BN * DQ;
  static constexpr int kVBytes = BN * DP;
  static constexpr int offQ = 0;
  static constexpr int offK = offQ + NQ * kQBytes;
  static constexpr int offV = offK + 2 * kKBytes;
  static constexpr int offKoff = offV + 2 * kVBytes;
  static constexpr int offScale = offKoff + 2 * BN * 4;
  static constexpr int offBar = offScale + 128 * 4;
  static constexpr int kNumBars = 6 + 3 * NQ;
  static constexpr int offMisc = offBar + kNumBars * 8;
  static constexpr int kBytes = offMisc + 16;
  static constexpr int kTabOff = (kBytes + 127) / 128 * 128;
  // Tensor-memory columns of query tile q: S (fp32, 128), P (u8 codes, 32), O (s32, DP).
  __host__ __device__ static constexpr uint32_t tS(int q) { return q * 256; }
  __host__ __device__ static constexpr uint32_t tP(int q) { return q * 256 + 128; }
  __host__ __device__ static constexpr uint32_t tO(int q) { return q * 256 + 160; }
  static_assert(tO(NQ - 1) + DP <= 512, "tensor memory budget");
};

// Barrier slots.
enum { kKvFull = 0, kKvEmpty = 2, kQFull = 4, kDrain = 5, kSFull = 6 };
template <int NQ> struct Bars {
  __host__ __device__ static constexpr int pfull(int q) { return kSFull + NQ + q; }
  __host__ __device__ static constexpr int odone(int q) { return kSFull + 2 * NQ + q; }
};

// Waits for the phase of `bar` with the given parity. Gives up after kTimeoutNs (recording the
// timeout in the device status word and raising the CTA's abort flag) or, when `yield` is set,
// as soon as another role has raised the abort flag.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             bool yield = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (yield && *abort_flag) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      *abort_flag = 1;
      atomicExch(&g_device_status, 1);
      return false;
    }
  }
}

// Warp-uniform variant: every lane waits, and the warp proceeds only if all lanes succeeded.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = wait_bounded(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t channel_mask(int c0, int d) {
  const int n = d - c0;
  return n >= 4 ? 0xffffffffu : (n <= 0 ? 0u : ((1u << (8 * n)) - 1u));
}

// 1-bit sign rows -> fp8 e4m3 +-1 (bit 1 = negative) in the K-major no-swizzle core-matrix
// layout: byte (row r, channel c) at (c/16)*2048 + r*16 + c%16. Channels >= d and rows >= N
// are 0 so they add nothing to the dot products.
template <int DQ>
__device__ __forceinline__ void expand_signs(uint8_t* dst, const uint4* bits_rows, int row0, int N, int d,
                                             int lane) {
#pragma unroll
  for (int u = 0; u < BM / 32; ++u) {
    const int r = lane + 32 * u;
    const int tok = row0 + r;
    const bool ok = tok < N;
    const uint4 b = ok ? bits_rows[tok] : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int kc = 0; kc < DQ / 16; ++kc) {
      const uint32_t bits16 = (w[kc >> 1] >> (16 * (kc & 1))) & 0xffffu;
      uint32_t o[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint32_t nib = (bits16 >> (4 * g)) & 0xfu;
        const uint32_t val = ((nib * 0x10204080u) & 0x80808080u) | 0x38383838u;
        o[g] = ok ? (val & channel_mask(16 * kc + 4 * g, d)) : 0u;
      }
      *reinterpret_cast<uint4*>(dst + kc * 2048 + r * 16) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

template <int DP, int BK>
__global__ void __launch_bounds__(Cfg<DP>::kThreads, 1)
    attn_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmap_v, int tab_mode, int tsize,
                   int kmax) {
  using C = Cfg<DP>;
  constexpr int NQ = C::NQ, DQ = C::DQ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::offQ;
  uint8_t* sK = smem + C::offK;
  uint8_t* sV = smem + C::offV;
  int* koff = reinterpret_cast<int*>(smem + C::offKoff);
  float* sscale = reinterpret_cast<float*>(smem + C::offScale);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::offBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::offMisc + 4);
  // Rel-pos table of this CTA's head, staged when it fits: tab_mode 1 = table only,
  // 2 = table followed by 2*tsize zeros (targets of prefix rows and prefix keys).
  float* stab = reinterpret_cast<float*>(smem + C::kTabOff);

  const int N = p.N, d = p.d;
  const int ctas_per_bh = static_cast<int>(ceil_div(N, BM * NQ));
  const int64_t bh = blockIdx.x / ctas_per_bh;
  const int q0 = static_cast<int>(blockIdx.x - bh * ctas_per_bh) * BM * NQ;
  const int64_t b = bh / p.H, h = bh - b * p.H;
  const int T = static_cast<int>(ceil_div(N, BN));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kKvFull + 0], 2);
    mbar_init(&bars[kKvFull + 1], 2);
    mbar_init(&bars[kKvEmpty + 0], 1);
    mbar_init(&bars[kKvEmpty + 1], 1);
    mbar_init(&bars[kQFull], 1);
    mbar_init(&bars[kDrain], 1);
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&bars[kSFull + q], 1);
      mbar_init(&bars[Bars<NQ>::pfull(q)], 4);
      mbar_init(&bars[Bars<NQ>::odone(q)], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmap_v);
  }
  if (threadIdx.x < 128)
    sscale[threadIdx.x] = (threadIdx.x < d) ? p.v_scale[bh * d + threadIdx.x] * (1.0f / 255.0f) : 0.0f;
  if (BK == BA_BIAS_RELPOS2D && tab_mode != 0) {
    const float* src = p.bias.data + h * static_cast<int64_t>(tsize);
    const int n = (tab_mode == 2) ? 3 * tsize : tsize;
    for (int e = threadIdx.x; e < n; e += C::kThreads) stab[e] = (e < tsize) ? __ldg(src + e) : 0.0f;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint4* qrows = reinterpret_cast<const uint4*>(p.bits_q) + bh * N;
    const uint4* krows = reinterpret_cast<const uint4*>(p.bits_k) + bh * N;
    for (int q = 0; q < NQ; ++q) expand_signs<DQ>(sQ + q * C::kQBytes, qrows, q0 + q * BM, N, d, lane);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kQFull]);
    const int W2 = 2 * p.bias.table_w - 1;
    int issued = 0;
    for (int t = 0; t < T; ++t) {
      const int s = t & 1;
      if (t >= 2 && !wait_warp(&bars[kKvEmpty + s], ((t >> 1) - 1) & 1, abort_flag)) break;
      issued = t + 1;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars[kKvFull + s], C::kVBytes);
        tma_load_4d(sV + s * C::kVBytes, &tmap_v, &bars[kKvFull + s], 0, t * BN, 0, static_cast<int>(bh));
      }
      expand_signs<DQ>(sK + s * C::kKBytes, krows, t * BN, N, d, lane);
      if (BK == BA_BIAS_RELPOS2D) {
#pragma unroll
        for (int u = 0; u < BN / 32; ++u) {
          const int j = lane + 32 * u, tok = t * BN + j;
          // Keys past N read a valid entry (their P is masked); prefix keys read the zeros
          // after the staged table (or are marked -1 for the general path).
          int v = (tab_mode == 2) ? -tsize : -1;
          if (tok >= N) {
            v = 0;
          } else if (tok >= p.bias.n_prefix) {
            const int tj = tok - p.bias.n_prefix;
            const int yj = tj / p.bias.grid_w;
            v = yj * W2 + (tj - yj * p.bias.grid_w);
          }
          koff[s * BN + j] = v;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kKvFull + s]);
    }
    // Leave no TMA copy in flight: wait (bounded, even after an abort) for the last two
    // stages this warp filled.
    for (int t = (issued > 2 ? issued - 2 : 0); t < issued; ++t)
      wait_bounded(&bars[kKvFull + (t & 1)], (t >> 1) & 1, abort_flag, false);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                (static_cast<uint32_t>(BM >> 4) << 24);
      const uint32_t idesc_pv = (2u << 4) | (0u << 7) | (1u << 10) | (1u << 16) |
                                (static_cast<uint32_t>(DP >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
      if (wait_bounded(&bars[kQFull], 0, abort_flag)) {
        tc_fence_after();
        for (int t = 0; t <= T; ++t) {
          if (t < T) {
            if (!wait_bounded(&bars[kKvFull + (t & 1)], (t >> 1) & 1, abort_flag)) break;
            tc_fence_after();
          }
          bool ok = true;
          for (int q = 0; q < NQ; ++q) {
            if (t > 0) {
              if (!wait_bounded(&bars[Bars<NQ>::pfull(q)], (t - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t vbase = smem_u32(sV + ((t - 1) & 1) * C::kVBytes);
#pragma unroll
              for (int kk = 0; kk < BN / 32; ++kk)
                mma_i8_ts(tmem + C::tO(q), tmem + C::tP(q) + 8 * kk, smem_desc(vbase + 512 * kk, 128, 2048),
                          idesc_pv, (t > 1 || kk > 0) ? 1u : 0u);
            }
            if (t < T) {
              const uint32_t qb = smem_u32(sQ + q * C::kQBytes), kb = smem_u32(sK + (t & 1) * C::kKBytes);
#pragma unroll
              for (int kk = 0; kk < DQ / 32; ++kk)
                mma_f8f6f4_ss(tmem + C::tS(q), smem_desc(qb + kk * 4096, 2048, 128),
                              smem_desc(kb + kk * 4096, 2048, 128), idesc_qk, kk > 0 ? 1u : 0u);
              tc_commit(&bars[kSFull + q]);
            } else {
              tc_commit(&bars[Bars<NQ>::odone(q)]);
            }
          }
          if (!ok) break;
          if (t > 0) tc_commit(&bars[kKvEmpty + ((t - 1) & 1)]);
        }
      }
      // Every MMA this thread issued has completed before tensor memory is released.
      tc_commit(&bars[kDrain]);
      wait_bounded(&bars[kDrain], 0, abort_flag, false);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroups
    const int q = (warp - 4) >> 2, w4 = warp & 3;
    const int r = w4 * 32 + lane;
    const int i = q0 + q * BM + r;
    const bool row_ok = i < N;
    const int ic = row_ok ? i : N - 1;  // rows past N read the bias of row N-1 (never stored)
    const uint32_t lane_base = static_cast<uint32_t>(w4 * 32) << 16;
    const uint32_t aS = tmem + lane_base + C::tS(q);
    const uint32_t aP = tmem + lane_base + C::tP(q);
    const uint32_t aO = tmem + lane_base + C::tO(q);
    const float alpha = __fmul_rn(__fmul_rn(p.softmax_scale, p.mu_q[bh]), p.mu_k[bh]);
    const float2 alpha2 = make_float2(alpha, alpha);

    // Bias addressing. Dense: this row of [H][N][N]. Rel-pos: b_ij = tab[a_i - koff_j], where
    // tab is the head's table (in shared memory when staged, followed by zeros that prefix
    // rows and prefix keys index into).
    const float* brow = nullptr;
    const float* tab = nullptr;
    int a_i = 0;
    if (BK == BA_BIAS_DENSE) brow = p.bias.data + b * p.bias.batch_stride + (h * N + ic) * N;
    if (BK == BA_BIAS_RELPOS2D) {
      const int W2 = 2 * p.bias.table_w - 1;
      tab = (tab_mode != 0) ? stab : p.bias.data + h * static_cast<int64_t>(2 * p.bias.table_h - 1) * W2;
      if (ic >= p.bias.n_prefix) {
        const int ti = ic - p.bias.n_prefix;
        const int yi = ti / p.bias.grid_w;
        a_i = (yi + p.bias.table_h - 1) * W2 + (ti - yi * p.bias.grid_w) + p.bias.table_w - 1;
      } else {
        a_i = (tab_mode == 2) ? tsize + kmax : -1;  // prefix row: zeros (or the slow path)
      }
    }
    // Fast path: full key blocks, no debug output, aligned dense rows, prefix handled by zeros.
    const bool fast_ok = (p.dbg_logits == nullptr) &&
                         (BK != BA_BIAS_DENSE || ((N & 3) == 0 && (p.bias.batch_stride & 3) == 0)) &&
                         (BK != BA_BIAS_RELPOS2D || p.bias.n_prefix == 0 || tab_mode == 2);

    float m = -CUDART_INF_F, l = 0.0f;
    float of[DP];
#pragma unroll
    for (int c = 0; c < DP; ++c) of[c] = 0.0f;
    bool alive = true;

    for (int t = 0; t < T && alive; ++t) {
      const int s = t & 1;
      const int nk = min(BN, N - t * BN);
      if (BK == BA_BIAS_RELPOS2D && !wait_warp(&bars[kKvFull + s], (t >> 1) & 1, abort_flag)) {
        alive = false;
        break;
      }
      if (!wait_warp(&bars[kSFull + q], t & 1, abort_flag)) {
        alive = false;
        break;
      }
      tc_fence_after();
      const int* ko = koff + s * BN;

      // Pass 1: s = alpha * x + b written back over S in TMEM; block max.
      float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
      if (fast_ok && nk == BN) {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float bv[32];
          if (BK == BA_BIAS_DENSE) {
            const float4* src = reinterpret_cast<const float4*>(brow + t * BN + 32 * c);
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
              const float4 v4 = __ldg(src + k4);
              bv[4 * k4] = v4.x; bv[4 * k4 + 1] = v4.y; bv[4 * k4 + 2] = v4.z; bv[4 * k4 + 3] = v4.w;
            }
          } else if (BK == BA_BIAS_RELPOS2D) {
            const int4* kv = reinterpret_cast<const int4*>(ko + 32 * c);
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
              const int4 o4 = kv[k4];
              bv[4 * k4] = tab[a_i - o4.x];
              bv[4 * k4 + 1] = tab[a_i - o4.y];
              bv[4 * k4 + 2] = tab[a_i - o4.z];
              bv[4 * k4 + 3] = tab[a_i - o4.w];
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) bv[u] = 0.0f;
          }
          uint32_t x[32];
          tmem_ld32(aS + 32 * c, x);
          tmem_ld_wait32(x);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float2 s2 = __ffma2_rn(alpha2, make_float2(__uint_as_float(x[2 * k]), __uint_as_float(x[2 * k + 1])),
                                         make_float2(bv[2 * k], bv[2 * k + 1]));
            x[2 * k] = __float_as_uint(s2.x);
            x[2 * k + 1] = __float_as_uint(s2.y);
            if (k & 1)
              mx1 = fmax3(mx1, s2.x, s2.y);
            else
              mx0 = fmax3(mx0, s2.x, s2.y);
          }
          tmem_st32(aS + 32 * c, x);
        }
      } else {
        // General path: a partial last block, prefix tokens without zero padding, unaligned
        // dense rows, or the debug logits.
        auto bias_of = [&](int j) -> float {
          if (BK == BA_BIAS_DENSE) return __ldg(brow + t * BN + j);
          if (BK == BA_BIAS_RELPOS2D) {
            const int kj = ko[j];
            return (a_i >= 0 && kj >= 0) ? tab[a_i - kj] : 0.0f;
          }
          return 0.0f;
        };
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t x[32];
          tmem_ld32(aS + 32 * c, x);
          tmem_ld_wait32(x);
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int j = 32 * c + u;
            float sv = -CUDART_INF_F;
            if (j < nk) {
              const float xf = __uint_as_float(x[u]);
              sv = __fmaf_rn(alpha, xf, bias_of(j));
              if (p.dbg_logits != nullptr && row_ok)
                p.dbg_logits[(bh * N + i) * N + t * BN + j] = __float2int_rn(xf);
            }
            mx0 = fmaxf(mx0, sv);
            x[u] = __float_as_uint(sv);
          }
          tmem_st32(aS + 32 * c, x);
        }
      }
      const float m_new = fmaxf(m, fmaxf(mx0, mx1));
      tmem_st_wait();

      // Pass 2: P~ = 2^((s - m) log2 e) (masked keys hold s = -inf: P~ = 0), row sum, codes -> TMEM.
      const float2 negm2 = make_float2(-m_new, -m_new);
      const float2 log2e2 = make_float2(kLog2e, kLog2e);
      const float2 c255 = make_float2(255.0f, 255.0f);
      const float2 magic2 = make_float2(12582912.0f, 12582912.0f);
      float2 lt2 = make_float2(0.0f, 0.0f);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t x[32];
        tmem_ld32(aS + 32 * c, x);
        tmem_ld_wait32(x);
        uint32_t pk[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          uint32_t y[4];
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int u = 4 * w + 2 * e2;
            // s - m first (exact near the max), then the scale to base 2.
            const float2 t2 = __fmul2_rn(
                __fadd2_rn(make_float2(__uint_as_float(x[u]), __uint_as_float(x[u + 1])), negm2), log2e2);
            const float2 p2 = make_float2(ex2_approx(t2.x), ex2_approx(t2.y));
            lt2 = __fadd2_rn(lt2, p2);
            // 255 P~ + 1.5 * 2^23: one rounding to the nearest integer (ties to even); the
            // integer sits in the low byte of the result (P~ <= 1).
            const float2 y2 = __ffma2_rn(p2, c255, magic2);
            y[2 * e2] = __float_as_uint(y2.x);
            y[2 * e2 + 1] = __float_as_uint(y2.y);
          }
          pk[w] = __byte_perm(__byte_perm(y[0], y[1], 0x0040), __byte_perm(y[2], y[3], 0x0040), 0x5410);
        }
        tmem_st8(aP + 8 * c, pk);
      }
      const float lt = lt2.x + lt2.y;
      const float ct = (m == -CUDART_INF_F) ? 0.0f : ex2_approx((m - m_new) * kLog2e);
      l = l * ct + lt;
      const bool flush = (t > 0) && (m_new > m);
      if (__any_sync(0xffffffffu, flush)) {
#pragma unroll
        for (int cc = 0; cc < DP / 16; ++cc) {
          uint32_t a[16];
          tmem_ld16(aO + 16 * cc, a);
          tmem_ld_wait16(a);
          if (flush) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              of[16 * cc + e] = (of[16 * cc + e] + __int2float_rn(static_cast<int>(a[e]))) * ct;
              a[e] = 0u;
            }
          }
          tmem_st16(aO + 16 * cc, a);
        }
      }
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Bars<NQ>::pfull(q)]);
    }

    if (alive && wait_warp(&bars[Bars<NQ>::odone(q)], 0, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
#pragma unroll
      for (int cc = 0; cc < DP / 16; ++cc) {
        uint32_t a[16];
        tmem_ld16(aO + 16 * cc, a);
        tmem_ld_wait16(a);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = 16 * cc + e;
          if (row_ok && c < d) {
            const float val = (of[c] + __int2float_rn(static_cast<int>(a[e]))) * sscale[c] * inv_l;
            store_out(p.o, (bh * N + i) * d + c, val, p.o_dt);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  if (warp != 2 && warp != 3) {
    tc_fence_before();
    named_barrier_sync(1, C::kThreads - 64);
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

constexpr int kMaxSmem = 227 * 1024;

template <int DP, int BK>
cudaError_t launch_dp_bk(const AttnParams& p, const CUtensorMap& tm, cudaStream_t s) {
  using C = Cfg<DP>;
  int tab_mode = 0, tsize = 0, kmax = 0;
  if (BK == BA_BIAS_RELPOS2D) {
    tsize = (2 * p.bias.table_h - 1) * (2 * p.bias.table_w - 1);
    kmax = (p.bias.grid_h - 1) * (2 * p.bias.table_w - 1) + p.bias.grid_w - 1;
    const int64_t room = kMaxSmem - 1024 - C::kTabOff;
    if (p.bias.n_prefix > 0 && 3ll * tsize * 4 <= room)
      tab_mode = 2;
    else if (static_cast<int64_t>(tsize) * 4 <= room)
      tab_mode = 1;
  }
  const int tab_bytes = tab_mode == 0 ? 0 : (tab_mode == 2 ? 3 : 1) * tsize * 4;
  // At least 116 KB of shared memory per CTA keeps one CTA per SM (it owns all 512 TMEM columns).
  int smem = C::kTabOff + tab_bytes + 1024;
  if (smem < 116 * 1024) smem = 116 * 1024;
  static int configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DP, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  const int64_t grid = static_cast<int64_t>(p.B) * p.H * ceil_div(p.N, BM * C::NQ);
  attn_tc_kernel<DP, BK><<<static_cast<unsigned>(grid), C::kThreads, smem, s>>>(p, tm, tab_mode, tsize, kmax);
  return cudaGetLastError();
}

template <int DP>
cudaError_t launch_dp(const AttnParams& p, const CUtensorMap& tm, cudaStream_t s) {
  switch (p.bias.kind) {
    case BA_BIAS_DENSE: return launch_dp_bk<DP, BA_BIAS_DENSE>(p, tm, s);
    case BA_BIAS_RELPOS2D: return launch_dp_bk<DP, BA_BIAS_RELPOS2D>(p, tm, s);
    default: return launch_dp_bk<DP, BA_BIAS_NONE>(p, tm, s);
  }
}

}  // namespace

bool attn_tc_supported(const AttnParams& p) {
  return p.dp >= 16 && p.dp <= 128 && (p.dp % 16) == 0 && p.N >= 1 && encode_fn() != nullptr;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  // V [BH][N][dp] int8 viewed as 4-D (16 bytes, key, 16-byte chunk, bh) so that a box of
  // (16, 128, dp/16, 1) lands as [chunk][key][16 B]: the MN-major core-matrix layout.
  CUtensorMap tm;
  const cuuint64_t dims[4] = {16, static_cast<cuuint64_t>(p.N), static_cast<cuuint64_t>(p.dp / 16),
                              static_cast<cuuint64_t>(p.B) * p.H};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(p.dp), 16,
                                 static_cast<cuuint64_t>(p.N) * static_cast<cuuint64_t>(p.dp)};
  const cuuint32_t box[4] = {16, static_cast<cuuint32_t>(BN), static_cast<cuuint32_t>(p.dp / 16), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<int8_t*>(p.vq), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  switch (p.dp) {
    case 16: return launch_dp<16>(p, tm, s);
    case 32: return launch_dp<32>(p, tm, s);
    case 48: return launch_dp<48>(p, tm, s);
    case 64: return launch_dp<64>(p, tm, s);
    case 80: return launch_dp<80>(p, tm, s);
    case 96: return launch_dp<96>(p, tm, s);
    case 112: return launch_dp<112>(p, tm, s);
    case 128: return launch_dp<128>(p, tm, s);
    default: return cudaErrorNotSupported;
  }
}

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
