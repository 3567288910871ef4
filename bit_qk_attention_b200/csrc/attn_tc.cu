// Fused BinaryAttention forward on 5th-generation tensor cores (sm_100a: tcgen05 + TMEM + TMA).
//
// What it computes is the blockwise forward of the CUDA-core kernel (attn_simt.cu) and of the
// CPU reference: binary QK (gist.science/zh technical summary 2.1-2.2(1)), bias b_ij (2.2(2)),
// FlashAttention-2-style online softmax over ascending 128-key blocks (2.3), 8-bit P on [0,1]
// (2.2(3)), per-channel int8 V and an integer P.V (the u8 x s8 -> s32 instruction class named
// on every page).
//
// How, on B200:
//   * A work item is NQ query tiles of 128 rows of one (b, h): one tile in 256 tensor-memory
//     columns (two CTAs per SM) when the head and the bias table fit, else two tiles in 512.
//     For heads up to 80 channels the CTAs are persistent (as many as fit at once): each walks
//     a list of items, grouped by head when the head's rel-pos table is staged, while its
//     producers and MMA thread run ahead into the next item (the K/V ring continues across
//     items; consecutive items start on alternate P.V accumulators, so an item's epilogue
//     overlaps the next item's first MMAs). Wider heads run one item per CTA
//     (attn_tc_single_kernel), which measured faster there.
//   * Warps 2 and 3 expand the 1-bit sign rows of Q (once) and of each K block into fp8 +-1
//     operands in shared memory (channels >= d become 0); warp 0 TMA-loads the int8 V block
//     (a 4-D tensor map that lands it in the MN-major core-matrix layout the MMA reads) and
//     writes the block's rel-pos key offsets. A 4-stage ring of K/V blocks decouples them from
//     the MMAs.
//   * Warp 1 issues the MMAs from one thread:
//       S  = Q . K^T   tcgen05.mma kind::f8f6f4 (e4m3 +-1, fp32 accumulate: exact integers)
//       O += P . V     tcgen05.mma kind::i8, A = the uint8 codes read from TMEM, B = int8 V
//     both accumulators live in tensor memory.
//   * Warpgroup 1+q (one thread per query row) runs the softmax of query tile q: it reads its
//     row of S from TMEM, forms s = fmaf(alpha, x, b), the running max, P~ = 2^((s-m) log2 e),
//     the row sum, and writes the 8-bit codes back to TMEM as the A operand of P.V.
//   * The int32 P.V accumulator keeps accumulating across key blocks while no row of the tile
//     raises its running max (every rescale factor is exactly 1 then). When a row's max rises,
//     P.V of that block starts the tile's second accumulator instead, and while the MMAs run
//     the softmax threads fold the first one into their fp32 running outputs,
//     O~ = (O~ + acc) * exp(m_old - m_new) (factor 1 for rows whose max did not rise). This is
//     the same arithmetic as rescaling every block, off the softmax's critical path.
//   * Every wait is bounded (1 s): on expiry the kernel records BA_ERR_TIMEOUT in a device
//     status word, every role leaves its loop, and the CTA frees its tensor memory.
#include <cuda.h>
#include <math_constants.h>

#include <algorithm>
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

template <int DP, int NQ_>
struct Cfg {
  static constexpr int DQ = (DP + 31) / 32 * 32;   // QK contraction width: fp8 K-steps of 32
  static constexpr int NQ = NQ_;                    // query tiles per CTA
  static constexpr int kThreads = 128 + 128 * NQ;   // 4 service warps + NQ softmax warpgroups
  // The fp32 running output F of a row lives in shared memory for heads up to 64 wide (tensor
  // memory then holds S and two accumulators per tile), else in tensor memory.
  static constexpr bool kFSmem = DP <= 64;
  static constexpr int kQBytes = BM * DQ;
  static constexpr int kKBytes = BN * DQ;
  static constexpr int kVBytes = BN * DP;
  static constexpr int kStages = (NQ == 1 && DP <= 64) ? 3 : 4;  // K/V pipeline depth
  static constexpr int offQ = 0;
  static constexpr int offK = offQ + NQ * kQBytes;
  static constexpr int offV = offK + kStages * kKBytes;
  static constexpr int offKoff = offV + kStages * kVBytes;
  static constexpr int offScale = offKoff + kStages * BN * 4;  // V scales (single-item kernel)
  static constexpr int offBar = offScale + 128 * 4;
  static constexpr int kNumBars = 2 * kStages + 3 + 3 * NQ;
  static constexpr int offMisc = offBar + kNumBars * 8;           // tmem base, abort flag
  static constexpr int offVotes = offMisc + 16;                    // [2][NQ][4] u32
  static constexpr int offF = (offVotes + 2 * NQ * 4 * 4 + 15) / 16 * 16;
  static constexpr int kFBytes = kFSmem ? NQ * BM * DP * 4 : 0;   // [DP/4][NQ*128] float4
  static constexpr int kBytes = offF + kFBytes;
  static constexpr int kTabOff = (kBytes + 127) / 128 * 128;
  // Tensor-memory columns of query tile q: S (fp32, 128 columns; the softmax overwrites it
  // with s and then its first 32 columns with the u8 codes P — the MMAs of one CTA run in
  // issue order, so P.V reads P before the next QK rewrites S), two s32 P.V accumulators
  // O0/O1 (DP each: P.V switches to the other one when a row's max rises, while the softmax
  // threads fold the first into F) and, for wide heads, F (fp32, DP).
  __host__ __device__ static constexpr uint32_t tS(int q) { return q * 256; }
  __host__ __device__ static constexpr uint32_t tP(int q) { return q * 256; }
  __host__ __device__ static constexpr uint32_t tO(int q, int b) { return q * 256 + 128 + b * DP; }
  __host__ __device__ static constexpr uint32_t tF(int q) { return q * 256 + 128 + 2 * DP; }
  static constexpr int kTmemUsed = tO(NQ - 1, 1) + DP + (kFSmem ? 0 : DP);
  static_assert(kTmemUsed <= 512, "tensor memory budget");
  static_assert(NQ == 1 || kFSmem, "two tiles per CTA need F in shared memory");
  // Columns allocated: a CTA whose tiles fit in half of tensor memory takes 256 columns and
  // shares its SM with a second CTA.
  static constexpr int kTmemCols = kTmemUsed <= 256 ? 256 : 512;
  static constexpr int kCtasPerSm = 512 / kTmemCols;
};

// Barrier slots: kv_full[S], kv_empty[S], q_full, q_empty, drain, s_full[NQ], p_full[NQ],
// o_done[NQ]. Phases count K/V blocks (kv_*: per stage; s_full, p_full: per block) or work
// items (q_*, o_done) across all the items a CTA processes.
template <int S, int NQ> struct Bars {
  __host__ __device__ static constexpr int kvfull(int s) { return s; }
  __host__ __device__ static constexpr int kvempty(int s) { return S + s; }
  __host__ __device__ static constexpr int qfull() { return 2 * S; }
  __host__ __device__ static constexpr int qempty() { return 2 * S + 1; }
  __host__ __device__ static constexpr int drain() { return 2 * S + 2; }
  __host__ __device__ static constexpr int sfull(int q) { return 2 * S + 3 + q; }
  __host__ __device__ static constexpr int pfull(int q) { return 2 * S + 3 + NQ + q; }
  __host__ __device__ static constexpr int odone(int q) { return 2 * S + 3 + 2 * NQ + q; }
};

// Work items: NQ query tiles of one (b, h). With the head's rel-pos table staged in shared
// memory (by_head), the CTAs of head h are h, h + H, h + 2H, ... (gridDim.x = H * k) and CTA j
// of head h takes items j, j + k, j + 2k, ... of the B * nqb items of that head (nqb = query
// blocks per (b, h)), so the table is staged once. Otherwise CTA c takes items c, c + G,
// c + 2G, ... of all B * H * nqb items (G = gridDim.x), item m covering query block m % nqb of
// slice m / nqb. Recomputed from the launch geometry where needed.
__device__ __forceinline__ int item_count(bool by_head, int B, int H, int nqb) {
  const int total = by_head ? B * nqb : B * H * nqb;
  const int first = by_head ? static_cast<int>(blockIdx.x) / H : static_cast<int>(blockIdx.x);
  const int stride = by_head ? static_cast<int>(gridDim.x) / H : static_cast<int>(gridDim.x);
  return first < total ? (total - first + stride - 1) / stride : 0;
}

__device__ __forceinline__ void item_at(bool by_head, int it, int H, int nqb, int rows_per_item, int64_t& bh,
                                        int& q0) {
  if (by_head) {
    const int m = static_cast<int>(blockIdx.x) / H + it * (static_cast<int>(gridDim.x) / H);
    const int b = m / nqb;
    bh = static_cast<int64_t>(b) * H + static_cast<int>(blockIdx.x) % H;
    q0 = (m - b * nqb) * rows_per_item;
  } else {
    const int64_t m = static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(it) * gridDim.x;
    bh = m / nqb;
    q0 = static_cast<int>(m - bh * nqb) * rows_per_item;
  }
}

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

// One 1-bit sign row -> fp8 e4m3 +-1 (bit 1 = negative) in the K-major no-swizzle core-matrix
// layout: byte (row r, channel c) at (c/16)*2048 + r*16 + c%16. Channels >= d, and rows past
// the end (ok = false), are 0 so they add nothing to the dot products.
template <int DQ>
__device__ __forceinline__ void expand_row(uint8_t* dst, const uint4& b, bool ok, int r, int d) {
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

// Bias variants of the kernel: BA_BIAS_NONE, BA_BIAS_DENSE, BA_BIAS_RELPOS2D with the head's
// table staged in shared memory, and kRelposGlobal with the table read from global memory.
constexpr int kRelposGlobal = 3;
__host__ __device__ constexpr bool is_relpos(int bk) { return bk == BA_BIAS_RELPOS2D || bk == kRelposGlobal; }

// Fast path of pass 1 for one 32-key block of one row: bias (dense row, or rel-pos table in
// shared or global memory), s = alpha * x + b in place, running maxima. PARTIAL masks keys
// at or past nk to -inf.
template <int BK, bool PARTIAL>
__device__ __forceinline__ void fast_block(uint32_t (&x)[32], int c, int nk, float2 alpha2, const float* brow_t,
                                           uint32_t ko_s, uint32_t tb, const float* grow, int tab_mode,
                                           float (&mx)[4]) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float bv[8];
    if (BK == BA_BIAS_DENSE) {
      const float4* src = reinterpret_cast<const float4*>(brow_t + 32 * c + 8 * g);
      const float4 v0 = __ldg(src), v1 = __ldg(src + 1);
      bv[0] = v0.x; bv[1] = v0.y; bv[2] = v0.z; bv[3] = v0.w;
      bv[4] = v1.x; bv[5] = v1.y; bv[6] = v1.z; bv[7] = v1.w;
    } else if (is_relpos(BK)) {
      const int4 o0 = lds_s32x4(ko_s + 4u * (32 * c + 8 * g));
      const int4 o1 = lds_s32x4(ko_s + 4u * (32 * c + 8 * g + 4));
      if (BK == BA_BIAS_RELPOS2D) {
        bv[0] = lds_f32(tb - o0.x); bv[1] = lds_f32(tb - o0.y);
        bv[2] = lds_f32(tb - o0.z); bv[3] = lds_f32(tb - o0.w);
        bv[4] = lds_f32(tb - o1.x); bv[5] = lds_f32(tb - o1.y);
        bv[6] = lds_f32(tb - o1.z); bv[7] = lds_f32(tb - o1.w);
      } else {
        bv[0] = __ldg(grow - (o0.x >> 2)); bv[1] = __ldg(grow - (o0.y >> 2));
        bv[2] = __ldg(grow - (o0.z >> 2)); bv[3] = __ldg(grow - (o0.w >> 2));
        bv[4] = __ldg(grow - (o1.x >> 2)); bv[5] = __ldg(grow - (o1.y >> 2));
        bv[6] = __ldg(grow - (o1.z >> 2)); bv[7] = __ldg(grow - (o1.w >> 2));
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) bv[u] = 0.0f;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int u = 8 * g + 2 * k;
      const float2 s2 = __ffma2_rn(alpha2, make_float2(__uint_as_float(x[u]), __uint_as_float(x[u + 1])),
                                   make_float2(bv[2 * k], bv[2 * k + 1]));
      float sx = s2.x, sy = s2.y;
      if (PARTIAL) {
        if (32 * c + u >= nk) sx = -CUDART_INF_F;
        if (32 * c + u + 1 >= nk) sy = -CUDART_INF_F;
      }
      x[u] = __float_as_uint(sx);
      x[u + 1] = __float_as_uint(sy);
      mx[k] = fmax3(mx[k], sx, sy);
    }
  }
}

// 2^t for a pair of t <= 0 on the FMA and integer pipes, for the share of the softmax's
// exponentials that the transcendental unit (which computes the rest, and is the softmax's
// bottleneck) does not take. t is clamped to -125 (2^-125: a u8 code of 0, a negligible
// addition to the row sum; masked keys arrive as -inf); j = rint(t) by adding and subtracting
// 1.5 * 2^23, f = t - j in [-1/2, 1/2]; 2^f by a degree-5 polynomial with c0 = 1 (a weighted
// least-squares fit in relative error on Chebyshev nodes, bit_qk_attention_b200/exp2_poly.py;
// at most 1.6e-7 relative error in float32); 2^j is added to the exponent bits: the bit
// pattern of t + 1.5 * 2^23 holds j in its low bits, and shifted left by 23 it is j << 23.
__device__ __forceinline__ float2 exp2_poly2(float2 t) {
  t.x = fmaxf(t.x, -125.0f);
  t.y = fmaxf(t.y, -125.0f);
  const float2 r = __fadd2_rn(t, make_float2(12582912.0f, 12582912.0f));
  const float2 j = __fadd2_rn(r, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), t);
  float2 q = __ffma2_rn(make_float2(1.321867225e-03f, 1.321867225e-03f), f,
                        make_float2(9.671698324e-03f, 9.671698324e-03f));
  q = __ffma2_rn(q, f, make_float2(5.550893024e-02f, 5.550893024e-02f));
  q = __ffma2_rn(q, f, make_float2(2.402223796e-01f, 2.402223796e-01f));
  q = __ffma2_rn(q, f, make_float2(6.931468844e-01f, 6.931468844e-01f));
  q = __ffma2_rn(q, f, make_float2(1.0f, 1.0f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(r.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(r.y) << 23)));
}

// Pairs (of the 16 in a 32-key chunk) whose exponentials take the polynomial: the bits of
// kPolyPairs, spread over the chunk. Off by default: a quarter measured 2-4 % faster on B200,
// but any fast exponential can move a u8 code across a rounding tie relative to the exact
// exp(s - m), and which codes move depends on the mix; the default keeps one implementation
// (the hardware ex2) for every logit.
#ifndef BA_POLY_PAIRS
#define BA_POLY_PAIRS 0x0u
#endif
constexpr uint32_t kPolyPairs = BA_POLY_PAIRS;

// Folding an s32 P.V accumulator row into the fp32 running output of the row:
// F = (F + acc) * ct, in groups of NC chunks of 16 columns starting at chunk C0. fold_load
// issues a group's tensor-memory loads (the accumulator, and F when it lives in tensor
// memory); fold_finish waits for them and completes the group. `fresh`: F holds nothing yet
// (read as 0). `one_block`: the accumulator holds a single block's P.V,
// |acc| <= 255 * 127 * 128 < 2^22, which converts exactly by adding it to the bit pattern of
// 1.5 * 2^23 and subtracting that value as a float; otherwise the hardware conversion is used.
// F lives in shared memory ([DP/4][NQ*128] float4, `fr` = this row's first entry) or in tensor
// memory (`aF`).
template <class C>
struct FoldShape {
  static constexpr int NCH = C::kVBytes / BN / 16;  // chunks per row
  // 2 chunks (32 columns) per group when F is in shared memory (those CTAs share an SM: 128
  // 2 chunks (32 columns) per group when F is in shared memory (those CTAs share an SM: 128
  // registers per thread), 4 when it is in tensor memory (one CTA per SM).
  static constexpr int G = C::kFSmem ? 2 : 4;
  __host__ __device__ static constexpr int nc(int c0) { return (NCH - c0 < G) ? NCH - c0 : G; }
};

template <class C, int C0, int NC>
__device__ __forceinline__ void fold_load(uint32_t acc, uint32_t aF, bool fresh, uint32_t (&a)[NC][16],
                                          uint32_t (&fb)[NC][16]) {
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    tmem_ld16(acc + 16 * (C0 + k), a[k]);
    if (!C::kFSmem && !fresh) tmem_ld16(aF + 16 * (C0 + k), fb[k]);
  }
}

template <class C, int C0, int NC>
__device__ __forceinline__ void fold_finish(uint32_t aF, float4* fr, float2 ct2, bool fresh, bool one_block,
                                            uint32_t (&a)[NC][16], uint32_t (&fb)[NC][16]) {
  tmem_ld_wait();
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    reg_fence16(a[k]);
    if (!C::kFSmem && !fresh) reg_fence16(fb[k]);
  }
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    float f[16];
    if constexpr (C::kFSmem) {
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const float4 v = fresh ? make_float4(0.0f, 0.0f, 0.0f, 0.0f) : fr[(4 * (C0 + k) + k4) * (C::NQ * BM)];
        f[4 * k4] = v.x; f[4 * k4 + 1] = v.y; f[4 * k4 + 2] = v.z; f[4 * k4 + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) f[e] = fresh ? 0.0f : __uint_as_float(fb[k][e]);
    }
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      float2 av;
      if (one_block) {
        av = __fadd2_rn(make_float2(__uint_as_float(a[k][e] + 0x4B400000u), __uint_as_float(a[k][e + 1] + 0x4B400000u)),
                        make_float2(-12582912.0f, -12582912.0f));
      } else {
        av = make_float2(__int2float_rn(static_cast<int>(a[k][e])), __int2float_rn(static_cast<int>(a[k][e + 1])));
      }
      const float2 v = __fmul2_rn(__fadd2_rn(make_float2(f[e], f[e + 1]), av), ct2);
      f[e] = v.x; f[e + 1] = v.y;
    }
    if constexpr (C::kFSmem) {
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4)
        fr[(4 * (C0 + k) + k4) * (C::NQ * BM)] = make_float4(f[4 * k4], f[4 * k4 + 1], f[4 * k4 + 2], f[4 * k4 + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) fb[k][e] = __float_as_uint(f[e]);
      tmem_st16(aF + 16 * (C0 + k), fb[k]);
    }
  }
}

// The groups from chunk C0 to the end of the row.
template <class C, int C0>
__device__ __forceinline__ void fold_rest(uint32_t acc, uint32_t aF, float4* fr, float2 ct2, bool fresh,
                                          bool one_block) {
  if constexpr (C0 < FoldShape<C>::NCH) {
    constexpr int NC = FoldShape<C>::nc(C0);
    uint32_t a[NC][16], fb[NC][16];
    fold_load<C, C0, NC>(acc, aF, fresh, a, fb);
    fold_finish<C, C0, NC>(aF, fr, ct2, fresh, one_block, a, fb);
    fold_rest<C, C0 + NC>(acc, aF, fr, ct2, fresh, one_block);
  }
}

template <int DP, int BK, int NQ_>
__global__ void __launch_bounds__(Cfg<DP, NQ_>::kThreads, Cfg<DP, NQ_>::kCtasPerSm)
    attn_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmap_v, int tab_mode, int tsize,
                   int kmax) {
  using C = Cfg<DP, NQ_>;
  constexpr int NQ = C::NQ, DQ = C::DQ, S = C::kStages;
  using Bar = Bars<S, NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::offQ;
  uint8_t* sK = smem + C::offK;
  uint8_t* sV = smem + C::offV;
  int* koff = reinterpret_cast<int*>(smem + C::offKoff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::offBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::offMisc + 4);
  // Per block parity, tile and softmax warp: whether a row of that warp raised its max.
  uint32_t* votes = reinterpret_cast<uint32_t*>(smem + C::offVotes);
  float4* sF = reinterpret_cast<float4*>(smem + C::offF);  // [DP/4][NQ*128]
  // Rel-pos table of this CTA's head, staged when it fits: tab_mode 1 = table only,
  // 2 = table followed by 2*tsize zeros (targets of prefix rows and prefix keys).
  float* stab = reinterpret_cast<float*>(smem + C::kTabOff);

  const int N = p.N, d = p.d;
  const int nqb = static_cast<int>(ceil_div(N, BM * NQ));
  // Items grouped by head when the head's rel-pos table is staged in shared memory.
  const bool by_head = is_relpos(BK) && tab_mode != 0;
  const int n_items = item_count(by_head, p.B, p.H, nqb);
  const int T = static_cast<int>(ceil_div(N, BN));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int st = 0; st < C::kStages; ++st) {
      // kv_full: the V copy's expect_tx arrival + warp 0 (key offsets) + the two expanding warps.
      mbar_init(&bars[Bar::kvfull(st)], 4);
      mbar_init(&bars[Bar::kvempty(st)], 1);
    }
    mbar_init(&bars[Bar::qfull()], 2);
    mbar_init(&bars[Bar::qempty()], 1);
    mbar_init(&bars[Bar::drain()], 1);
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&bars[Bar::sfull(q)], 1);
      mbar_init(&bars[Bar::pfull(q)], 4);
      mbar_init(&bars[Bar::odone(q)], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmap_v);
  }
  // Everything above reads only the caller's inputs; from here on the kernel reads the sign
  // rows, mu and int8 V, which the preparation kernel before it in the stream may still be
  // writing when this kernel was launched as its programmatic dependent.
  grid_dependency_wait();
  // Warps 2 and 3 load the sign rows of their Q rows and of key block 0 of the first item
  // before the setup barrier, so the loads overlap the setup.
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  uint4 pre_q[NQ][2], pre_k[2];
  if ((warp == 2 || warp == 3) && n_items > 0) {
    const int half = warp - 2;
    int64_t bh;
    int q0;
    item_at(by_head, 0, p.H, nqb, BM * NQ, bh, q0);
    const uint4* qrows = reinterpret_cast<const uint4*>(p.bits_q) + bh * N;
    const uint4* krows = reinterpret_cast<const uint4*>(p.bits_k) + bh * N;
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int row = q0 + q * BM + 64 * half + lane + 32 * u;
        pre_q[q][u] = row < N ? __ldg(qrows + row) : zero4;
      }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int row = 64 * half + lane + 32 * u;
      pre_k[u] = row < N ? __ldg(krows + row) : zero4;
    }
  }
  if (by_head) {
    const float* src = p.bias.data + static_cast<int64_t>(blockIdx.x % p.H) * tsize;
    const int n = (tab_mode == 2) ? 3 * tsize : tsize;
    for (int e = threadIdx.x; e < n; e += C::kThreads) stab[e] = (e < tsize) ? __ldg(src + e) : 0.0f;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer: V blocks, key offsets
    // Blocks are counted across the items (g): stage g % S, phase g / S.
    const int W2 = 2 * p.bias.table_w - 1;
    int g = 0;
    bool ok = true;
    for (int it = 0; it < n_items && ok; ++it) {
      int64_t bh;
      int q0;
      item_at(by_head, it, p.H, nqb, BM * NQ, bh, q0);
      for (int t = 0; t < T; ++t, ++g) {
        const int st = g % S;
        if (g >= S && !wait_warp(&bars[Bar::kvempty(st)], ((g / S) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars[Bar::kvfull(st)], C::kVBytes);
          tma_load_4d(sV + st * C::kVBytes, &tmap_v, &bars[Bar::kvfull(st)], 0, t * BN, 0, static_cast<int>(bh));
        }
        if (is_relpos(BK)) {
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
            koff[st * BN + j] = 4 * v;  // byte offset into the staged table
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Bar::kvfull(st)]);
      }
    }
    // Leave no TMA copy in flight: wait (bounded, even after an abort) for the stages this
    // warp filled last.
    for (int k = (g > S ? g - S : 0); k < g; ++k) wait_bounded(&bars[Bar::kvfull(k % S)], (k / S) & 1, abort_flag, false);
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ producer: sign expansion
    // Warp 2 expands rows 0..63 and warp 3 rows 64..127 of every Q tile and K block. The sign
    // rows of the next K block are loaded into registers before this block is written. The Q
    // tiles of an item are written once the MMAs of the previous item have read them (q_empty).
    const int half = warp - 2;
    int g = 0;
    bool ok = true;
    uint4 nb[2] = {pre_k[0], pre_k[1]};
    for (int it = 0; it < n_items && ok; ++it) {
      int64_t bh;
      int q0;
      item_at(by_head, it, p.H, nqb, BM * NQ, bh, q0);
      if (it > 0) {
        const uint4* qrows = reinterpret_cast<const uint4*>(p.bits_q) + bh * N;
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int row = q0 + q * BM + 64 * half + lane + 32 * u;
            pre_q[q][u] = row < N ? __ldg(qrows + row) : zero4;
          }
        if (!wait_warp(&bars[Bar::qempty()], (it - 1) & 1, abort_flag)) break;
      }
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int u = 0; u < 2; ++u)
          expand_row<DQ>(sQ + q * C::kQBytes, pre_q[q][u], q0 + q * BM + 64 * half + lane + 32 * u < N,
                         64 * half + lane + 32 * u, d);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Bar::qfull()]);
      for (int t = 0; t < T; ++t, ++g) {
        const int st = g % S;
        const uint4 cb[2] = {nb[0], nb[1]};
        // Sign rows of the next K block: this item's next block, or block 0 of the next item.
        {
          int64_t nbh = bh;
          int nt = t + 1;
          bool any = true;
          if (nt == T) {
            nt = 0;
            if (it + 1 < n_items) {
              int nq0;
              item_at(by_head, it + 1, p.H, nqb, BM * NQ, nbh, nq0);
            } else {
              any = false;
            }
          }
          const uint4* nrows = reinterpret_cast<const uint4*>(p.bits_k) + nbh * N;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int row = nt * BN + 64 * half + lane + 32 * u;
            nb[u] = (any && row < N) ? __ldg(nrows + row) : zero4;
          }
        }
        if (g >= S && !wait_warp(&bars[Bar::kvempty(st)], ((g / S) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int r = 64 * half + lane + 32 * u;
          expand_row<DQ>(sK + st * C::kKBytes, cb[u], t * BN + r < N, r, d);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Bar::kvfull(st)]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per block n (counted across items): P.V of block n-1 first (it needs no new operands),
    // then QK of block n into the same S columns (issue order keeps P read before S is
    // rewritten). The first P.V of an item starts the tile's other accumulator, so the previous
    // item's epilogue can still read the one it ended in.
    if (lane == 0) {
      const uint32_t idesc_qk = (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                (static_cast<uint32_t>(BM >> 4) << 24);
      const uint32_t idesc_pv = (2u << 4) | (0u << 7) | (1u << 10) | (1u << 16) |
                                (static_cast<uint32_t>(DP >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
      bool ok = true;
      uint32_t cur_acc = (1u << NQ) - 1u;  // bit q: the accumulator P.V of tile q adds into
      const int nblocks = n_items * T;
      // Step n: P.V of block n - 1 (if n > 0), then QK of block n (if n < nblocks); t is the
      // item-relative index of block n.
      for (int n = 0, it = 0, t = 0; n <= nblocks && ok; ++n) {
        if (n < nblocks && t == 0) {
          if (!wait_bounded(&bars[Bar::qfull()], it & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const int tp = (t == 0 ? T : t) - 1;  // item-relative index of block n - 1
        for (int q = 0; q < NQ && ok; ++q) {
          if (n > 0) {
            if (!wait_bounded(&bars[Bar::pfull(q)], (n - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // Switch to the other accumulator (overwriting it) at an item's first block and
            // when a row of the tile raised its max: the softmax warps' votes, written before
            // their p_full arrivals.
            bool fresh = tp == 0;
            if (!fresh) {
              const volatile uint32_t* vt = votes + (((n - 1) & 1) * NQ + q) * 4;
              fresh = (vt[0] | vt[1] | vt[2] | vt[3]) != 0u;
            }
            if (fresh) cur_acc ^= 1u << q;
            const uint32_t acc = tmem + C::tO(q, (cur_acc >> q) & 1u);
            const uint32_t vbase = smem_u32(sV + ((n - 1) % S) * C::kVBytes);
#pragma unroll
            for (int kk = 0; kk < BN / 32; ++kk)
              mma_i8_ts(acc, tmem + C::tP(q) + 8 * kk, smem_desc(vbase + 512 * kk, 128, 2048), idesc_pv,
                        (fresh && kk == 0) ? 0u : 1u);
            if (tp == T - 1) tc_commit(&bars[Bar::odone(q)]);
          }
          if (n < nblocks) {
            if (q == 0) {
              if (!wait_bounded(&bars[Bar::kvfull(n % S)], (n / S) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const uint32_t qb = smem_u32(sQ + q * C::kQBytes), kb = smem_u32(sK + (n % S) * C::kKBytes);
#pragma unroll
            for (int kk = 0; kk < DQ / 32; ++kk)
              mma_f8f6f4_ss(tmem + C::tS(q), smem_desc(qb + kk * 4096, 2048, 128),
                            smem_desc(kb + kk * 4096, 2048, 128), idesc_qk, kk > 0 ? 1u : 0u);
            tc_commit(&bars[Bar::sfull(q)]);
          }
        }
        if (!ok) break;
        if (n > 0) tc_commit(&bars[Bar::kvempty((n - 1) % S)]);
        // The item's Q tiles are free once its last QKs have read them.
        if (n < nblocks && t == T - 1) tc_commit(&bars[Bar::qempty()]);
        if (++t == T) {
          t = 0;
          ++it;
        }
      }
      // Every MMA this thread issued has completed before tensor memory is released.
      tc_commit(&bars[Bar::drain()]);
      wait_bounded(&bars[Bar::drain()], 0, abort_flag, false);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroups
    const int q = (warp - 4) >> 2, w4 = warp & 3;
    const int r = w4 * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(w4 * 32) << 16;
    const uint32_t aS = tmem + lane_base + C::tS(q);
    const uint32_t aP = tmem + lane_base + C::tP(q);
    const uint32_t aO0 = tmem + lane_base + C::tO(q, 0);
    const uint32_t aO1 = tmem + lane_base + C::tO(q, 1);
    const uint32_t aF = tmem + lane_base + C::tF(q);  // unused when F is in shared memory
    // Fast path: full key blocks, no debug output, aligned dense rows, rel-pos table in shared
    // memory with the class tokens handled by the zero padding.
    const bool fast_ok = (p.dbg_logits == nullptr) &&
                         (BK != BA_BIAS_DENSE || ((N & 3) == 0 && (p.bias.batch_stride & 3) == 0)) &&
                         (!is_relpos(BK) || p.bias.n_prefix == 0 || tab_mode == 2);
    bool alive = true;
    // Accumulator that P.V of the current block adds into (tile-uniform): every item starts on
    // the other one, as the MMA thread does.
    int cur = 1;
    float mu_q_next = 0.0f, mu_k_next = 0.0f;  // mu of the item about to start (loaded one item ahead)
    int n0 = 0;  // index, counted across items, of the item's first key block
    for (int it = 0; it < n_items && alive; ++it, n0 += T) {
    int64_t bh;
    int q0;
    item_at(by_head, it, p.H, nqb, BM * NQ, bh, q0);
    const int64_t b = bh / p.H, h = bh - b * p.H;
    const int i = q0 + q * BM + r;
    const bool row_ok = i < N;
    const int ic = row_ok ? i : N - 1;  // rows past N read the bias of row N-1 (never stored)
    if (it == 0) {
      mu_q_next = p.mu_q[bh];
      mu_k_next = p.mu_k[bh];
    }
    const float alpha = __fmul_rn(__fmul_rn(p.softmax_scale, mu_q_next), mu_k_next);
    const float2 alpha2 = make_float2(alpha, alpha);

    // Bias addressing. Dense: this row of [H][N][N]. Rel-pos: b_ij = tab[a_i - koff_j] with
    // tab the head's table (staged in shared memory when it fits, followed by zeros that
    // class-token rows and keys index into), koff_j kept as byte offsets.
    const float* brow = nullptr;
    const float* gtab = nullptr;
    int a_i = 0;
    if (BK == BA_BIAS_DENSE) brow = p.bias.data + b * p.bias.batch_stride + (h * N + ic) * N;
    if (is_relpos(BK)) {
      const int W2 = 2 * p.bias.table_w - 1;
      gtab = p.bias.data + h * static_cast<int64_t>(2 * p.bias.table_h - 1) * W2;
      if (ic >= p.bias.n_prefix) {
        const int ti = ic - p.bias.n_prefix;
        const int yi = ti / p.bias.grid_w;
        a_i = (yi + p.bias.table_h - 1) * W2 + (ti - yi * p.bias.grid_w) + p.bias.table_w - 1;
      } else {
        a_i = (tab_mode == 2) ? tsize + kmax : -1;  // class-token row: the zeros (or the general path)
      }
    }
    const uint32_t tb = smem_u32(stab) + 4u * static_cast<uint32_t>(a_i);  // this row's table base
    const float* grow = gtab + a_i;  // this row's base in a table left in global memory

    float m = -CUDART_INF_F, l = 0.0f;
    // Whether F holds anything yet, and how many blocks the current accumulator holds.
    int nblk = 1;
    bool f_valid = false;
    cur ^= 1;

    for (int t = 0; t < T && alive; ++t) {
      const int n = n0 + t;
      const int st = n % S;
      const int nk = min(BN, N - t * BN);
      // 32-key chunks that hold keys of this block. The P codes of the chunks past them are
      // left as they are: they multiply V rows past N, which the V copy fills with zeros.
      const int nch = (nk + 31) >> 5;
      if (is_relpos(BK) && !wait_warp(&bars[Bar::kvfull(st)], (n / S) & 1, abort_flag)) {
        alive = false;
        break;
      }
      if (!wait_warp(&bars[Bar::sfull(q)], n & 1, abort_flag)) {
        alive = false;
        break;
      }
      tc_fence_after();
      const uint32_t ko_s = smem_u32(koff + st * BN);

      // Pass 1: s = alpha * x + b written back over S in TMEM; block max. The next 32-column
      // block is loaded from TMEM while this one is computed.
      float mx[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
      // The fast path also takes a partial last block (keys past N are masked to -inf after
      // the fact; their rel-pos offsets point at valid entries), except for dense bias rows,
      // which end at N.
      const bool fast = fast_ok && (nk == BN || BK != BA_BIAS_DENSE);
      {
        // One copy of the block body (a small hot loop stays in the instruction cache; the
        // other softmax warps of the SM cover the TMEM load latency).
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          uint32_t x[32];
          tmem_ld32(aS + 32 * c, x);
          tmem_ld_wait();
          reg_fence32(x);
          if (fast) {
            if (nk == BN)
              fast_block<BK, false>(x, c, nk, alpha2, brow + t * BN, ko_s, tb, grow, tab_mode, mx);
            else
              fast_block<BK, true>(x, c, nk, alpha2, brow + t * BN, ko_s, tb, grow, tab_mode, mx);
          } else {
            // General path: a partial last block, class tokens without zero padding,
            // unaligned dense rows, a table in global memory, or the debug logits.
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int j = 32 * c + u;
              float sv = -CUDART_INF_F;
              if (j < nk) {
                const float xf = __uint_as_float(x[u]);
                float bias = 0.0f;
                if (BK == BA_BIAS_DENSE) bias = __ldg(brow + t * BN + j);
                if (is_relpos(BK)) {
                  const int kj = lds_s32(ko_s + 4u * j) >> 2;
                  if (a_i >= 0 && kj >= 0)
                    bias = (tab_mode != 0) ? lds_f32(smem_u32(stab) + 4u * static_cast<uint32_t>(a_i - kj))
                                           : __ldg(gtab + (a_i - kj));
                }
                sv = __fmaf_rn(alpha, xf, bias);
                if (p.dbg_logits != nullptr && row_ok)
                  p.dbg_logits[(bh * N + i) * N + t * BN + j] = __float2int_rn(xf);
              }
              mx[u & 3] = fmaxf(mx[u & 3], sv);
              x[u] = __float_as_uint(sv);
            }
          }
          tmem_st32(aS + 32 * c, x);
        }
      }
      const float m_new = fmaxf(m, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
      tmem_st_wait();

      // Pass 2: P~ = 2^((s - m) log2 e) (masked keys hold s = -inf: P~ = 0), row sum, u8 codes
      // -> TMEM columns 0..31 (their s values were read in the first step of this pass).
      const float2 negm2 = make_float2(-m_new, -m_new);
      const float2 log2e2 = make_float2(kLog2e, kLog2e);
      const float2 c255 = make_float2(255.0f, 255.0f);
      const float2 magic2 = make_float2(12582912.0f, 12582912.0f);
      float2 lt2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
      {
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          uint32_t x[32];
          tmem_ld32(aS + 32 * c, x);
          tmem_ld_wait();
          reg_fence32(x);
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
              const float2 p2 = ((kPolyPairs >> (2 * w + e2)) & 1u) ? exp2_poly2(t2)
                                                                    : make_float2(ex2_approx(t2.x), ex2_approx(t2.y));
              lt2[e2] = __fadd2_rn(lt2[e2], p2);
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
      }
      const float lt = (lt2[0].x + lt2[0].y) + (lt2[1].x + lt2[1].y);
      // Rescale factor of the row's earlier blocks: exactly 1 while its max is unchanged.
      const float ct = (m == -CUDART_INF_F) ? 0.0f : (m_new > m ? ex2_approx((m - m_new) * kLog2e) : 1.0f);
      l = l * ct + lt;
      // Vote (per warp) whether a row raised its max; the MMA thread reads the votes of the
      // tile's four warps after their p_full arrivals.
      const bool rose = __any_sync(0xffffffffu, t > 0 && m_new > m);
      if (lane == 0) votes[((n & 1) * NQ + q) * 4 + w4] = rose ? 1u : 0u;
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Bar::pfull(q)]);
      if (t == 0) continue;
      // While the MMAs of the next block run: if any row of the tile raised its max, P.V of
      // this block goes to the other accumulator, and the old one is folded into F with this
      // row's factor (1 for rows whose max did not rise).
      if (!wait_warp(&bars[Bar::pfull(q)], n & 1, abort_flag)) {
        alive = false;
        break;
      }
      const volatile uint32_t* vt = votes + ((n & 1) * NQ + q) * 4;
      if ((vt[0] | vt[1] | vt[2] | vt[3]) != 0u) {
        fold_rest<C, 0>(cur ? aO1 : aO0, aF, sF + q * BM + r, make_float2(ct, ct), !f_valid, nblk == 1);
        if (!C::kFSmem) tmem_st_wait();
        cur ^= 1;
        f_valid = true;
        nblk = 1;
      } else {
        ++nblk;
      }
    }

    // This item's V scales / 255 (lane l of every warp holds channels l, l + 32, ..., read by
    // shuffles in the epilogue) and the next item's mu, loaded while the last P.V runs.
    float scv[(DP + 31) / 32];
#pragma unroll
    for (int k = 0; k < (DP + 31) / 32; ++k)
      scv[k] = (32 * k + lane < d) ? p.v_scale[bh * d + 32 * k + lane] * (1.0f / 255.0f) : 0.0f;
    if (it + 1 < n_items) {
      int64_t nbh;
      int nq0;
      item_at(by_head, it + 1, p.H, nqb, BM * NQ, nbh, nq0);
      mu_q_next = p.mu_q[nbh];
      mu_k_next = p.mu_k[nbh];
    }
    if (alive && wait_warp(&bars[Bar::odone(q)], it & 1, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      // Rows whose byte length is a multiple of 16 are written with 16-byte stores (each
      // thread owns one row); other shapes fall back to element stores.
      const int esz = (p.o_dt == BA_F32) ? 4 : 2;
      const bool vec = ((d * esz) & 15) == 0;
      char* orow = reinterpret_cast<char*>(p.o) + ((bh * N + i) * d) * esz;
      const uint32_t aO = cur ? aO1 : aO0;
      const float4* fr = sF + q * BM + r;
#pragma unroll 1
      for (int cc = 0; cc < DP / 16; ++cc) {
        uint32_t a[16], fb[16];
        tmem_ld16(aO + 16 * cc, a);
        if constexpr (!C::kFSmem) tmem_ld16(aF + 16 * cc, fb);  // read even before the first fold
        tmem_ld_wait();
        reg_fence16(a);
        if constexpr (!C::kFSmem) reg_fence16(fb);
        float val[16];
        // Scales of channels 16 cc .. 16 cc + 15: held by lanes 16 (cc & 1) ... of register cc / 2.
        float sreg = scv[0];
#pragma unroll
        for (int k = 1; k < (DP + 31) / 32; ++k)
          if (cc >= 2 * k) sreg = scv[k];  // constant comparisons keep scv in registers
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float fv;
          if constexpr (C::kFSmem) {
            const float4 v4 = fr[(4 * cc + (e >> 2)) * (NQ * BM)];
            fv = (e & 3) == 0 ? v4.x : ((e & 3) == 1 ? v4.y : ((e & 3) == 2 ? v4.z : v4.w));
          } else {
            fv = __uint_as_float(fb[e]);
          }
          if (!f_valid) fv = 0.0f;
          const float sc = __shfl_sync(0xffffffffu, sreg, 16 * (cc & 1) + e);
          val[e] = (fv + __int2float_rn(static_cast<int>(a[e]))) * sc * inv_l;
        }
        if (!row_ok) continue;
        if (vec && 16 * cc + 16 <= d) {
          if (p.o_dt == BA_F32) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              reinterpret_cast<float4*>(orow + (16 * cc + 4 * k4) * 4)[0] =
                  make_float4(val[4 * k4], val[4 * k4 + 1], val[4 * k4 + 2], val[4 * k4 + 3]);
          } else {
            uint32_t h[8];
#pragma unroll
            for (int k2 = 0; k2 < 8; ++k2) {
              if (p.o_dt == BA_F16) {
                const __half2 v = __floats2half2_rn(val[2 * k2], val[2 * k2 + 1]);
                h[k2] = *reinterpret_cast<const uint32_t*>(&v);
              } else {
                const __nv_bfloat162 v = __floats2bfloat162_rn(val[2 * k2], val[2 * k2 + 1]);
                h[k2] = *reinterpret_cast<const uint32_t*>(&v);
              }
            }
            reinterpret_cast<uint4*>(orow + 16 * cc * 2)[0] = make_uint4(h[0], h[1], h[2], h[3]);
            reinterpret_cast<uint4*>(orow + 16 * cc * 2)[1] = make_uint4(h[4], h[5], h[6], h[7]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (16 * cc + e < d) store_out(p.o, (bh * N + i) * d + 16 * cc + e, val[e], p.o_dt);
        }
      }
    }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  named_barrier_sync(1, C::kThreads);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// The same forward with one work item per CTA (no persistent loop): used for heads wider than
// 80 channels (one 128-row tile per CTA, F in tensor memory), where it measured faster than the
// persistent kernel on B200.
template <int DP, int BK, int NQ_>
__global__ void __launch_bounds__(Cfg<DP, NQ_>::kThreads, Cfg<DP, NQ_>::kCtasPerSm)
    attn_tc_single_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmap_v, int tab_mode, int tsize,
                   int kmax) {
  using C = Cfg<DP, NQ_>;
  constexpr int NQ = C::NQ, DQ = C::DQ, S = C::kStages;
  using Bar = Bars<S, NQ>;
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
  // Per block parity, tile and softmax warp: whether a row of that warp raised its max.
  uint32_t* votes = reinterpret_cast<uint32_t*>(smem + C::offVotes);
  float4* sF = reinterpret_cast<float4*>(smem + C::offF);  // [DP/4][NQ*128]
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
    for (int st = 0; st < C::kStages; ++st) {
      // kv_full: the V copy's expect_tx arrival + warp 0 (key offsets) + the two expanding warps.
      mbar_init(&bars[Bar::kvfull(st)], 4);
      mbar_init(&bars[Bar::kvempty(st)], 1);
    }
    mbar_init(&bars[Bar::qfull()], 2);
    mbar_init(&bars[Bar::drain()], 1);
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&bars[Bar::sfull(q)], 1);
      mbar_init(&bars[Bar::pfull(q)], 4);
      mbar_init(&bars[Bar::odone(q)], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmap_v);
  }
  // Warps 2 and 3 load the sign rows of their Q rows and of key block 0 before the setup barrier,
  // so the loads overlap the setup.
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  uint4 pre_q[NQ][2], pre_k[2];
  if (warp == 2 || warp == 3) {
    const int half = warp - 2;
    const uint4* qrows = reinterpret_cast<const uint4*>(p.bits_q) + bh * N;
    const uint4* krows = reinterpret_cast<const uint4*>(p.bits_k) + bh * N;
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int row = q0 + q * BM + 64 * half + lane + 32 * u;
        pre_q[q][u] = row < N ? __ldg(qrows + row) : zero4;
      }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int row = 64 * half + lane + 32 * u;
      pre_k[u] = row < N ? __ldg(krows + row) : zero4;
    }
  }
  if (threadIdx.x < 128)
    sscale[threadIdx.x] = (threadIdx.x < d) ? p.v_scale[bh * d + threadIdx.x] * (1.0f / 255.0f) : 0.0f;
  if (is_relpos(BK) && tab_mode != 0) {
    const float* src = p.bias.data + h * static_cast<int64_t>(tsize);
    const int n = (tab_mode == 2) ? 3 * tsize : tsize;
    for (int e = threadIdx.x; e < n; e += C::kThreads) stab[e] = (e < tsize) ? __ldg(src + e) : 0.0f;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer: V blocks, key offsets
    const int W2 = 2 * p.bias.table_w - 1;
    int issued = 0;
    for (int t = 0; t < T; ++t) {
      const int st = t % S;
      if (t >= S && !wait_warp(&bars[Bar::kvempty(st)], ((t / S) - 1) & 1, abort_flag)) break;
      issued = t + 1;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars[Bar::kvfull(st)], C::kVBytes);
        tma_load_4d(sV + st * C::kVBytes, &tmap_v, &bars[Bar::kvfull(st)], 0, t * BN, 0, static_cast<int>(bh));
      }
      if (is_relpos(BK)) {
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
          koff[st * BN + j] = 4 * v;  // byte offset into the staged table
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Bar::kvfull(st)]);
    }
    // Leave no TMA copy in flight: wait (bounded, even after an abort) for the stages this
    // warp filled last.
    for (int t = (issued > S ? issued - S : 0); t < issued; ++t)
      wait_bounded(&bars[Bar::kvfull(t % S)], (t / S) & 1, abort_flag, false);
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ producer: sign expansion
    // Warp 2 expands rows 0..63 and warp 3 rows 64..127 of every Q tile and K block. The
    // sign rows of the next block are loaded into registers before this block is written.
    const int half = warp - 2;
    const uint4* krows = reinterpret_cast<const uint4*>(p.bits_k) + bh * N;
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int u = 0; u < 2; ++u)
        expand_row<DQ>(sQ + q * C::kQBytes, pre_q[q][u], q0 + q * BM + 64 * half + lane + 32 * u < N,
                       64 * half + lane + 32 * u, d);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[Bar::qfull()]);
    uint4 nb[2] = {pre_k[0], pre_k[1]};
    for (int t = 0; t < T; ++t) {
      const int st = t % S;
      const uint4 cb[2] = {nb[0], nb[1]};
      if (t + 1 < T) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int row = (t + 1) * BN + 64 * half + lane + 32 * u;
          nb[u] = row < N ? __ldg(krows + row) : zero4;
        }
      }
      if (t >= S && !wait_warp(&bars[Bar::kvempty(st)], ((t / S) - 1) & 1, abort_flag)) break;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int r = 64 * half + lane + 32 * u;
        expand_row<DQ>(sK + st * C::kKBytes, cb[u], t * BN + r < N, r, d);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Bar::kvfull(st)]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                (static_cast<uint32_t>(BM >> 4) << 24);
      const uint32_t idesc_pv = (2u << 4) | (0u << 7) | (1u << 10) | (1u << 16) |
                                (static_cast<uint32_t>(DP >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
      if (wait_bounded(&bars[Bar::qfull()], 0, abort_flag)) {
        tc_fence_after();
        bool ok = true;
        uint32_t cur_acc = 0;  // bit q: the accumulator P.V of tile q adds into
        for (int t = 0; t <= T && ok; ++t) {
          for (int q = 0; q < NQ && ok; ++q) {
            // P.V of the previous block first (it needs no new operands), then QK of this
            // block into the same S columns (issue order keeps P read before S is rewritten).
            if (t > 0) {
              if (!wait_bounded(&bars[Bar::pfull(q)], (t - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              // Block 0 starts accumulator 0. Later blocks switch to the other accumulator
              // (overwriting it) when a row of the tile raised its max: the softmax warps'
              // votes, written before their p_full arrivals.
              bool fresh = (t == 1);
              if (t > 1) {
                const volatile uint32_t* vt = votes + (((t - 1) & 1) * NQ + q) * 4;
                if ((vt[0] | vt[1] | vt[2] | vt[3]) != 0u) {
                  cur_acc ^= 1u << q;
                  fresh = true;
                }
              }
              const uint32_t acc = tmem + C::tO(q, (cur_acc >> q) & 1u);
              const uint32_t vbase = smem_u32(sV + ((t - 1) % S) * C::kVBytes);
#pragma unroll
              for (int kk = 0; kk < BN / 32; ++kk)
                mma_i8_ts(acc, tmem + C::tP(q) + 8 * kk, smem_desc(vbase + 512 * kk, 128, 2048), idesc_pv,
                          (fresh && kk == 0) ? 0u : 1u);
            }
            if (t < T) {
              if (q == 0) {
                if (!wait_bounded(&bars[Bar::kvfull(t % S)], (t / S) & 1, abort_flag)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
              }
              const uint32_t qb = smem_u32(sQ + q * C::kQBytes), kb = smem_u32(sK + (t % S) * C::kKBytes);
#pragma unroll
              for (int kk = 0; kk < DQ / 32; ++kk)
                mma_f8f6f4_ss(tmem + C::tS(q), smem_desc(qb + kk * 4096, 2048, 128),
                              smem_desc(kb + kk * 4096, 2048, 128), idesc_qk, kk > 0 ? 1u : 0u);
              tc_commit(&bars[Bar::sfull(q)]);
            } else {
              tc_commit(&bars[Bar::odone(q)]);
            }
          }
          if (ok && t > 0) tc_commit(&bars[Bar::kvempty((t - 1) % S)]);
        }
      }
      // Every MMA this thread issued has completed before tensor memory is released.
      tc_commit(&bars[Bar::drain()]);
      wait_bounded(&bars[Bar::drain()], 0, abort_flag, false);
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
    const uint32_t aO0 = tmem + lane_base + C::tO(q, 0);
    const uint32_t aO1 = tmem + lane_base + C::tO(q, 1);
    const uint32_t aF = tmem + lane_base + C::tF(q);  // unused when F is in shared memory
    const float alpha = __fmul_rn(__fmul_rn(p.softmax_scale, p.mu_q[bh]), p.mu_k[bh]);
    const float2 alpha2 = make_float2(alpha, alpha);

    // Bias addressing. Dense: this row of [H][N][N]. Rel-pos: b_ij = tab[a_i - koff_j] with
    // tab the head's table (staged in shared memory when it fits, followed by zeros that
    // class-token rows and keys index into), koff_j kept as byte offsets.
    const float* brow = nullptr;
    const float* gtab = nullptr;
    int a_i = 0;
    if (BK == BA_BIAS_DENSE) brow = p.bias.data + b * p.bias.batch_stride + (h * N + ic) * N;
    if (is_relpos(BK)) {
      const int W2 = 2 * p.bias.table_w - 1;
      gtab = p.bias.data + h * static_cast<int64_t>(2 * p.bias.table_h - 1) * W2;
      if (ic >= p.bias.n_prefix) {
        const int ti = ic - p.bias.n_prefix;
        const int yi = ti / p.bias.grid_w;
        a_i = (yi + p.bias.table_h - 1) * W2 + (ti - yi * p.bias.grid_w) + p.bias.table_w - 1;
      } else {
        a_i = (tab_mode == 2) ? tsize + kmax : -1;  // class-token row: the zeros (or the general path)
      }
    }
    const uint32_t tb = smem_u32(stab) + 4u * static_cast<uint32_t>(a_i);  // this row's table base
    // Fast path: full key blocks, no debug output, aligned dense rows, rel-pos table in shared
    // memory with the class tokens handled by the zero padding.
    const bool fast_ok = (p.dbg_logits == nullptr) &&
                         (BK != BA_BIAS_DENSE || ((N & 3) == 0 && (p.bias.batch_stride & 3) == 0)) &&
                         (!is_relpos(BK) || p.bias.n_prefix == 0 || tab_mode == 2);
    const float* grow = gtab + a_i;  // this row's base in a table left in global memory

    float m = -CUDART_INF_F, l = 0.0f;
    bool alive = true;
    // Accumulator that P.V of the current block adds into (tile-uniform), whether F holds
    // anything yet, and how many blocks that accumulator holds.
    int cur = 0, nblk = 1;
    bool f_valid = false;

    for (int t = 0; t < T && alive; ++t) {
      const int st = t % S;
      const int nk = min(BN, N - t * BN);
      // 32-key chunks that hold keys of this block. The P codes of the chunks past them are
      // left as they are: they multiply V rows past N, which the V copy fills with zeros.
      const int nch = (nk + 31) >> 5;
      if (is_relpos(BK) && !wait_warp(&bars[Bar::kvfull(st)], (t / S) & 1, abort_flag)) {
        alive = false;
        break;
      }
      if (!wait_warp(&bars[Bar::sfull(q)], t & 1, abort_flag)) {
        alive = false;
        break;
      }
      tc_fence_after();
      const uint32_t ko_s = smem_u32(koff + st * BN);

      // Pass 1: s = alpha * x + b written back over S in TMEM; block max. The next 32-column
      // block is loaded from TMEM while this one is computed.
      float mx[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
      // The fast path also takes a partial last block (keys past N are masked to -inf after
      // the fact; their rel-pos offsets point at valid entries), except for dense bias rows,
      // which end at N.
      const bool fast = fast_ok && (nk == BN || BK != BA_BIAS_DENSE);
      {
        // One copy of the block body (a small hot loop stays in the instruction cache; the
        // other softmax warps of the SM cover the TMEM load latency).
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          uint32_t x[32];
          tmem_ld32(aS + 32 * c, x);
          tmem_ld_wait();
          reg_fence32(x);
          if (fast) {
            if (nk == BN)
              fast_block<BK, false>(x, c, nk, alpha2, brow + t * BN, ko_s, tb, grow, tab_mode, mx);
            else
              fast_block<BK, true>(x, c, nk, alpha2, brow + t * BN, ko_s, tb, grow, tab_mode, mx);
          } else {
            // General path: a partial last block, class tokens without zero padding,
            // unaligned dense rows, a table in global memory, or the debug logits.
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int j = 32 * c + u;
              float sv = -CUDART_INF_F;
              if (j < nk) {
                const float xf = __uint_as_float(x[u]);
                float bias = 0.0f;
                if (BK == BA_BIAS_DENSE) bias = __ldg(brow + t * BN + j);
                if (is_relpos(BK)) {
                  const int kj = lds_s32(ko_s + 4u * j) >> 2;
                  if (a_i >= 0 && kj >= 0)
                    bias = (tab_mode != 0) ? lds_f32(smem_u32(stab) + 4u * static_cast<uint32_t>(a_i - kj))
                                           : __ldg(gtab + (a_i - kj));
                }
                sv = __fmaf_rn(alpha, xf, bias);
                if (p.dbg_logits != nullptr && row_ok)
                  p.dbg_logits[(bh * N + i) * N + t * BN + j] = __float2int_rn(xf);
              }
              mx[u & 3] = fmaxf(mx[u & 3], sv);
              x[u] = __float_as_uint(sv);
            }
          }
          tmem_st32(aS + 32 * c, x);
        }
      }
      const float m_new = fmaxf(m, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
      tmem_st_wait();

      // Pass 2: P~ = 2^((s - m) log2 e) (masked keys hold s = -inf: P~ = 0), row sum, u8 codes
      // -> TMEM columns 0..31 (their s values were read in the first step of this pass).
      const float2 negm2 = make_float2(-m_new, -m_new);
      const float2 log2e2 = make_float2(kLog2e, kLog2e);
      const float2 c255 = make_float2(255.0f, 255.0f);
      const float2 magic2 = make_float2(12582912.0f, 12582912.0f);
      float2 lt2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
      {
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          uint32_t x[32];
          tmem_ld32(aS + 32 * c, x);
          tmem_ld_wait();
          reg_fence32(x);
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
              const float2 p2 = ((kPolyPairs >> (2 * w + e2)) & 1u) ? exp2_poly2(t2)
                                                                    : make_float2(ex2_approx(t2.x), ex2_approx(t2.y));
              lt2[e2] = __fadd2_rn(lt2[e2], p2);
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
      }
      const float lt = (lt2[0].x + lt2[0].y) + (lt2[1].x + lt2[1].y);
      // Rescale factor of the row's earlier blocks: exactly 1 while its max is unchanged.
      const float ct = (m == -CUDART_INF_F) ? 0.0f : (m_new > m ? ex2_approx((m - m_new) * kLog2e) : 1.0f);
      l = l * ct + lt;
      // Vote (per warp) whether a row raised its max; the MMA thread reads the votes of the
      // tile's four warps after their p_full arrivals.
      const bool rose = __any_sync(0xffffffffu, t > 0 && m_new > m);
      if (lane == 0) votes[((t & 1) * NQ + q) * 4 + w4] = rose ? 1u : 0u;
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Bar::pfull(q)]);
      if (t == 0) continue;
      // While the MMAs of the next block run: if any row of the tile raised its max, P.V of
      // this block goes to the other accumulator, and the old one is folded into F with this
      // row's factor (1 for rows whose max did not rise).
      if (!wait_warp(&bars[Bar::pfull(q)], t & 1, abort_flag)) {
        alive = false;
        break;
      }
      const volatile uint32_t* vt = votes + ((t & 1) * NQ + q) * 4;
      if ((vt[0] | vt[1] | vt[2] | vt[3]) != 0u) {
        fold_rest<C, 0>(cur ? aO1 : aO0, aF, sF + q * BM + r, make_float2(ct, ct), !f_valid, nblk == 1);
        if (!C::kFSmem) tmem_st_wait();
        cur ^= 1;
        f_valid = true;
        nblk = 1;
      } else {
        ++nblk;
      }
    }

    if (alive && wait_warp(&bars[Bar::odone(q)], 0, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      // Rows whose byte length is a multiple of 16 are written with 16-byte stores (each
      // thread owns one row); other shapes fall back to element stores.
      const int esz = (p.o_dt == BA_F32) ? 4 : 2;
      const bool vec = ((d * esz) & 15) == 0;
      char* orow = reinterpret_cast<char*>(p.o) + ((bh * N + i) * d) * esz;
      const uint32_t aO = cur ? aO1 : aO0;
      const float4* fr = sF + q * BM + r;
#pragma unroll 1
      for (int cc = 0; cc < DP / 16; ++cc) {
        uint32_t a[16];
        float f[16];
        tmem_ld16(aO + 16 * cc, a);
        if constexpr (C::kFSmem) {
          tmem_ld_wait();
          reg_fence16(a);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const float4 v = f_valid ? fr[(4 * cc + k4) * (NQ * BM)] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            f[4 * k4] = v.x; f[4 * k4 + 1] = v.y; f[4 * k4 + 2] = v.z; f[4 * k4 + 3] = v.w;
          }
        } else {
          uint32_t fb[16];
          if (f_valid) tmem_ld16(aF + 16 * cc, fb);
          tmem_ld_wait();
          reg_fence16(a);
          if (f_valid) reg_fence16(fb);
#pragma unroll
          for (int e = 0; e < 16; ++e) f[e] = f_valid ? __uint_as_float(fb[e]) : 0.0f;
        }
        float val[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          val[e] = (f[e] + __int2float_rn(static_cast<int>(a[e]))) * sscale[16 * cc + e] * inv_l;
        if (!row_ok) continue;
        if (vec && 16 * cc + 16 <= d) {
          if (p.o_dt == BA_F32) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              reinterpret_cast<float4*>(orow + (16 * cc + 4 * k4) * 4)[0] =
                  make_float4(val[4 * k4], val[4 * k4 + 1], val[4 * k4 + 2], val[4 * k4 + 3]);
          } else {
            uint32_t h[8];
#pragma unroll
            for (int k2 = 0; k2 < 8; ++k2) {
              if (p.o_dt == BA_F16) {
                const __half2 v = __floats2half2_rn(val[2 * k2], val[2 * k2 + 1]);
                h[k2] = *reinterpret_cast<const uint32_t*>(&v);
              } else {
                const __nv_bfloat162 v = __floats2bfloat162_rn(val[2 * k2], val[2 * k2 + 1]);
                h[k2] = *reinterpret_cast<const uint32_t*>(&v);
              }
            }
            reinterpret_cast<uint4*>(orow + 16 * cc * 2)[0] = make_uint4(h[0], h[1], h[2], h[3]);
            reinterpret_cast<uint4*>(orow + 16 * cc * 2)[1] = make_uint4(h[4], h[5], h[6], h[7]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (16 * cc + e < d) store_out(p.o, (bh * N + i) * d + 16 * cc + e, val[e], p.o_dt);
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  named_barrier_sync(1, C::kThreads);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
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

constexpr int kMaxSmem = 227 * 1024;      // per CTA
constexpr int kSmPerSmem = 228 * 1024;    // per SM
constexpr int kSmemReserved = 1024;       // per CTA, taken by the runtime

// Dynamic shared memory a CTA of configuration C may use.
template <class C>
constexpr int smem_room() {
  return C::kCtasPerSm == 1 ? kMaxSmem : kSmPerSmem / C::kCtasPerSm - kSmemReserved;
}

// 0: rel-pos table read from global memory; 1: staged in shared memory; 2: staged and followed
// by 2 * tsize zeros that class-token rows and keys index into.
template <class C>
int relpos_table_mode(const AttnParams& p) {
  const int64_t tsize = static_cast<int64_t>(2 * p.bias.table_h - 1) * (2 * p.bias.table_w - 1);
  const int64_t room = smem_room<C>() - 1024 - C::kTabOff;
  if (p.bias.n_prefix > 0 && 3 * tsize * 4 <= room) return 2;
  if (tsize * 4 <= room) return 1;
  return 0;
}

template <int DP, int BK, int NQ>
constexpr auto pick_kernel() {
  if constexpr (DP > 80)
    return attn_tc_single_kernel<DP, BK, NQ>;
  else
    return attn_tc_kernel<DP, BK, NQ>;
}

template <int DP, int BK, int NQ>
cudaError_t launch_cfg(const AttnParams& p, const CUtensorMap& tm, cudaStream_t s) {
  using C = Cfg<DP, NQ>;
  int tab_mode = 0, tsize = 0, kmax = 0;
  if (is_relpos(BK)) {
    tsize = (2 * p.bias.table_h - 1) * (2 * p.bias.table_w - 1);
    kmax = (p.bias.grid_h - 1) * (2 * p.bias.table_w - 1) + p.bias.grid_w - 1;
    tab_mode = relpos_table_mode<C>(p);
  }
  const int tab_bytes = tab_mode == 0 ? 0 : (tab_mode == 2 ? 3 : 1) * tsize * 4;
  // A CTA that owns all 512 tensor-memory columns takes enough shared memory to be alone on its
  // SM; one that owns 256 takes enough that no third CTA fits.
  int smem = C::kTabOff + tab_bytes + 1024;
  const int floor_bytes = C::kCtasPerSm == 1 ? 116 * 1024 : 80 * 1024;
  if (smem < floor_bytes) smem = floor_bytes;
  // Heads wider than 80 channels: one work item per CTA; otherwise the persistent kernel.
  constexpr bool kSingle = DP > 80;
  auto kernel = pick_kernel<DP, BK, NQ>();
  static int configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  // Persistent CTAs: as many as fit at once (CTAs per SM x SMs), H per group, each walking the
  // items of its head; at least one CTA per head.
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t per_head = static_cast<int64_t>(p.B) * ceil_div(p.N, BM * C::NQ);
  const int64_t slots = static_cast<int64_t>(C::kCtasPerSm) * sms;
  int64_t grid;
  if (kSingle) {
    grid = per_head * p.H;
  } else if (is_relpos(BK) && tab_mode != 0) {  // items grouped by head (the kernel's by_head)
    const int64_t k = std::max<int64_t>(1, std::min<int64_t>(per_head, slots / p.H));
    grid = k * p.H;
  } else {
    grid = std::min<int64_t>(per_head * p.H, slots);
  }
  if constexpr (kSingle) {
    kernel<<<static_cast<unsigned>(grid), C::kThreads, smem, s>>>(p, tm, tab_mode, tsize, kmax);
    return cudaGetLastError();
  } else {
    // Programmatic dependent of the preparation kernel: the launch, and the barrier set-up of
    // the CTAs that find an SM free, overlap the last preparation CTAs; each CTA waits for the
    // preparation grid (grid_dependency_wait) before it reads anything that grid writes.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p, tm, tab_mode, tsize, kmax);
  }
}

template <int DP, int NQ>
cudaError_t launch_nq(const AttnParams& p, const CUtensorMap& tm, cudaStream_t s) {
  switch (p.bias.kind) {
    case BA_BIAS_DENSE: return launch_cfg<DP, BA_BIAS_DENSE, NQ>(p, tm, s);
    case BA_BIAS_RELPOS2D:
      return relpos_table_mode<Cfg<DP, NQ>>(p) != 0 ? launch_cfg<DP, BA_BIAS_RELPOS2D, NQ>(p, tm, s)
                                                     : launch_cfg<DP, kRelposGlobal, NQ>(p, tm, s);
    default: return launch_cfg<DP, BA_BIAS_NONE, NQ>(p, tm, s);
  }
}

// Head dimensions up to 64 run one query tile per CTA in half of tensor memory, two CTAs per
// SM (the CTAs' prologues, pipeline fills and epilogues overlap each other's work), unless the
// rel-pos table only fits in the shared memory of a CTA that has the SM to itself; then one CTA
// runs two tiles.
template <int DP>
cudaError_t launch_dp(const AttnParams& p, const CUtensorMap& tm, cudaStream_t s) {
  if constexpr (DP <= 64) {
    const bool table_fits = p.bias.kind != BA_BIAS_RELPOS2D || relpos_table_mode<Cfg<DP, 1>>(p) != 0;
    return table_fits ? launch_nq<DP, 1>(p, tm, s) : launch_nq<DP, 2>(p, tm, s);
  } else {
    return launch_nq<DP, 1>(p, tm, s);
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
