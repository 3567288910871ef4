// Fused BinaryAttention forward on 5th-generation tensor cores (sm_100a: tcgen05 + TMEM + TMA).
//
// What it computes is the blockwise forward of the CUDA-core kernel (attn_simt.cu) and of the
// CPU reference: binary QK (gist.science/zh technical summary 2.1-2.2(1)), bias b_ij (2.2(2)),
// FlashAttention-2-style online softmax over ascending 128-key blocks (2.3), 8-bit P on [0,1]
// (2.2(3)), per-channel int8 V and an integer P.V (the u8 x s8 -> s32 instruction class named
// on every page).
//
// How, on B200:
//   * One CTA per SM (all 512 tensor-memory columns), persistent: each walks a list of work
//     items, grouped by head when the head's rel-pos table is staged in shared memory; its
//     producers and MMA thread run ahead into the next item. A work item is NQ query tiles of
//     128 rows of one (b, h).
//   * Warps 2 and 3 expand the 1-bit sign rows of Q (once per item) and of each K block into
//     fp8 +-1 operands in shared memory (channels >= d become 0); warp 0 TMA-loads the int8 V
//     block (a 4-D tensor map that lands it in the MN-major core-matrix layout the MMA reads)
//     and stages the block's bias data. A 4-stage ring of K/V blocks decouples them from the
//     MMAs.
//   * Warp 1 issues the MMAs from one thread:
//       S    = Q . K^T   tcgen05.mma kind::f8f6f4 (e4m3 +-1, fp32 accumulate: exact integers)
//       acc  = P . V     tcgen05.mma kind::i8, A = the uint8 codes read from TMEM, B = int8 V
//     acc holds one block's product.
//   * Two softmax warpgroups, one thread per query row each. Heads up to 64 channels: two
//     tiles per item, one per group (tile ping-pong: one tile's MMAs run while the other's
//     softmax works). Wider heads: one tile, S double-buffered, the groups taking alternate key
//     blocks (block ping-pong), the running maximum passed from group to group. Per block a
//     thread reads its row of S from TMEM, forms s = fmaf(alpha, x, b) and the block maximum,
//     then P~ = 2^((s - m) log2 e), its row sum and the 8-bit codes rne(255 P~), which it writes
//     back over S as the A operand of P.V.
//   * Each block's product is weighted by e_j = exp(m_j - m_ref) against a per-row reference
//     maximum: the output sum F' = sum_j acc_j e_j (tensor memory, fp32) and the softmax sum
//     L' = sum_j l_j e_j give O = F' v_scale / (255 L'), the blockwise online softmax's result.
//     Each P.V accumulates onto the bit pattern of 1.5 * 2^23, so a block's product
//     (|acc| <= 255 * 127 * 128 < 2^22) reads directly as the float 1.5 * 2^23 + acc.
//   * Near-tie codes are made exact: where a code of the fast exponential could differ from the
//     definition's (two roundings of 255 P~, scaled by 1 -+ eps, disagree), the key's
//     double-precision d = s - m is compared with a host-computed threshold table. This check
//     runs in every block of rows whose running softmax sum is still small against the head's
//     largest |V| (where one changed code could move an output by a set share of the error
//     bar), or everywhere on request.
//   * Every wait is bounded (1 s): on expiry the kernel records BA_ERR_TIMEOUT in a device
//     status word, every role leaves its loop, and the CTA frees its tensor memory.
#include <cuda.h>
#include <math_constants.h>

#include <algorithm>
#include <cmath>
#include <type_traits>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace binattn {

__device__ int g_device_status = 0;

namespace {

using namespace ptx;

constexpr int BM = 128;       // query rows per tile = MMA M
constexpr int BN = kKvBlock;  // keys per block = MMA N of QK, K of P.V
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kMagicBits = 0x4B400000u;  // bit pattern of 1.5 * 2^23
constexpr float kMagic = 12582912.0f;         // 1.5 * 2^23
constexpr int kWinFloats = 1024;              // rel-pos window per (tile, stage)

// Bias variants of the kernel.
constexpr int kBiasNone = 0;
constexpr int kBiasDense = 1;
constexpr int kRelSmem = 2;    // rel-pos, the head's whole table staged in shared memory
constexpr int kRelGlobal = 3;  // rel-pos, table read from global memory
constexpr int kRelWindow = 4;  // rel-pos on a grid of width 32k without class tokens: per (tile,
                               // block) window of the table staged by the producer
__host__ __device__ constexpr bool is_relpos_general(int bk) { return bk == kRelSmem || bk == kRelGlobal; }

template <int DP, int BK>
struct Cfg {
  // Heads up to 64 channels: two 128-row query tiles per item, one S buffer each; softmax
  // warpgroup q owns tile q (the tiles ping-pong: one's MMAs run while the other's softmax
  // works). Wider heads: one tile, S double-buffered, the two softmax warpgroups taking
  // alternate key blocks (the blocks ping-pong).
  static constexpr bool kTilePP = DP <= 64;
  static constexpr int NQ = kTilePP ? 2 : 1;   // query tiles per item
  static constexpr int SB = kTilePP ? 1 : 2;   // S buffers per tile
  static constexpr int DQ = (DP + 31) / 32 * 32;  // QK contraction width: fp8 K-steps of 32
  static constexpr int DH = DP / 2;            // accumulator / output columns per softmax half
  static constexpr int kThreads = 384;  // 4 service warps, 2 softmax warpgroups
  // Service warps: warp 0 V copies and bias data, warp 1 issues the MMAs (of both tiles, when
  // there are two), warps 2 and 3 expand the sign rows. (One MMA warp per tile, with one
  // expanding warp, measured 5-20 % slower on d = 64 heads.)
  static constexpr int kExpWarps = 2;
  static constexpr int kMmaWarps = 1;
  static constexpr int kRowsPerLane = BM / (32 * kExpWarps);  // sign rows a lane expands per tile
  static constexpr int kStages = 4;
  static constexpr int kQBytes = BM * DQ;
  static constexpr int kKBytes = BN * DQ;
  static constexpr int kVBytes = BN * DP;
  static constexpr int kWinBytes = BK == kRelWindow ? kStages * NQ * kWinFloats * 4 : 0;
  static constexpr int kWinKBytes = BK == kRelWindow ? kStages * NQ * 4 * 4 : 0;
  static constexpr int kKoffBytes = is_relpos_general(BK) ? kStages * BN * 4 : 0;
  static constexpr int offQ = 0;
  static constexpr int offK = offQ + NQ * kQBytes;
  static constexpr int offV = offK + kStages * kKBytes;
  static constexpr int offWin = offV + kStages * kVBytes;  // [S][NQ][kWinFloats] f32
  static constexpr int offWinK = offWin + kWinBytes;       // [S][NQ][4] s32 chunk offsets
  static constexpr int offKoff = offWinK + kWinKBytes;     // [S][BN] s32 key offsets
  static constexpr int offX = offKoff + kKoffBytes;  // per row: m_j [2][BM]; (L', m_ref) [2][BM]
  static constexpr int offBar = offX + 2 * BM * 4 + 2 * BM * 8;
  static constexpr int kNumBars = 2 * kStages + 3 + 2 + 2 + 2 + 2 + 1 + 4;
  static constexpr int offMisc = offBar + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kBytes = offMisc + 16;
  static constexpr int kTabOff = (kBytes + 127) / 128 * 128;  // staged rel-pos table (kRelSmem)
  // Tensor-memory columns of tile q: S buffer b (fp32, 128 columns; the softmax overwrites its
  // first 32 columns with the uint8 codes P — the MMAs of one CTA run in issue order, so P.V
  // reads P before the next QK into that buffer rewrites it), the s32 P.V accumulator of one
  // block (DP) and the fp32 running output F' (DP): 256 columns per tile for two tiles, or
  // 2 x 128 + 2 DP for one.
  __host__ __device__ static constexpr uint32_t tS(int q, int b) { return q * 256 + b * 128; }
  __host__ __device__ static constexpr uint32_t tAcc(int q) { return q * 256 + SB * 128; }
  __host__ __device__ static constexpr uint32_t tF(int q) { return tAcc(q) + DP; }
  static_assert(tF(NQ - 1) + DP <= 512, "tensor memory budget");
  static_assert(DP % 16 == 0 && DP >= 16 && DP <= 128, "head width");
};

// Barrier slots. Phases count K/V blocks (kv_*: per stage; s_full: per use of the S buffer;
// p_full, pv_done: per block), work items (q_*) or pair exchanges, across all the items a CTA
// processes.
template <class C>
struct Bars {
  static constexpr int S = C::kStages, NQ = C::NQ, SB = C::SB;
  __host__ __device__ static constexpr int kvfull(int s) { return s; }
  __host__ __device__ static constexpr int kvempty(int s) { return S + s; }
  __host__ __device__ static constexpr int qfull() { return 2 * S; }
  __host__ __device__ static constexpr int qempty() { return 2 * S + 1; }
  __host__ __device__ static constexpr int drain() { return 2 * S + 2; }
  // s_full per S buffer; p_full, pv_done, fold_done per softmax group g (the blocks j with
  // j % 2 == g, phase j / 2): a parity wait is exact only while the phase before it has
  // completed, so every waiter walks the phases of a barrier in order; epi_done per item;
  // mchain per row quarter (the running maximum passed between the groups, one phase per block).
  __host__ __device__ static constexpr int sfull(int q, int b) { return 2 * S + 3 + q * SB + b; }
  __host__ __device__ static constexpr int pfull(int g) { return 2 * S + 5 + g; }
  __host__ __device__ static constexpr int pvdone(int g) { return 2 * S + 7 + g; }
  __host__ __device__ static constexpr int folddone(int g) { return 2 * S + 9 + g; }
  __host__ __device__ static constexpr int epidone() { return 2 * S + 11; }
  __host__ __device__ static constexpr int mchain(int w4) { return 2 * S + 12 + w4; }
  static_assert(NQ * SB == 2, "two S buffers: one per tile, or two for one tile");
  static_assert(mchain(3) + 1 == C::kNumBars, "barrier count");
};

// Work items: NQ query tiles of one (b, h). With the head's rel-pos table staged in shared
// memory (by_head), the CTAs of head h are h, h + H, h + 2H, ... (gridDim.x = H * k) and CTA j
// of head h takes items j, j + k, j + 2k, ... of the B * nqb items of that head (nqb = query
// blocks per (b, h)), so the table is staged once. Otherwise CTA c takes items c, c + G,
// c + 2G, ... of all B * H * nqb items (G = gridDim.x), item m covering query block m % nqb of
// slice m / nqb.
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
// Between checks the thread sleeps in the barrier wait (up to 20 us, woken when the phase
// completes), so waiting warps take no issue slots from the working ones.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             bool yield = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (yield && *abort_flag) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      *abort_flag = 1;
      atomicExch(&g_device_status, 1);
      return false;
    }
  }
}

// As wait_bounded, polling without a suspend hint: for the warps whose waits sit on the
// softmax's critical path, where waking from a suspension costs more than the polls (measured
// 2-4 % faster on 128-channel heads).
__device__ __forceinline__ bool wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      *abort_flag = 1;
      atomicExch(&g_device_status, 1);
      return false;
    }
  }
}

// Warp-uniform variant: every lane waits, and the warp proceeds only if all lanes succeeded.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = wait_spin(bar, parity, abort_flag);
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

// Tensor-memory loads and stores of N consecutive columns (N a multiple of 8) of this warp's
// 32 lanes, split into x32 / x16 / x8 pieces; r points at a register array indexed by
// constants only.
template <int N, int O = 0>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* r) {
  if constexpr (N - O >= 32) {
    tmem_ld32p(taddr + O, r + O);
    tmem_ld_cols<N, O + 32>(taddr, r);
  } else if constexpr (N - O >= 16) {
    tmem_ld16p(taddr + O, r + O);
    tmem_ld_cols<N, O + 16>(taddr, r);
  } else if constexpr (N - O >= 8) {
    tmem_ld8p(taddr + O, r + O);
    tmem_ld_cols<N, O + 8>(taddr, r);
  }
}

template <int N, int O = 0>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t* r) {
  if constexpr (N - O >= 32) {
    tmem_st32p(taddr + O, r + O);
    tmem_st_cols<N, O + 32>(taddr, r);
  } else if constexpr (N - O >= 16) {
    tmem_st16p(taddr + O, r + O);
    tmem_st_cols<N, O + 16>(taddr, r);
  } else if constexpr (N - O >= 8) {
    tmem_st8p(taddr + O, r + O);
    tmem_st_cols<N, O + 8>(taddr, r);
  }
}

// Re-defines registers after tmem_ld_wait() so that no use of a loaded value is scheduled
// before the wait.
template <int N, int O = 0>
__device__ __forceinline__ void reg_fence_cols(uint32_t* r) {
  if constexpr (O < N) {
    reg_fence8(r + O);
    reg_fence_cols<N, O + 8>(r);
  }
}

// Exact 8-bit codes at a rounding tie. The definition's code of a logit s against the running
// max m is rne(fl32(255 fl32(exp(d)))), capped at 255, with d = (double)s - (double)m. It is a
// non-decreasing function of d, so code(d) >= k + 1 exactly when d >= thr[k], the least double
// whose code exceeds k. The host computes the 255 thresholds once, by bisection over doubles.
struct TieTable {
  double thr[256];
};

// Check mode rounds each 255 P~ twice, scaled by (1 - eps) and by (1 + eps). The two codes
// differ only where 255 P~ lies within a relative eps of a rounding tie. eps bounds the
// relative error of the fast path's P~ against fl32(exp(d)): the rounding of s - m and of its
// product with log2 e (|t| <= 9 for a nonzero code), the hardware 2^t and the definition's two
// fp32 roundings add up to about 1.2e-6.
constexpr float kTieEps = 4.0e-6f;
constexpr float kC255Lo = 255.0f * (1.0f - kTieEps);
constexpr float kC255Hi = 255.0f * (1.0f + kTieEps);

// One packed word of four codes: `hi` from the (1 + eps) rounding (the code wherever the two
// agree), `lo` from the (1 - eps) one. Where they differ the exact code is lo or lo + 1, and
// the key's d against thr[lo] decides.
__device__ __forceinline__ uint32_t settle_ties(uint32_t hi, uint32_t lo, const uint32_t* xs, float m,
                                                const TieTable& tt) {
  uint32_t out = hi;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t cl = (lo >> (8 * b)) & 0xFFu;
    if (cl != ((hi >> (8 * b)) & 0xFFu)) {
      const double dd = static_cast<double>(__uint_as_float(xs[b])) - static_cast<double>(m);
      const uint32_t code = cl + (dd >= tt.thr[cl] ? 1u : 0u);
      out = (out & ~(0xFFu << (8 * b))) | (code << (8 * b));
    }
  }
  return out;
}

// DBG: the instantiation that writes the debug logits and P codes; the product launches use the
// one without, whose hot loops carry no debug stores.
template <int DP, int BK, bool DBG>
__global__ void __launch_bounds__(Cfg<DP, BK>::kThreads, 1)
    attn_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmap_v, int tab_mode, int tsize,
                   int kmax, int win_stride, const __grid_constant__ TieTable tie) {
  using C = Cfg<DP, BK>;
  constexpr int NQ = C::NQ, SB = C::SB, DQ = C::DQ, DH = C::DH, S = C::kStages;
  using Bar = Bars<C>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the __shared__ array by an offset (not through an integer
  // cast), so that the compiler keeps every access through it a shared-memory access.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + C::offQ;
  uint8_t* sK = smem + C::offK;
  uint8_t* sV = smem + C::offV;
  float* swin = reinterpret_cast<float*>(smem + C::offWin);
  int* swink = reinterpret_cast<int*>(smem + C::offWinK);
  int* koff = reinterpret_cast<int*>(smem + C::offKoff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::offBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::offMisc + 4);
  // Rel-pos table of this CTA's head (kRelSmem): tab_mode 1 = table only, 2 = table followed by
  // 2*tsize zeros (targets of class-token rows and keys).
  float* stab = reinterpret_cast<float*>(smem + C::kTabOff);

  const int N = p.N, d = p.d;
  const int nqb = static_cast<int>(ceil_div(N, BM * NQ));
  const bool by_head = BK == kRelSmem;
  const int n_items = item_count(by_head, p.B, p.H, nqb);
  const int T = static_cast<int>(ceil_div(N, BN));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) {
      // kv_full: the V copy's expect_tx arrival + warp 0 (bias data) + the expanding warps;
      // kv_empty: one commit per MMA-issuing warp.
      mbar_init(&bars[Bar::kvfull(st)], 2 + C::kExpWarps);
      mbar_init(&bars[Bar::kvempty(st)], C::kMmaWarps);
    }
    mbar_init(&bars[Bar::qfull()], C::kExpWarps);
    mbar_init(&bars[Bar::qempty()], C::kMmaWarps);
    mbar_init(&bars[Bar::drain()], C::kMmaWarps);
    for (int q = 0; q < NQ; ++q)
      for (int b = 0; b < SB; ++b) mbar_init(&bars[Bar::sfull(q, b)], 1);
    for (int g = 0; g < 2; ++g) mbar_init(&bars[Bar::pfull(g)], 4);  // the group's four warps
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bars[Bar::pvdone(g)], 1);
      mbar_init(&bars[Bar::folddone(g)], 4);  // the folding group's four warps
    }
    mbar_init(&bars[Bar::epidone()], 8);   // both groups
    for (int w4 = 0; w4 < 4; ++w4) mbar_init(&bars[Bar::mchain(w4)], 1);
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmap_v);
  }
  // Everything above reads only the caller's inputs; from here on the kernel reads the sign
  // rows, mu and int8 V, which the preparation kernel before it in the stream may still be
  // writing when this kernel was launched as its programmatic dependent.
  grid_dependency_wait();
  if (by_head) {
    const float* src = p.bias.data + static_cast<int64_t>(blockIdx.x % p.H) * tsize;
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
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);

  if (warp == 0) {
    // ------------------------------------------------------------ producer: V blocks, bias data
    // Blocks are counted across the items (g): stage g % S, phase g / S.
    const int W2 = 2 * p.bias.table_w - 1;
    const int gw = p.bias.grid_w;
    int g = 0;
    bool ok = true;
    for (int it = 0; it < n_items && ok; ++it) {
      int64_t bh;
      int q0;
      item_at(by_head, it, p.H, nqb, BM * NQ, bh, q0);
      const int h = static_cast<int>(bh % p.H);
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
        if constexpr (is_relpos_general(BK)) {
#pragma unroll
          for (int u = 0; u < BN / 32; ++u) {
            const int j = lane + 32 * u, tok = t * BN + j;
            // Keys past N read a valid entry (their P is masked); prefix keys read the zeros
            // after the staged table (or are marked -1 for the per-key test).
            int v = (tab_mode == 2) ? -tsize : -1;
            if (tok >= N) {
              v = 0;
            } else if (tok >= p.bias.n_prefix) {
              const int tj = tok - p.bias.n_prefix;
              const int yj = tj / gw;
              v = yj * W2 + (tj - yj * gw);
            }
            koff[st * BN + j] = v;
          }
        } else if constexpr (BK == kRelWindow) {
          // For each tile: the rectangle of (dy, dx) offsets that its rows and this block's keys
          // form, copied from the head's table with row stride win_stride, and for each 32-key
          // chunk (one grid row) the offset K_c with which a query row reads its bias as
          // window[A_i - K_c - u], A_i = y_i * win_stride + x_i.
          const float* tab = p.bias.data + static_cast<int64_t>(h) * tsize;
          const int j0 = t * BN, j1 = min(j0 + BN, N) - 1;
          const int yk_lo = j0 / gw, yk_hi = j1 / gw;
          const int xk_min = yk_hi > yk_lo ? 0 : j0 - yk_lo * gw;
          const int xk_max = yk_hi > yk_lo ? gw - 1 : j1 - yk_lo * gw;
#pragma unroll 1
          for (int qq = 0; qq < NQ; ++qq) {
            const int i0 = min(q0 + qq * BM, N - 1), i1 = min(q0 + qq * BM + BM - 1, N - 1);
            const int yq_lo = i0 / gw, yq_hi = i1 / gw;
            const int xq_min = yq_hi > yq_lo ? 0 : i0 - yq_lo * gw;
            const int xq_max = yq_hi > yq_lo ? gw - 1 : i1 - yq_lo * gw;
            const int dy_lo = yq_lo - yk_hi, ndy = (yq_hi - yq_lo) + (yk_hi - yk_lo) + 1;
            const int dx_lo = xq_min - xk_max, width = (xq_max - xq_min) + (xk_max - xk_min) + 1;
            float* win = swin + (st * NQ + qq) * kWinFloats;
            // The ndy x width entries in batches of 8 loads per lane, all in flight before any is
            // stored (width >= 32, so a lane's next entry is at most one window row further).
            const float* tab0 = tab + static_cast<int64_t>(dy_lo + p.bias.table_h - 1) * W2 + (dx_lo + p.bias.table_w - 1);
            int rr = 0, cc = lane;
            while (rr < ndy) {
              float v[8];
              int dst[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                dst[k] = rr < ndy ? rr * win_stride + cc : -1;
                if (rr < ndy) v[k] = __ldg(tab0 + static_cast<int64_t>(rr) * W2 + cc);
                cc += 32;
                if (cc >= width) {
                  cc -= width;
                  ++rr;
                }
              }
#pragma unroll
              for (int k = 0; k < 8; ++k)
                if (dst[k] >= 0) win[dst[k]] = v[k];
            }
            if (lane < BN / 32) {
              const int jc = j0 + 32 * lane;
              const int yk = jc / gw;
              swink[(st * NQ + qq) * 4 + lane] =
                  jc < N ? (yk + dy_lo) * win_stride + (jc - yk * gw) + dx_lo : 0;
            }
          }
        }
        __syncwarp();
#ifdef BA_TEST_SKIP_ARRIVE
        // Test build only: the first block's arrival is withheld, so every wait on it runs into
        // its time limit and the kernel reports BA_ERR_TIMEOUT.
        if (lane == 0 && g != 0) mbar_arrive(&bars[Bar::kvfull(st)]);
#else
        if (lane == 0) mbar_arrive(&bars[Bar::kvfull(st)]);
#endif
      }
    }
    // Leave no TMA copy in flight: wait (bounded, even after an abort) for the stages this
    // warp filled last.
    for (int k = (g > S ? g - S : 0); k < g; ++k) wait_bounded(&bars[Bar::kvfull(k % S)], (k / S) & 1, abort_flag, false);
  } else if (warp < 4 && warp >= 4 - C::kExpWarps) {
    // ------------------------------------------------------------ producer: sign expansion
    // The expanding warps split the 128 rows of every Q tile and K block (warp 2 rows 0..63 and
    // warp 3 rows 64..127). The sign rows of the next K block are loaded
    // into registers before this block is written. The Q tiles of an item are written once the
    // MMAs of the previous item have read them (q_empty).
    constexpr int RPL = C::kRowsPerLane;
    const int half = warp - (4 - C::kExpWarps);
    const int rbase = half * (BM / C::kExpWarps);
    int g = 0;
    bool ok = true;
    uint4 nb[RPL];
#pragma unroll
    for (int u = 0; u < RPL; ++u) nb[u] = zero4;
    uint4 pre_q[NQ][RPL];
    for (int it = 0; it < n_items && ok; ++it) {
      int64_t bh;
      int q0;
      item_at(by_head, it, p.H, nqb, BM * NQ, bh, q0);
      const uint4* qrows = reinterpret_cast<const uint4*>(p.bits_q) + bh * N;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int u = 0; u < RPL; ++u) {
          const int row = q0 + q * BM + rbase + lane + 32 * u;
          pre_q[q][u] = row < N ? __ldg(qrows + row) : zero4;
        }
      if (it == 0) {
        const uint4* krows = reinterpret_cast<const uint4*>(p.bits_k) + bh * N;
#pragma unroll
        for (int u = 0; u < RPL; ++u) {
          const int row = rbase + lane + 32 * u;
          nb[u] = row < N ? __ldg(krows + row) : zero4;
        }
      } else if (!wait_warp(&bars[Bar::qempty()], (it - 1) & 1, abort_flag)) {
        break;
      }
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int u = 0; u < RPL; ++u)
          expand_row<DQ>(sQ + q * C::kQBytes, pre_q[q][u], q0 + q * BM + rbase + lane + 32 * u < N,
                         rbase + lane + 32 * u, d);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Bar::qfull()]);
      for (int t = 0; t < T; ++t, ++g) {
        const int st = g % S;
        uint4 cb[RPL];
#pragma unroll
        for (int u = 0; u < RPL; ++u) cb[u] = nb[u];
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
          for (int u = 0; u < RPL; ++u) {
            const int row = nt * BN + rbase + lane + 32 * u;
            nb[u] = (any && row < N) ? __ldg(nrows + row) : zero4;
          }
        }
        if (g >= S && !wait_warp(&bars[Bar::kvempty(st)], ((g / S) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int u = 0; u < RPL; ++u) {
          const int r = rbase + lane + 32 * u;
          expand_row<DQ>(sK + st * C::kKBytes, cb[u], t * BN + r < N, r, d);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Bar::kvfull(st)]);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ MMA issuer(s)
    // In order over the blocks j (counted across items): P.V(j) once group j % 2 has written
    // P(j) and the fold of block j - 1 has read the accumulator; then QK(j + 2) into the S buffer
    // that P(j) occupied (issue order keeps P read before S is rewritten). QK(0) and QK(1) first.
    if (lane == 0) {
      const uint32_t idesc_qk = (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                (static_cast<uint32_t>(BM >> 4) << 24);
      const uint32_t idesc_pv = (2u << 4) | (0u << 7) | (1u << 10) | (1u << 16) |
                                (static_cast<uint32_t>(DP >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
      const int nblocks = n_items * T;
      auto qk = [&](int j) -> bool {
        const int t = j % T;
        if (t == 0) {
          if (!wait_bounded(&bars[Bar::qfull()], (j / T) & 1, abort_flag)) return false;
          tc_fence_after();
        }
        if (!wait_bounded(&bars[Bar::kvfull(j % S)], (j / S) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t qb = smem_u32(sQ), kb = smem_u32(sK + (j % S) * C::kKBytes);
#pragma unroll
        for (int kk = 0; kk < DQ / 32; ++kk)
          mma_f8f6f4_ss(tmem + C::tS(0, j & 1), smem_desc(qb + kk * 4096, 2048, 128),
                        smem_desc(kb + kk * 4096, 2048, 128), idesc_qk, kk > 0 ? 1u : 0u);
        tc_commit(&bars[Bar::sfull(0, j & 1)]);
        if (t == T - 1) tc_commit(&bars[Bar::qempty()]);  // the item's Q tile is free
        return true;
      };
      if constexpr (C::kTilePP) {
        // Two tiles, one S buffer and one accumulator each: P.V(q, n) once tile q's softmax has
        // written P(n) (it folds block n - 1 out of the accumulator before that), then QK(q, n + 1)
        // into the same S buffer (issue order keeps P read before S is rewritten). Tile 0's next
        // QK is issued before tile 1's P.V wait, so neither tile's softmax waits on the other's.
        auto qk_tile = [&](int q, int n) -> bool {
          const int t = n % T;
          if (q == 0) {
            if (t == 0 && !wait_bounded(&bars[Bar::qfull()], (n / T) & 1, abort_flag)) return false;
            if (!wait_bounded(&bars[Bar::kvfull(n % S)], (n / S) & 1, abort_flag)) return false;
            tc_fence_after();
          }
          const uint32_t qb = smem_u32(sQ + q * C::kQBytes), kb = smem_u32(sK + (n % S) * C::kKBytes);
#pragma unroll
          for (int kk = 0; kk < DQ / 32; ++kk)
            mma_f8f6f4_ss(tmem + C::tS(q, 0), smem_desc(qb + kk * 4096, 2048, 128),
                          smem_desc(kb + kk * 4096, 2048, 128), idesc_qk, kk > 0 ? 1u : 0u);
          tc_commit(&bars[Bar::sfull(q, 0)]);
          if (q == 1 && t == T - 1) tc_commit(&bars[Bar::qempty()]);  // both tiles of the item read Q
          return true;
        };
        auto pv_tile = [&](int q, int n) -> bool {
          if (!wait_bounded(&bars[Bar::pfull(q)], n & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t vbase = smem_u32(sV + (n % S) * C::kVBytes);
#pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk)
            mma_i8_ts(tmem + C::tAcc(q), tmem + C::tS(q, 0) + 8 * kk, smem_desc(vbase + 512 * kk, 128, 2048),
                      idesc_pv, 1u);
          tc_commit(&bars[Bar::pvdone(q)]);
          if (q == 1) tc_commit(&bars[Bar::kvempty(n % S)]);  // the last reader of stage n
          return true;
        };
        bool ok = nblocks == 0 || (qk_tile(0, 0) && qk_tile(1, 0));
        for (int n = 0; n < nblocks && ok; ++n) {
          const bool more = n + 1 < nblocks;
          ok = pv_tile(0, n) && (!more || qk_tile(0, n + 1)) && pv_tile(1, n) && (!more || qk_tile(1, n + 1));
        }
      } else {
      bool ok = nblocks == 0 || qk(0);
      if (ok && nblocks > 1) ok = qk(1);
      for (int j = 0; j < nblocks && ok; ++j) {
        if (!wait_bounded(&bars[Bar::pfull(j & 1)], (j >> 1) & 1, abort_flag)) break;
        if (j > 0 && !wait_bounded(&bars[Bar::folddone((j - 1) & 1)], ((j - 1) >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t vbase = smem_u32(sV + (j % S) * C::kVBytes);
#pragma unroll
        for (int kk = 0; kk < BN / 32; ++kk)
          mma_i8_ts(tmem + C::tAcc(0), tmem + C::tS(0, j & 1) + 8 * kk, smem_desc(vbase + 512 * kk, 128, 2048),
                    idesc_pv, 1u);
        tc_commit(&bars[Bar::pvdone(j & 1)]);
        tc_commit(&bars[Bar::kvempty(j % S)]);
        if (j + 2 < nblocks && !qk(j + 2)) break;
      }
      }
      // Every MMA this thread issued has completed before tensor memory is released.
      tc_commit(&bars[Bar::drain()]);
      wait_bounded(&bars[Bar::drain()], 0, abort_flag, false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    // Group g (warps 4 + 4g .. 7 + 4g) takes the key blocks j with j % 2 == g, one thread per
    // query row (warp w reads tensor-memory lanes 32 (w % 4) ..). While one group evaluates the
    // exponentials of its block, the other forms the logits of the next: the two phases use
    // different units (transcendental unit against shared-memory loads) and overlap.
    //   * The running maximum passes from group to group: the group of block j waits for m_{j-1}
    //     (mchain), forms m_j and publishes it.
    //   * Each block is weighted by e_j = exp(m_j - m_ref) against a per-row reference m_ref
    //     (the item's first block maximum, moved up when e_j would leave float range): the
    //     output sum F' = sum_j acc_j e_j (tensor memory) and the softmax sum L' = sum_j l_j e_j
    //     (shared memory) give O = F' v_scale / (255 L'), the blockwise online softmax's result.
    //   * The fold of block j (F' += acc_j e_j, L' += l_j e_j) is done by block j's group after
    //     P.V(j); P.V(j + 1) waits for it (one accumulator), so the folds, and every update of
    //     F', L' and m_ref, run in block order.
    const int grp = (warp - 4) >> 2, w4 = warp & 3;
    const int qt = C::kTilePP ? grp : 0;  // this group's query tile
    const int r = w4 * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(w4 * 32) << 16;
    const uint32_t aAcc = tmem + lane_base + C::tAcc(qt);
    const uint32_t aF = tmem + lane_base + C::tF(qt);
    float* s_m = reinterpret_cast<float*>(smem + C::offX);  // [2][BM] m_j by block parity
    // [tile][BM] (L', m_ref) of each row, stored as one 8-byte pair so that a reader outside the
    // fold chain sees a consistent pair.
    float2* s_Lm = reinterpret_cast<float2*>(s_m + 2 * BM) + qt * BM;
    uint64_t* mch = &bars[Bar::mchain(w4)];
    // Largest change of an output that one fast code off by one may cause in a row that is not
    // checked (a quarter of a 2e-3 output tolerance).
    constexpr float kCheckTau = 5.0e-4f;
    bool alive = true;
    float mu_q_next = 0.0f, mu_k_next = 0.0f;  // mu of the item about to start (loaded one item ahead)
    int n0 = 0;  // index, counted across items, of the item's first key block
    // The P.V accumulator holds the bit pattern of 1.5 * 2^23 whenever no product is in it: every
    // P.V accumulates onto it, so a block's s32 result reads directly as the float
    // 1.5 * 2^23 + acc (|acc| < 2^22), and whoever reads a product restores the pattern. Each
    // group sets its rows once here (tile ping-pong: its own tile; block ping-pong: group 0 for
    // the shared accumulator), before its first P arrival.
    uint32_t kmag[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) kmag[k] = kMagicBits;
    if (C::kTilePP || grp == 0) {
#pragma unroll
      for (int c = 0; c < DP; c += 16) tmem_st_cols<16>(aAcc + c, kmag);
    }
    for (int it = 0; it < n_items && alive; ++it, n0 += T) {
      int64_t bh;
      int q0;
      item_at(by_head, it, p.H, nqb, BM * NQ, bh, q0);
      const int64_t b = bh / p.H, h = bh - b * p.H;
      const int i = q0 + qt * BM + r;
      const bool row_ok = i < N;
      const int ic = row_ok ? i : N - 1;  // rows past N read the bias of row N-1 (never stored)
      if (it == 0) {
        mu_q_next = p.mu_q[bh];
        mu_k_next = p.mu_k[bh];
      }
      const float alpha = __fmul_rn(__fmul_rn(p.softmax_scale, mu_q_next), mu_k_next);
      const float2 alpha2 = make_float2(alpha, alpha);
      // The head's largest |V| (127 times its largest channel scale) bounds what one changed
      // code can move an output by: |v| / (255 l). Blocks of rows whose softmax sum l is below
      // l_check = max|V| / (255 tau) get their near-tie codes recomputed exactly.
      float vmax = 0.0f;
#pragma unroll
      for (int k = 0; k < (DP + 31) / 32; ++k)
        if (32 * k + lane < d) vmax = fmaxf(vmax, p.v_scale[bh * d + 32 * k + lane]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      const float l_check = (127.0f * vmax) / (255.0f * kCheckTau);

      // Bias addressing. Dense: this row of [H][N][N]. General rel-pos: b_ij = tab[a_i - koff_j]
      // (table staged in shared memory when it fits, followed by zeros that class-token rows and
      // keys index into). Window: b_ij = window[A_i - K_c - u].
      const float* brow = nullptr;
      const float* gtab = nullptr;
      int a_i = 0;
      if constexpr (BK == kBiasDense) brow = p.bias.data + b * p.bias.batch_stride + (h * N + ic) * N;
      if constexpr (is_relpos_general(BK)) {
        const int W2 = 2 * p.bias.table_w - 1;
        gtab = p.bias.data + h * static_cast<int64_t>(2 * p.bias.table_h - 1) * W2;
        if (ic >= p.bias.n_prefix) {
          const int ti = ic - p.bias.n_prefix;
          const int yi = ti / p.bias.grid_w;
          a_i = (yi + p.bias.table_h - 1) * W2 + (ti - yi * p.bias.grid_w) + p.bias.table_w - 1;
        } else {
          a_i = (tab_mode == 2) ? tsize + kmax : -1;  // class-token row: the zeros (or the per-key test)
        }
      }
      int A_i = 0;
      if constexpr (BK == kRelWindow) {
        const int yi = ic / p.bias.grid_w;
        A_i = yi * win_stride + (ic - yi * p.bias.grid_w);
      }
      const bool dense_vec = BK == kBiasDense && (N & 3) == 0 && (p.bias.batch_stride & 3) == 0;
      // (L', m_ref) after this group's last fold in the item (own registers: the check decision
      // below must not depend on when the other group's fold lands, or results would vary
      // from run to run); L' = 0 before the group's first fold of the item.
      float own_L = 0.0f, own_mref = 0.0f;
      // Tile ping-pong: the running maximum, and the sum and maximum of the block awaiting its
      // fold, in registers.
      float m_run = -CUDART_INF_F, lt_prev = 0.0f;

      // The fold of block tb (item-relative; running maximum m_b, sum of P~ lt_b):
      // F' += acc e, L' += lt_b e with e = exp(m_b - m_ref) (the item's first block sets F' = acc,
      // L' = lt_b, m_ref = m_b; e beyond 2^64 moves m_ref up to m_b, rescaling F' and L').
      auto fold_block = [&](int tb, float m_b, float lt_b) {
        float e = 1.0f, ratio = 1.0f;
        float mref = m_b, Lp = 0.0f;
        if (tb > 0) {
          const float2 lm = s_Lm[r];
          Lp = lm.x;
          mref = lm.y;
          e = ex2_approx((m_b - mref) * kLog2e);
          if (e > 1.8446744e19f) {
            ratio = 1.0f / e;
            e = 1.0f;
            mref = m_b;
          }
        }
        const bool rescale = __any_sync(0xffffffffu, ratio != 1.0f);
        auto fold = [&](auto first) {
          constexpr bool FIRST = decltype(first)::value;
#pragma unroll 1
          for (int c0 = 0; c0 < DP; c0 += 32) {
            constexpr int G = 32;
            uint32_t a[G], f[G];
            if (c0 + G <= DP) {
              tmem_ld_cols<G>(aAcc + c0, a);
              if (!FIRST) tmem_ld_cols<G>(aF + c0, f);
            } else {
              tmem_ld_cols<16>(aAcc + c0, a);
              if (!FIRST) tmem_ld_cols<16>(aF + c0, f);
            }
            tmem_ld_wait();
            reg_fence_cols<G>(a);
            if (!FIRST) reg_fence_cols<G>(f);
            const float2 e2 = make_float2(e, e), rt2 = make_float2(ratio, ratio);
#pragma unroll
            for (int k = 0; k < G; k += 2) {
              const float2 a2 = __fadd2_rn(make_float2(__uint_as_float(a[k]), __uint_as_float(a[k + 1])),
                                           make_float2(-kMagic, -kMagic));
              float2 f2;
              if (FIRST) {
                f2 = a2;
              } else {
                float2 fo = make_float2(__uint_as_float(f[k]), __uint_as_float(f[k + 1]));
                if (rescale) fo = __fmul2_rn(fo, rt2);
                f2 = __ffma2_rn(a2, e2, fo);
              }
              f[k] = __float_as_uint(f2.x);
              f[k + 1] = __float_as_uint(f2.y);
            }
            if (c0 + G <= DP) {
              tmem_st_cols<G>(aF + c0, f);
              tmem_st_cols<G>(aAcc + c0, kmag);
            } else {
              tmem_st_cols<16>(aF + c0, f);
              tmem_st_cols<16>(aAcc + c0, kmag);
            }
          }
        };
        if (tb == 0)
          fold(std::true_type{});
        else
          fold(std::false_type{});
        own_L = (tb == 0) ? lt_b : __fmaf_rn(lt_b, e, Lp * ratio);
        own_mref = mref;
        s_Lm[r] = make_float2(own_L, own_mref);
      };

      for (int t = C::kTilePP ? 0 : (grp ^ (n0 & 1)); t < T && alive; t += C::kTilePP ? 1 : 2) {
        const int n = n0 + t;
        const int st = n % S;
        const int j0 = t * BN;
        const int nk = min(BN, N - j0);  // valid keys of this block
        const uint32_t aS = tmem + lane_base + (C::kTilePP ? C::tS(qt, 0) : C::tS(0, n & 1));
        if constexpr (BK == kRelWindow || is_relpos_general(BK)) {
          if (!wait_warp(&bars[Bar::kvfull(st)], (n / S) & 1, abort_flag)) {
            alive = false;
            break;
          }
        }
        if (!wait_warp(&bars[C::kTilePP ? Bar::sfull(qt, 0) : Bar::sfull(0, n & 1)],
                       C::kTilePP ? (n & 1) : ((n >> 1) & 1), abort_flag)) {
          alive = false;
          break;
        }
        tc_fence_after();

        // ---- pass 1: s = alpha x + b over four 32-key chunks (the next chunk's load in flight
        // while this one is formed), written back over S; the block maximum.
        float mx[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
        auto pass1 = [&](auto masked) {
          constexpr bool MASK = decltype(masked)::value;
          // A rolled loop over pairs of chunks (two copies of the chunk body, not four, keep the
          // hot code in the instruction cache); buffers xa / xb alternate, the next chunk's load
          // in flight while this one is worked on.
          uint32_t xa[32], xb[32];
          tmem_ld_cols<32>(aS, xa);
#pragma unroll 1
          for (int cp = 0; cp < BN / 64; ++cp)
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int c = 2 * cp + h2;
            uint32_t* x = h2 ? xb : xa;
            uint32_t* xn = h2 ? xa : xb;
            tmem_ld_wait();
            reg_fence_cols<32>(x);
            if (c + 1 < BN / 32) tmem_ld_cols<32>(aS + 32 * (c + 1), xn);
            const int jc = j0 + 32 * c;  // first key of this chunk
            if (DBG && p.dbg_logits != nullptr && row_ok) {
#pragma unroll
              for (int u = 0; u < 32; ++u)
                if (32 * c + u < nk) p.dbg_logits[(bh * N + i) * N + jc + u] = __float2int_rn(__uint_as_float(x[u]));
            }
            const float* wrow = nullptr;
            (void)wrow;
            if constexpr (BK == kRelWindow) {
              // Every chunk lies in one grid row (grid width a multiple of 32, N = grid size), so
              // its 32 biases are a descending run of the window. Chunks past N are masked.
              const int kc = jc < N ? swink[(st * NQ + qt) * 4 + c] : A_i - 31;
              wrow = swin + (st * NQ + qt) * kWinFloats + (A_i - kc);
            }
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              float bv[8];
              const int j8 = jc + 8 * g8;
              (void)j8;
              if constexpr (BK == kBiasNone) {
#pragma unroll
                for (int u = 0; u < 8; ++u) bv[u] = 0.0f;
              } else if constexpr (BK == kBiasDense) {
                if (dense_vec && j8 + 8 <= N) {
                  const float4 v0 = __ldg(reinterpret_cast<const float4*>(brow + j8));
                  const float4 v1 = __ldg(reinterpret_cast<const float4*>(brow + j8) + 1);
                  bv[0] = v0.x; bv[1] = v0.y; bv[2] = v0.z; bv[3] = v0.w;
                  bv[4] = v1.x; bv[5] = v1.y; bv[6] = v1.z; bv[7] = v1.w;
                } else {
#pragma unroll
                  for (int u = 0; u < 8; ++u) bv[u] = (j8 + u < N) ? __ldg(brow + j8 + u) : 0.0f;
                }
              } else if constexpr (BK == kRelWindow) {
#pragma unroll
                for (int u = 0; u < 8; ++u) bv[u] = wrow[-(8 * g8 + u)];
              } else {
                const uint32_t ko = smem_u32(koff + st * BN + 32 * c + 8 * g8);
                if (BK == kRelSmem && tab_mode == 2) {
                  const uint32_t tb = smem_u32(stab) + 4u * static_cast<uint32_t>(a_i);
                  const int4 o0 = lds_s32x4(ko), o1 = lds_s32x4(ko + 16u);
                  bv[0] = lds_f32(tb - 4u * o0.x); bv[1] = lds_f32(tb - 4u * o0.y);
                  bv[2] = lds_f32(tb - 4u * o0.z); bv[3] = lds_f32(tb - 4u * o0.w);
                  bv[4] = lds_f32(tb - 4u * o1.x); bv[5] = lds_f32(tb - 4u * o1.y);
                  bv[6] = lds_f32(tb - 4u * o1.z); bv[7] = lds_f32(tb - 4u * o1.w);
                } else {
#pragma unroll
                  for (int u = 0; u < 8; ++u) {
                    const int kj = lds_s32(ko + 4u * u);
                    float bias = 0.0f;
                    if (a_i >= 0 && kj >= 0)
                      bias = (BK == kRelSmem) ? lds_f32(smem_u32(stab) + 4u * static_cast<uint32_t>(a_i - kj))
                                              : __ldg(gtab + (a_i - kj));
                    bv[u] = bias;
                  }
                }
              }
#pragma unroll
              for (int u = 0; u < 8; u += 2) {
                const int k = 8 * g8 + u;
                float2 s2;
                if constexpr (BK == kBiasNone)
                  s2 = __fmul2_rn(alpha2, make_float2(__uint_as_float(x[k]), __uint_as_float(x[k + 1])));
                else
                  s2 = __ffma2_rn(alpha2, make_float2(__uint_as_float(x[k]), __uint_as_float(x[k + 1])),
                                  make_float2(bv[u], bv[u + 1]));
                if (MASK) {
                  if (32 * c + k >= nk) s2.x = -CUDART_INF_F;
                  if (32 * c + k + 1 >= nk) s2.y = -CUDART_INF_F;
                }
                x[k] = __float_as_uint(s2.x);
                x[k + 1] = __float_as_uint(s2.y);
                mx[(u >> 1) & 3] = fmax3(mx[(u >> 1) & 3], s2.x, s2.y);
              }
            }
            tmem_st_cols<32>(aS + 32 * c, x);
          }
        };
        if (nk < BN)
          pass1(std::true_type{});
        else
          pass1(std::false_type{});
        const float bmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        tmem_st_wait();  // s is in S before pass 2 reads it back

        // ---- the running maximum: tile ping-pong, in a register; block ping-pong, m_{n-1} from
        // the other group (block n - 1), then m_n out
        float m_prev = -CUDART_INF_F;
        if constexpr (C::kTilePP) {
          m_prev = (t == 0) ? -CUDART_INF_F : m_run;
        } else {
          if (n > 0) {
            if (!wait_warp(mch, (n - 1) & 1, abort_flag)) {
              alive = false;
              break;
            }
            if (t > 0) m_prev = s_m[((n - 1) & 1) * BM + r];
          }
        }
        const float m_new = fmaxf(m_prev, bmax);
        if constexpr (!C::kTilePP) {
          s_m[(n & 1) * BM + r] = m_new;
          __syncwarp();
          if (lane == 0) mbar_arrive(mch);
        } else if (t > 0) {
          // Fold block n - 1 (its P.V completed before QK(n), which this block's S came from).
          if (!wait_warp(&bars[Bar::pvdone(qt)], (n - 1) & 1, abort_flag)) {
            alive = false;
            break;
          }
          tc_fence_after();
          fold_block(t - 1, m_prev, lt_prev);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[Bar::folddone(qt)]);
        }
        // Rows whose softmax sum so far is small get the exact near-tie check. The sum is taken
        // as of this group's own last fold (an underestimate of the row's true sum).
        const float l_so_far = own_L > 0.0f ? own_L * ex2_approx((own_mref - m_new) * kLog2e) : 0.0f;
        const bool check = p.p_check_all || __any_sync(0xffffffffu, l_so_far + 1.0f < l_check);

        // ---- pass 2: P~ = 2^((s - m) log2 e), row sum, 8-bit codes (masked keys: s = -inf,
        // P~ = 0) per 32-key chunk; in check mode each 4-key word's near-tie codes are settled in
        // place. The codes go to columns 8c .. 8c + 7 of the S buffer (keys 0..31 of S, read
        // already).
        const float2 negm2 = make_float2(-m_new, -m_new);
        const float2 log2e2 = make_float2(kLog2e, kLog2e);
        const float2 c255 = make_float2(255.0f, 255.0f);
        const float2 c255lo = make_float2(kC255Lo, kC255Lo);
        const float2 c255hi = make_float2(kC255Hi, kC255Hi);
        const float2 magic2 = make_float2(kMagic, kMagic);
        float2 lt2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
        auto pass2 = [&](auto checked) {
          constexpr bool CHECK = decltype(checked)::value;
          // A rolled loop over pairs of chunks (two copies of the chunk body, not four, keep the
          // hot code in the instruction cache); buffers xa / xb alternate, the next chunk's load
          // in flight while this one is worked on.
          uint32_t xa[32], xb[32];
          tmem_ld_cols<32>(aS, xa);
#pragma unroll 1
          for (int cp = 0; cp < BN / 64; ++cp)
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int c = 2 * cp + h2;
            uint32_t* x = h2 ? xb : xa;
            uint32_t* xn = h2 ? xa : xb;
            tmem_ld_wait();
            reg_fence_cols<32>(x);
            if (c + 1 < BN / 32) tmem_ld_cols<32>(aS + 32 * (c + 1), xn);
            uint32_t pk[8], pl[8];
            uint32_t dif = 0u;  // check mode: nonzero where a word's two roundings disagree
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              uint32_t y[4], yl[4];
#pragma unroll
              for (int e2 = 0; e2 < 2; ++e2) {
                const int k = 4 * w + 2 * e2;
                // s - m first (exact near the maximum), then the scale to base 2.
                const float2 t2 = __fmul2_rn(
                    __fadd2_rn(make_float2(__uint_as_float(x[k]), __uint_as_float(x[k + 1])), negm2), log2e2);
                const float2 p2 = make_float2(ex2_approx(t2.x), ex2_approx(t2.y));
                lt2[e2] = __fadd2_rn(lt2[e2], p2);
                // 255 P~ + 1.5 * 2^23: one rounding to the nearest integer (ties to even); the
                // integer sits in the low byte of the result (P~ <= 1).
                const float2 y2 = __ffma2_rn(p2, CHECK ? c255hi : c255, magic2);
                y[2 * e2] = __float_as_uint(y2.x);
                y[2 * e2 + 1] = __float_as_uint(y2.y);
                if (CHECK) {
                  const float2 z2 = __ffma2_rn(p2, c255lo, magic2);
                  yl[2 * e2] = __float_as_uint(z2.x);
                  yl[2 * e2 + 1] = __float_as_uint(z2.y);
                }
              }
              pk[w] = __byte_perm(__byte_perm(y[0], y[1], 0x0040), __byte_perm(y[2], y[3], 0x0040), 0x5410);
              if (CHECK) {
                pl[w] = __byte_perm(__byte_perm(yl[0], yl[1], 0x0040), __byte_perm(yl[2], yl[3], 0x0040), 0x5410);
                dif |= pk[w] ^ pl[w];
              }
            }
            if (CHECK && dif != 0u) {
              // Rare: settle the chunk's near-tie words.
#pragma unroll
              for (int w = 0; w < 8; ++w)
                if (pl[w] != pk[w]) pk[w] = settle_ties(pk[w], pl[w], x + 4 * w, m_new, tie);
            }
            tmem_st_cols<8>(aS + 8 * c, pk);
            if (DBG && p.dbg_p != nullptr && row_ok) {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (32 * c + k < nk)
                  p.dbg_p[(bh * N + i) * N + j0 + 32 * c + k] = static_cast<uint8_t>(pk[k >> 2] >> (8 * (k & 3)));
            }
          }
        };
        if (check)
          pass2(std::true_type{});
        else
          pass2(std::false_type{});
        const float lt = (lt2[0].x + lt2[0].y) + (lt2[1].x + lt2[1].y);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Bar::pfull(grp)]);
        if constexpr (C::kTilePP) {
          m_run = m_new;
          lt_prev = lt;
          continue;
        }

        // ---- fold block n: F' += acc e_n, L' += l_n e_n (after P.V(n), which followed the fold
        // of block n - 1; at an item's first block also after both groups' previous epilogue)
        if (!wait_warp(&bars[Bar::pvdone(grp)], (n >> 1) & 1, abort_flag)) {
          alive = false;
          break;
        }
        if (n > 0 && !wait_warp(&bars[Bar::folddone(grp ^ 1)], ((n - 1) >> 1) & 1, abort_flag)) {
          alive = false;
          break;
        }
        if (t == 0 && it > 0 && !wait_warp(&bars[Bar::epidone()], (it - 1) & 1, abort_flag)) {
          alive = false;
          break;
        }
        tc_fence_after();
        fold_block(t, m_new, lt);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Bar::folddone(grp)]);
      }
      if (!alive) break;

      // ---- epilogue: O = F' v_scale / (255 L'), channels 64 grp .. (DP / 2 per group), once
      // the item's last block is folded; then both groups release F' for the next item.
      if (it + 1 < n_items) {
        int64_t nbh;
        int nq0;
        item_at(by_head, it + 1, p.H, nqb, BM * NQ, nbh, nq0);
        mu_q_next = p.mu_q[nbh];
        mu_k_next = p.mu_k[nbh];
      }
      const int nl = n0 + T - 1;  // the item's last block
      // Tile ping-pong: the last block is not folded into F'; the epilogue forms
      // O = (F' ratio + acc e) v_scale / (255 L') from both, with the fold's arithmetic.
      float e_last = 1.0f, r_last = 1.0f, L_fin;
      bool last_only = false;  // the item's only block: O = acc v_scale / (255 l)
      if constexpr (C::kTilePP) {
        if (!wait_warp(&bars[Bar::pvdone(qt)], nl & 1, abort_flag)) {
          alive = false;
          break;
        }
        last_only = (T == 1);
        float Lp = 0.0f;
        if (!last_only) {
          const float2 lm = s_Lm[r];
          Lp = lm.x;
          e_last = ex2_approx((m_run - lm.y) * kLog2e);
          if (e_last > 1.8446744e19f) {
            r_last = 1.0f / e_last;
            e_last = 1.0f;
          }
        }
        L_fin = last_only ? lt_prev : __fmaf_rn(lt_prev, e_last, Lp * r_last);
      } else {
        if (!wait_warp(&bars[Bar::folddone(nl & 1)], (nl >> 1) & 1, abort_flag)) {
          alive = false;
          break;
        }
        L_fin = 0.0f;
      }
      tc_fence_after();
      if constexpr (!C::kTilePP) L_fin = s_Lm[r].x;
      const float inv_l = 1.0f / (255.0f * L_fin);
      const int esz = (p.o_dt == BA_F32) ? 4 : 2;
      const bool vec = ((d * esz) & 15) == 0;
      // Block ping-pong: each group writes half of the row's channels; tile ping-pong: all.
      constexpr int kChan = C::kTilePP ? DP : DH;
#pragma unroll 1
      for (int g0 = 0; g0 < kChan; g0 += 8) {
        const int c0 = (C::kTilePP ? 0 : grp * DH) + g0;  // eight channels at a time
        uint32_t f[8];
        if constexpr (C::kTilePP) {
          uint32_t a[8];
          tmem_ld_cols<8>(aAcc + c0, a);
          if (!last_only) tmem_ld_cols<8>(aF + c0, f);
          tmem_ld_wait();
          reg_fence8(a);
          if (!last_only) reg_fence8(f);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float av = __fadd_rn(__uint_as_float(a[k]), -kMagic);
            const float fo = last_only ? 0.0f : (r_last != 1.0f ? __fmul_rn(__uint_as_float(f[k]), r_last)
                                                                : __uint_as_float(f[k]));
            f[k] = __float_as_uint(last_only ? av : __fmaf_rn(av, e_last, fo));
          }
          tmem_st_cols<8>(aAcc + c0, kmag);
        } else {
          tmem_ld_cols<8>(aF + c0, f);
          tmem_ld_wait();
          reg_fence8(f);
        }
        float val[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float sv = (c0 + k < d) ? __ldg(p.v_scale + bh * d + c0 + k) : 0.0f;
          val[k] = __uint_as_float(f[k]) * (sv * inv_l);
        }
        if (!row_ok) continue;
        char* orow = reinterpret_cast<char*>(p.o) + ((bh * N + i) * d + c0) * esz;
        if (vec && c0 + 8 <= d) {
          if (p.o_dt == BA_F32) {
            reinterpret_cast<float4*>(orow)[0] = make_float4(val[0], val[1], val[2], val[3]);
            reinterpret_cast<float4*>(orow)[1] = make_float4(val[4], val[5], val[6], val[7]);
          } else {
            uint32_t hw[4];
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              if (p.o_dt == BA_F16) {
                const __half2 hv = __floats2half2_rn(val[2 * k2], val[2 * k2 + 1]);
                hw[k2] = *reinterpret_cast<const uint32_t*>(&hv);
              } else {
                const __nv_bfloat162 hv = __floats2bfloat162_rn(val[2 * k2], val[2 * k2 + 1]);
                hw[k2] = *reinterpret_cast<const uint32_t*>(&hv);
              }
            }
            reinterpret_cast<uint4*>(orow)[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (c0 + k < d) store_out(p.o, (bh * N + i) * d + c0 + k, val[k], p.o_dt);
        }
      }
      if constexpr (!C::kTilePP) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Bar::epidone()]);
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  named_barrier_sync(1, C::kThreads);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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

constexpr int kMaxSmem = 227 * 1024;  // per CTA

// 0: rel-pos table read from global memory; 1: staged in shared memory; 2: staged and followed
// by 2 * tsize zeros that class-token rows and keys index into.
template <class C>
int relpos_table_mode(const AttnParams& p) {
  const int64_t tsize = static_cast<int64_t>(2 * p.bias.table_h - 1) * (2 * p.bias.table_w - 1);
  const int64_t room = kMaxSmem - 1024 - C::kTabOff;
  if (p.bias.n_prefix > 0 && 3 * tsize * 4 <= room) return 2;
  if (tsize * 4 <= room) return 1;
  return 0;
}

// Row stride of the rel-pos window, or 0 when the window form does not apply: it needs a grid
// width that is a multiple of 32 (so that every 32-key chunk lies in one grid row), no class
// tokens, and a window of at most kWinFloats entries for every (tile, block) pair. A run of 128
// tokens spans at most 127 / gw + 2 grid rows; the dx extent is at most 255 when the tiles and
// blocks cannot straddle grid rows (gw a multiple of 128), else 2 gw - 1.
int window_stride(const AttnParams& p) {
  if (p.bias.kind != BA_BIAS_RELPOS2D || p.bias.n_prefix != 0) return 0;
  const int gw = p.bias.grid_w;
  if (gw % 32 != 0) return 0;
  const int ws = (gw % 128 == 0) ? 256 : ((2 * gw - 1 + 3) / 4) * 4;
  const int ndy = 2 * (127 / gw + 2) - 1;
  return static_cast<int64_t>(ndy) * ws <= kWinFloats ? ws : 0;
}

// The thresholds of the exact P codes (TieTable): thr[k] is the least double d with
// code(d) >= k + 1, code(d) = min(255, rne(fl32(255 fl32(exp(d))))), found by bisection between
// adjacent doubles (code(-1000) = 0, code(0) = 255). Computed once per process.
const TieTable& tie_table() {
  static const TieTable table = [] {
    TieTable t{};
    auto code = [](double d) {
      const float pe = static_cast<float>(std::exp(d));
      const float c = std::nearbyint(255.0f * pe);
      return c > 255.0f ? 255 : static_cast<int>(c);
    };
    for (int k = 0; k < 255; ++k) {
      double lo = -1000.0, hi = 0.0;
      for (;;) {
        const double mid = lo + 0.5 * (hi - lo);
        if (!(mid > lo && mid < hi)) break;
        if (code(mid) >= k + 1)
          hi = mid;
        else
          lo = mid;
      }
      t.thr[k] = hi;
    }
    t.thr[255] = HUGE_VAL;  // a settled key's lower code is at most 254
    return t;
  }();
  return table;
}

template <int DP, int BK, bool DBG>
cudaError_t launch_cfg(const AttnParams& p, const CUtensorMap& tm, cudaStream_t s) {
  using C = Cfg<DP, BK>;
  int tab_mode = 0, tsize = 0, kmax = 0, wst = 0;
  if (BK == kRelSmem || BK == kRelGlobal || BK == kRelWindow) {
    tsize = (2 * p.bias.table_h - 1) * (2 * p.bias.table_w - 1);
    kmax = (p.bias.grid_h - 1) * (2 * p.bias.table_w - 1) + p.bias.grid_w - 1;
  }
  if (BK == kRelSmem) tab_mode = relpos_table_mode<C>(p);
  if (BK == kRelWindow) wst = window_stride(p);
  const int tab_bytes = tab_mode == 0 ? 0 : (tab_mode == 2 ? 3 : 1) * tsize * 4;
  // One CTA per SM (it owns all 512 tensor-memory columns): take enough shared memory that no
  // second CTA is placed beside it.
  int smem = C::kTabOff + tab_bytes + 1024;
  if (smem < 116 * 1024) smem = 116 * 1024;
  auto kernel = attn_tc_kernel<DP, BK, DBG>;
  static int configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // Persistent CTAs, one per SM; grouped by head (at least one CTA per head) when the head's
  // table is staged.
  const int64_t per_head = static_cast<int64_t>(p.B) * ceil_div(p.N, BM * C::NQ);
  int64_t grid;
  if (BK == kRelSmem) {
    const int64_t k = std::max<int64_t>(1, std::min<int64_t>(per_head, sms / p.H));
    grid = k * p.H;
  } else {
    grid = std::min<int64_t>(per_head * p.H, sms);
  }
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
  return cudaLaunchKernelEx(&cfg, kernel, p, tm, tab_mode, tsize, kmax, wst, tie_table());
}

template <int DP, int BK>
cudaError_t launch_bk(const AttnParams& p, const CUtensorMap& tm, cudaStream_t s) {
  if (p.dbg_logits != nullptr || p.dbg_p != nullptr) return launch_cfg<DP, BK, true>(p, tm, s);
  return launch_cfg<DP, BK, false>(p, tm, s);
}

template <int DP>
cudaError_t launch_dp(const AttnParams& p, const CUtensorMap& tm, cudaStream_t s) {
  switch (p.bias.kind) {
    case BA_BIAS_DENSE: return launch_bk<DP, kBiasDense>(p, tm, s);
    case BA_BIAS_RELPOS2D:
      if (window_stride(p) != 0) return launch_bk<DP, kRelWindow>(p, tm, s);
      return relpos_table_mode<Cfg<DP, kRelSmem>>(p) != 0 ? launch_bk<DP, kRelSmem>(p, tm, s)
                                                          : launch_bk<DP, kRelGlobal>(p, tm, s);
    default: return launch_bk<DP, kBiasNone>(p, tm, s);
  }
}

}  // namespace

double p_code_threshold(int k) { return (k >= 0 && k < 255) ? tie_table().thr[k] : std::nan(""); }

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
#ifdef BA_TEST_SKIP_ARRIVE
  // Test build: one kernel variant (d = 64, no bias) is enough to exercise the bounded waits.
  if (p.dp != 64 || p.bias.kind != BA_BIAS_NONE) return cudaErrorNotSupported;
  return launch_cfg<64, kBiasNone, false>(p, tm, s);
#endif
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
