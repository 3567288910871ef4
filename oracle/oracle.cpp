// BinaryAttention forward — CPU oracle (test infrastructure only).
//
// This file is a plain, slow, step-by-step restatement of the BinaryAttention
// forward pass: sign binarisation of Q and K with scale factors mu_q, mu_k,
// the XOR/popcount similarity, the additive bias b_ij, a blockwise (FlashAttention-2
// style) online softmax, an unsigned 8-bit P on [0,1], a per-channel int8 V and an
// integer P.V, dequantised at the end.
//
// It is NOT part of the product. Only the tests, the package's smoke check and the
// benchmark's CPU-baseline leg load it. It shares no code, header, table or helper
// with the CUDA library.
//
// Sources (all five pages are summaries of the paper "BinaryAttention: One-Bit
// QK-Attention for Vision and Diffusion Transformers", arXiv 2603.09582):
//   [zh] gist.science/zh/paper/2603.09582, section 技术摘要 (technical summary)
//   [nl] gist.science/nl/paper/2603.09582, section Technische samenvatting
//   [it] gist.science/it/paper/2603.09582, section sintesi tecnica
//   [fr] gist.science/fr/paper/2603.09582, section résumé technique
//   [pt] gist.science/pt/paper/2603.09582, section resumo técnico
//
// Precision: sums, the softmax normaliser and the output accumulation are carried in
// double. Every step whose floating-point result decides an integer code (the logit
// s_ij that feeds exp and the 8-bit P, and the V quantiser) is done in fp32, the
// precision the GPU kernel decides them in. The pages fix no precision.
//
// Where the pages leave a step open, the reading taken is stated at that step.
//
// Parity status: every function here is pinned by the CPU tests (identities, closed
// forms, brute force, statistical laws and a mutation suite); none is "parity unpinned".

#include <cmath>
#include <cstdint>
#include <cstring>
#include <cstdlib>
#include <limits>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr int kWordsPerRow = 4;  // 128 sign bits per token row (head dim d <= 128)

int popcount32(uint32_t v) {
  // Plain bit counting; no builtin, so the count is visibly what it says.
  int n = 0;
  while (v) {
    n += static_cast<int>(v & 1u);
    v >>= 1;
  }
  return n;
}

}  // namespace

extern "C" {

// Version tag so the Python side can check it loaded the right library.
int bao_version(void) { return 3; }

// Step 1 — sign binarisation of a query or key row.
// [zh] §2.2(1) and [fr] §2B: q and k are reduced to sign(q), sign(k) in {-1,+1}.
// Reading: sign(0) is not stated; +0.0, -0.0 and NaN are taken as +1 (bit 0).
// Bit (c mod 32) of word floor(c/32) is 1 iff x_c < 0. Pad bits are 0.
// x: [rows][d] fp32, bits: [rows][4] uint32.
void bao_pack_signs(const float* x, int64_t rows, int d, uint32_t* bits) {
  for (int64_t r = 0; r < rows; ++r) {
    uint32_t w[kWordsPerRow] = {0u, 0u, 0u, 0u};
    for (int c = 0; c < d; ++c) {
      const float v = x[r * d + c];
      if (v < 0.0f) w[c / 32] |= (1u << (c % 32));
    }
    for (int k = 0; k < kWordsPerRow; ++k) bits[r * kWordsPerRow + k] = w[k];
  }
}

// Step 2 — the scale factors mu_q, mu_k.
// [zh] §2.2(1): mu averages over both the token and the channel dimension; [nl] Methodologie 2
// and [pt] §2B say the same. Reading: one mu per (batch, head), the mean of |x| over
// all N*d entries of that slice (the mean of signed x would be ~0 and carry no
// magnitude). Summed in double, stored as fp32.
// x: [BH][N][d], mu: [BH].
void bao_mu(const float* x, int64_t BH, int64_t N, int d, float* mu) {
  for (int64_t s = 0; s < BH; ++s) {
    double acc = 0.0;
    const float* p = x + s * N * d;
    for (int64_t e = 0; e < N * d; ++e) acc += std::fabs(static_cast<double>(p[e]));
    const double cnt = static_cast<double>(N) * static_cast<double>(d);
    mu[s] = (N * d > 0) ? static_cast<float>(acc / cnt) : 0.0f;
  }
}

// Step 3 — binary similarity.
// [zh] §2.1 and [fr] §2A: the dot product of sign vectors equals a Hamming-distance
// form; [zh] §2.2(1) computes it with XNOR and popcount. With d true channels,
// <s,t> = d - 2*popc(s XOR t). Pad bits are 0 in both operands.
// bq, bk: [BH][N][4], x: [BH][N][N] int32.
void bao_logits(const uint32_t* bq, const uint32_t* bk, int64_t BH, int64_t N, int d,
                int32_t* x) {
  for (int64_t s = 0; s < BH; ++s)
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j) {
        int diff = 0;
        for (int k = 0; k < kWordsPerRow; ++k)
          diff += popcount32(bq[(s * N + i) * kWordsPerRow + k] ^ bk[(s * N + j) * kWordsPerRow + k]);
        x[(s * N + i) * N + j] = d - 2 * diff;
      }
}

// Step 5 — channel-aware 8-bit V.
// [zh] §2.2(3): V uses channel-aware 8-bit quantisation; [nl] Methodologie 2: values
// get a channel-specific scale; the P.V instruction named on every page takes a
// signed 8-bit B operand. Reading: symmetric, per (batch, head, channel) over all N
// tokens, range +-127, round to nearest even:
//   amax_c = max_j |v_jc|;  inv = 127/amax_c (fp32);  q = clamp(rne(v*inv), -127, 127);
//   sv_c = amax_c/127 (fp32). A zero channel gives q = 0 and sv_c = 0.
// Reading for a channel so small that 127/amax_c overflows fp32 (amax_c < 127/FLT_MAX, only
// reachable with bf16 inputs): inv is not a float there, so the channel is treated as a zero
// channel (q = 0, sv_c = 0); its whole contribution to O is below 1e-36.
// v: [BH][N][d], vq: [BH][N][d] int8, sv: [BH][d].
void bao_quant_v(const float* v, int64_t BH, int64_t N, int d, int8_t* vq, float* sv) {
  for (int64_t s = 0; s < BH; ++s)
    for (int c = 0; c < d; ++c) {
      float amax = 0.0f;
      for (int64_t j = 0; j < N; ++j) {
        const float a = std::fabs(v[(s * N + j) * d + c]);
        if (a > amax) amax = a;
      }
      if (amax == 0.0f || !std::isfinite(127.0f / amax)) {
        sv[s * d + c] = 0.0f;
        for (int64_t j = 0; j < N; ++j) vq[(s * N + j) * d + c] = 0;
        continue;
      }
      const float inv = 127.0f / amax;
      sv[s * d + c] = amax / 127.0f;
      for (int64_t j = 0; j < N; ++j) {
        const float prod = v[(s * N + j) * d + c] * inv;
        float r = std::nearbyint(prod);  // default rounding mode: nearest, ties to even
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        vq[(s * N + j) * d + c] = static_cast<int8_t>(r);
      }
    }
}

// Bias description shared by the functions below.
// [zh] §2.2(2) and [it] §2B: a learnable bias b_ij is added to the logits; it may be
// dense or position-sensitive. Two forms are built:
//   kind 0: none;
//   kind 1: dense fp32 [H][N][N] per batch, batch b at data + b*batch_stride
//           (batch_stride 0 broadcasts one tensor over the batch);
//   kind 2: 2-D relative position: a table [H][(2*th-1)*(2*tw-1)] indexed by the
//           query-minus-key offset on a gh x gw token grid that starts after
//           n_prefix leading tokens (a class token); prefix rows and columns get 0.
struct bao_bias {
  int kind;
  const float* data;
  int64_t batch_stride;
  int grid_h, grid_w, table_h, table_w, n_prefix;
};

static float bias_value(const bao_bias* bz, int64_t b, int64_t h, int64_t N, int64_t H,
                        int64_t i, int64_t j) {
  if (bz == nullptr || bz->kind == 0) return 0.0f;
  if (bz->kind == 1) return bz->data[b * bz->batch_stride + (h * N + i) * N + j];
  // kind 2: relative (dy, dx) = (query - key) on the grid, centred in the table.
  if (i < bz->n_prefix || j < bz->n_prefix) return 0.0f;
  const int64_t ti = i - bz->n_prefix, tj = j - bz->n_prefix;
  const int64_t yi = ti / bz->grid_w, xi = ti % bz->grid_w;
  const int64_t yj = tj / bz->grid_w, xj = tj % bz->grid_w;
  const int64_t row = yi - yj + (bz->table_h - 1);
  const int64_t col = xi - xj + (bz->table_w - 1);
  const int64_t tsize = static_cast<int64_t>(2 * bz->table_h - 1) * (2 * bz->table_w - 1);
  (void)H;
  return bz->data[h * tsize + row * (2 * bz->table_w - 1) + col];
}

// Writes the bias as a dense [H][N][N] tensor for batch 0, so a test can compare the
// relative-position gather with a dense tensor built independently.
void bao_bias_materialize(const bao_bias* bz, int64_t H, int64_t N, float* out) {
  for (int64_t h = 0; h < H; ++h)
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j) out[(h * N + i) * N + j] = bias_value(bz, 0, h, N, H, i, j);
}

// Arguments of the forward pass. Inputs are fp32 host arrays holding the exact values
// of the fp16/bf16 tensors, layout [B][H][N][d].
struct bao_fwd_args {
  int64_t B, H, N;
  int d;
  const float* q;
  const float* k;
  const float* v;
  bao_bias bias;
  float softmax_scale;  // <= 0 selects 1/sqrt(d)
  int block_c;          // key block of the online softmax (the tiling the P codes depend on)
  int rowsum_mode;      // 0: l from fp32 P~ (default); 1: l = sum P_u8 / 255 (alternative reading)
  int num_threads;      // OpenMP threads over rows (<= 0: all)
  int64_t n_rows;       // number of query rows computed per (b,h); rows == nullptr -> all N
  const int64_t* rows;  // query row indices, the same for every (b,h)
};

// Optional per-row diagnostics (any pointer may be null). Row r = ((b*H+h)*n_rows + r').
struct bao_fwd_debug {
  float* m_final;    // [rows] final running max
  double* l_final;   // [rows] final normaliser
  float* p_float;    // [rows][N] P~ = exp(s - m_t) of each key, against its block's running max
  uint8_t* p_u8;     // [rows][N] the 8-bit code of each key
  float* s_logit;    // [rows][N] s_ij = alpha*x_ij + b_ij (fp32)
};

// Steps 3-8 — the forward pass for one query row (b, h, i).
// [zh] §2.3 and [it] §2C: the kernel keeps FlashAttention-2's tiling, so the softmax
// is the online (blockwise) form: for each key block t in ascending order,
//   m_t = max(m_{t-1}, max_j s_ij),   c_t = exp(m_{t-1} - m_t)   (c_0 = 0),
//   P~_ij = exp(s_ij - m_t),          l_t = l_{t-1}*c_t + sum_j P~_ij,
//   P_ij  = rne(255 * P~_ij)          ([zh] §2.2(3): unsigned 8-bit on [0,1]),
//   acc   = sum_j P_ij * vq_jc        (integer; the u8 x s8 -> s32 instruction named on every page),
//   O~_c  = O~_c * c_t + acc_c.
// Output O_ic = O~_c * (sv_c / 255) / l.
// Logit: s_ij = fmaf(alpha, x_ij, b_ij) with alpha = (scale*mu_q)*mu_k in fp32.
// Readings: the bias is added after scaling and is not scaled; the normaliser l is the
// softmax sum of the unquantised P~ (rows of P~/l sum to 1 before quantisation); P is
// quantised against the running max of its block, so the result depends on block_c
// and the ascending order, both fixed by the caller.
static void forward_row(const bao_fwd_args* a, const uint32_t* bq, const uint32_t* bk,
                        const int8_t* vq, const float* sv, float alpha, int64_t b, int64_t h,
                        int64_t i, float* o_row, const bao_fwd_debug* dbg, int64_t dbg_row) {
  const int64_t N = a->N, H = a->H;
  const int d = a->d;
  const int64_t bh = b * H + h;
  const int Bc = a->block_c;

  float m = -std::numeric_limits<float>::infinity();
  double l = 0.0;
  std::vector<double> acc_o(d, 0.0);
  std::vector<float> s(Bc);
  std::vector<int64_t> acc(d);

  for (int64_t t0 = 0; t0 < N; t0 += Bc) {
    const int64_t t1 = (t0 + Bc < N) ? (t0 + Bc) : N;
    // logits of the block
    float mt = m;
    for (int64_t j = t0; j < t1; ++j) {
      int diff = 0;
      for (int k = 0; k < kWordsPerRow; ++k)
        diff += popcount32(bq[(bh * N + i) * kWordsPerRow + k] ^ bk[(bh * N + j) * kWordsPerRow + k]);
      const int x = d - 2 * diff;
      const float bias = bias_value(&a->bias, b, h, N, H, i, j);
      const float sj = std::fma(alpha, static_cast<float>(x), bias);
      s[j - t0] = sj;
      if (sj > mt) mt = sj;
      if (dbg && dbg->s_logit) dbg->s_logit[dbg_row * N + j] = sj;
    }
    // rescale factor of the previous state
    const double c = (m == -std::numeric_limits<float>::infinity())
                         ? 0.0
                         : std::exp(static_cast<double>(m) - static_cast<double>(mt));
    double lt = 0.0;
    for (int c2 = 0; c2 < d; ++c2) acc[c2] = 0;
    for (int64_t j = t0; j < t1; ++j) {
      const float p = static_cast<float>(std::exp(static_cast<double>(s[j - t0]) - static_cast<double>(mt)));
      float code = std::nearbyint(255.0f * p);
      if (code > 255.0f) code = 255.0f;
      if (code < 0.0f) code = 0.0f;
      const int pu8 = static_cast<int>(code);
      lt += (a->rowsum_mode == 0) ? static_cast<double>(p) : static_cast<double>(pu8) / 255.0;
      for (int c2 = 0; c2 < d; ++c2) acc[c2] += static_cast<int64_t>(pu8) * vq[(bh * N + j) * d + c2];
      if (dbg && dbg->p_float) dbg->p_float[dbg_row * N + j] = p;
      if (dbg && dbg->p_u8) dbg->p_u8[dbg_row * N + j] = static_cast<uint8_t>(pu8);
    }
    l = l * c + lt;
    for (int c2 = 0; c2 < d; ++c2) acc_o[c2] = acc_o[c2] * c + static_cast<double>(acc[c2]);
    m = mt;
  }
  for (int c2 = 0; c2 < d; ++c2) {
    const double scale_c = static_cast<double>(sv[bh * d + c2]) / 255.0;
    o_row[c2] = (N > 0) ? static_cast<float>(acc_o[c2] * scale_c / l) : 0.0f;
  }
  if (dbg && dbg->m_final) dbg->m_final[dbg_row] = m;
  if (dbg && dbg->l_final) dbg->l_final[dbg_row] = l;
}

// The whole forward pass. o: [B][H][n_rows][d] fp32 (n_rows = N when rows is null).
// Returns 0 on success, nonzero on an argument it does not support.
int bao_attention_fwd(const bao_fwd_args* a, float* o, const bao_fwd_debug* dbg) {
  if (a->d < 1 || a->d > 128 || a->block_c < 1 || a->N < 0 || a->B < 0 || a->H < 0) return 1;
  const int64_t B = a->B, H = a->H, N = a->N, BH = B * H;
  const int d = a->d;
  const int64_t nr = (a->rows != nullptr) ? a->n_rows : N;
  if (BH == 0 || N == 0) return 0;

  std::vector<float> scratch_mu_q(BH), scratch_mu_k(BH);
  std::vector<uint32_t> bq(BH * N * kWordsPerRow), bk(BH * N * kWordsPerRow);
  std::vector<int8_t> vq(BH * N * d);
  std::vector<float> sv(BH * d);
  bao_pack_signs(a->q, BH * N, d, bq.data());
  bao_pack_signs(a->k, BH * N, d, bk.data());
  bao_mu(a->q, BH, N, d, scratch_mu_q.data());
  bao_mu(a->k, BH, N, d, scratch_mu_k.data());
  bao_quant_v(a->v, BH, N, d, vq.data(), sv.data());

  const float scale = (a->softmax_scale > 0.0f) ? a->softmax_scale
                                                : 1.0f / std::sqrt(static_cast<float>(d));
  const int64_t total = BH * nr;
#ifdef _OPENMP
  const int nt = (a->num_threads > 0) ? a->num_threads : omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 4) num_threads(nt)
#endif
  for (int64_t r = 0; r < total; ++r) {
    const int64_t bh = r / nr, rr = r % nr;
    const int64_t b = bh / H, h = bh % H;
    const int64_t i = (a->rows != nullptr) ? a->rows[rr] : rr;
    const float alpha = (scale * scratch_mu_q[bh]) * scratch_mu_k[bh];
    forward_row(a, bq.data(), bk.data(), vq.data(), sv.data(), alpha, b, h, i, o + r * d, dbg, r);
  }
  return 0;
}

// A second, separately written definition for the single-block case: the softmax of
// the whole row at once (true row max), P quantised against that max, one integer
// P.V. With block_c >= N the blockwise pass above must give exactly this.
int bao_attention_twopass(const bao_fwd_args* a, float* o) {
  if (a->d < 1 || a->d > 128 || a->N < 0) return 1;
  const int64_t B = a->B, H = a->H, N = a->N, BH = B * H;
  const int d = a->d;
  if (BH == 0 || N == 0) return 0;
  std::vector<uint32_t> bq(BH * N * kWordsPerRow), bk(BH * N * kWordsPerRow);
  std::vector<int8_t> vq(BH * N * d);
  std::vector<float> sv(BH * d), muq(BH), muk(BH);
  bao_pack_signs(a->q, BH * N, d, bq.data());
  bao_pack_signs(a->k, BH * N, d, bk.data());
  bao_mu(a->q, BH, N, d, muq.data());
  bao_mu(a->k, BH, N, d, muk.data());
  bao_quant_v(a->v, BH, N, d, vq.data(), sv.data());
  std::vector<int32_t> x(N * N);
  const float scale = (a->softmax_scale > 0.0f) ? a->softmax_scale
                                                : 1.0f / std::sqrt(static_cast<float>(d));
  for (int64_t bh = 0; bh < BH; ++bh) {
    const int64_t b = bh / H, h = bh % H;
    bao_logits(bq.data() + bh * N * kWordsPerRow, bk.data() + bh * N * kWordsPerRow, 1, N, d, x.data());
    const float alpha = (scale * muq[bh]) * muk[bh];
    for (int64_t i = 0; i < N; ++i) {
      std::vector<float> s(N);
      float m = -std::numeric_limits<float>::infinity();
      for (int64_t j = 0; j < N; ++j) {
        s[j] = std::fma(alpha, static_cast<float>(x[i * N + j]), bias_value(&a->bias, b, h, N, H, i, j));
        if (s[j] > m) m = s[j];
      }
      double l = 0.0;
      std::vector<int64_t> acc(d, 0);
      for (int64_t j = 0; j < N; ++j) {
        const float p = static_cast<float>(std::exp(static_cast<double>(s[j]) - static_cast<double>(m)));
        l += static_cast<double>(p);
        float code = std::nearbyint(255.0f * p);
        code = code > 255.0f ? 255.0f : (code < 0.0f ? 0.0f : code);
        for (int c = 0; c < d; ++c) acc[c] += static_cast<int64_t>(code) * vq[(bh * N + j) * d + c];
      }
      for (int c = 0; c < d; ++c)
        o[(bh * N + i) * d + c] =
            static_cast<float>(static_cast<double>(acc[c]) * (static_cast<double>(sv[bh * d + c]) / 255.0) / l);
    }
  }
  return 0;
}

// Full-precision attention in double on the original q, k, v (no binarisation, no
// quantisation): softmax(scale * q.k + b) v. Only a loose sanity reference.
int bao_attention_fullprec(const bao_fwd_args* a, float* o) {
  const int64_t B = a->B, H = a->H, N = a->N, BH = B * H;
  const int d = a->d;
  const double scale = (a->softmax_scale > 0.0f) ? a->softmax_scale : 1.0 / std::sqrt(static_cast<double>(d));
  std::vector<double> s(N);
  for (int64_t bh = 0; bh < BH; ++bh) {
    const int64_t b = bh / H, h = bh % H;
    for (int64_t i = 0; i < N; ++i) {
      double m = -std::numeric_limits<double>::infinity();
      for (int64_t j = 0; j < N; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
          dot += static_cast<double>(a->q[(bh * N + i) * d + c]) * static_cast<double>(a->k[(bh * N + j) * d + c]);
        s[j] = scale * dot + static_cast<double>(bias_value(&a->bias, b, h, N, H, i, j));
        if (s[j] > m) m = s[j];
      }
      double l = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        s[j] = std::exp(s[j] - m);
        l += s[j];
      }
      for (int c = 0; c < d; ++c) {
        double accv = 0.0;
        for (int64_t j = 0; j < N; ++j) accv += s[j] * static_cast<double>(a->v[(bh * N + j) * d + c]);
        o[(bh * N + i) * d + c] = static_cast<float>(accv / l);
      }
    }
  }
  return 0;
}

}  // extern "C"
