// C-ABI layer of libbinattn: argument validation, workspace layout and launches.
// The entry points are declared and documented in include/binattn.h.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <vector>

#include "binattn.h"
#include "common.cuh"
#include "kernels.h"

using namespace binattn;

namespace {

thread_local int tl_last_cuda_error = 0;
thread_local int tl_last_impl = 0;
std::atomic<int> g_impl{0};

// Stage timing (measurement only): per call, kStages + 1 events recorded on the call's stream.
constexpr int kStages = 4;
struct StageTimer {
  std::mutex mu;
  bool enabled = false;
  std::vector<cudaEvent_t> pool;                      // free events
  std::vector<std::vector<cudaEvent_t>> recorded;     // one vector of kStages + 1 per call
};
StageTimer& timer() {
  static StageTimer t;
  return t;
}

// Events for one call, or an empty vector when timing is off.
std::vector<cudaEvent_t> timing_events() {
  StageTimer& t = timer();
  std::lock_guard<std::mutex> lk(t.mu);
  std::vector<cudaEvent_t> ev;
  if (!t.enabled) return ev;
  for (int k = 0; k <= kStages; ++k) {
    cudaEvent_t e = nullptr;
    if (!t.pool.empty()) {
      e = t.pool.back();
      t.pool.pop_back();
    } else if (cudaEventCreate(&e) != cudaSuccess) {
      for (cudaEvent_t x : ev) t.pool.push_back(x);
      return {};
    }
    ev.push_back(e);
  }
  return ev;
}

void record(const std::vector<cudaEvent_t>& ev, int k, cudaStream_t s) {
  if (!ev.empty()) cudaEventRecord(ev[k], s);
}

void keep(std::vector<cudaEvent_t>& ev, bool ok) {
  if (ev.empty()) return;
  StageTimer& t = timer();
  std::lock_guard<std::mutex> lk(t.mu);
  if (ok) {
    t.recorded.push_back(ev);
  } else {
    for (cudaEvent_t x : ev) t.pool.push_back(x);
  }
}

constexpr int64_t kMaxBH = 65536;
constexpr int64_t kMaxN = 1 << 20;

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ba_status check_dims(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0) return BA_ERR_INVALID_ARG;
  if (d < 1 || d > 128) return BA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H > kMaxBH || N > kMaxN) return BA_ERR_UNSUPPORTED;
  return BA_OK;
}

bool empty(int B, int H, int N) { return B == 0 || H == 0 || N == 0; }

PrepDims dims(int B, int H, int N, int d) {
  PrepDims g;
  g.BH = static_cast<int64_t>(B) * H;
  g.N = N;
  g.d = d;
  g.dp = v_row_bytes(d);
  g.nchunk = static_cast<int>(ceil_div(N, kPrepTokens));
  return g;
}

// Workspace regions (byte offsets, each 256-byte aligned).
struct WsLayout {
  size_t bits_q = 0, bits_k = 0, mu_q = 0, mu_k = 0, vq = 0, v_scale = 0;
  size_t part_mu_q = 0, part_mu_k = 0, part_amax = 0, total = 0;
};

enum { kWsPack = 1, kWsQuant = 2, kWsAll = 3 };

WsLayout layout(int B, int H, int N, int d, int what) {
  WsLayout L;
  if (empty(B, H, N)) return L;
  const PrepDims g = dims(B, H, N, d);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  if (what == kWsAll) {
    L.bits_q = take(static_cast<size_t>(g.BH) * N * 16);
    L.bits_k = take(static_cast<size_t>(g.BH) * N * 16);
    L.mu_q = take(static_cast<size_t>(g.BH) * 4);
    L.mu_k = take(static_cast<size_t>(g.BH) * 4);
    L.vq = take(static_cast<size_t>(g.BH) * N * g.dp);
    L.v_scale = take(static_cast<size_t>(g.BH) * d * 4);
  }
  if (what & kWsPack) {
    L.part_mu_q = take(static_cast<size_t>(g.BH) * g.nchunk * 8);
    if (what == kWsAll) L.part_mu_k = take(static_cast<size_t>(g.BH) * g.nchunk * 8);
  }
  if (what & kWsQuant) {
    L.part_amax = take(static_cast<size_t>(g.BH) * amax_parts(g) * g.dp * 4);
  }
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off);
}

ba_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return BA_OK;
  tl_last_cuda_error = static_cast<int>(e);
  return BA_ERR_CUDA;
}

ba_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return BA_OK;
  if (ws == nullptr || ws_bytes < need) return BA_ERR_WORKSPACE;
  if (!aligned16(ws)) return BA_ERR_ALIGNMENT;
  return BA_OK;
}

ba_status check_bias(const ba_bias* bz, int N, BiasParams* out) {
  BiasParams bp{};
  bp.kind = BA_BIAS_NONE;
  if (bz != nullptr && bz->kind != BA_BIAS_NONE) {
    if (bz->kind != BA_BIAS_DENSE && bz->kind != BA_BIAS_RELPOS2D) return BA_ERR_INVALID_ARG;
    if (bz->data == nullptr) return BA_ERR_INVALID_ARG;
    if (!aligned16(bz->data)) return BA_ERR_ALIGNMENT;
    bp.kind = bz->kind;
    bp.data = bz->data;
    if (bz->kind == BA_BIAS_DENSE) {
      if (bz->batch_stride < 0) return BA_ERR_INVALID_ARG;
      bp.batch_stride = bz->batch_stride;
    } else {
      if (bz->n_prefix < 0 || bz->grid_h < 1 || bz->grid_w < 1) return BA_ERR_INVALID_ARG;
      if (static_cast<int64_t>(bz->grid_h) * bz->grid_w != static_cast<int64_t>(N) - bz->n_prefix)
        return BA_ERR_INVALID_ARG;
      if (bz->table_h < bz->grid_h || bz->table_w < bz->grid_w) return BA_ERR_INVALID_ARG;
      if (static_cast<int64_t>(2 * bz->table_h - 1) * (2 * bz->table_w - 1) > (int64_t{1} << 31))
        return BA_ERR_UNSUPPORTED;
      bp.grid_h = bz->grid_h;
      bp.grid_w = bz->grid_w;
      bp.table_h = bz->table_h;
      bp.table_w = bz->table_w;
      bp.n_prefix = bz->n_prefix;
    }
  }
  *out = bp;
  return BA_OK;
}

ba_status run_pack(const void* x, int dt, const PrepDims& g, uint32_t* bits, float* mu, double* part,
                   cudaStream_t s) {
  PrepParams pp{};
  pp.g = g;
  pp.job[0] = PrepJob{x, kJobPack, bits, part, nullptr};
  pp.job[1] = pp.job[2] = pp.job[0];
  ba_status st = cuda_status(launch_prep(pp, dt, 1, s));
  if (st != BA_OK) return st;
  FinalizeParams fp{};
  fp.g = g;
  fp.npack = 1;
  fp.part_mu[0] = part;
  fp.mu[0] = mu;
  return cuda_status(launch_finalize(fp, s));
}

ba_status validate_packed(const uint32_t* bits_q, const float* mu_q, const uint32_t* bits_k,
                          const float* mu_k, const int8_t* vq, const float* v_scale, void* o,
                          ba_dtype o_dt, int32_t* dbg) {
  if (!bits_q || !mu_q || !bits_k || !mu_k || !vq || !v_scale || !o) return BA_ERR_INVALID_ARG;
  if (o_dt != BA_F16 && o_dt != BA_BF16 && o_dt != BA_F32) return BA_ERR_INVALID_ARG;
  for (const void* p : {static_cast<const void*>(bits_q), static_cast<const void*>(mu_q),
                        static_cast<const void*>(bits_k), static_cast<const void*>(mu_k),
                        static_cast<const void*>(vq), static_cast<const void*>(v_scale),
                        static_cast<const void*>(o), static_cast<const void*>(dbg)})
    if (!aligned16(p)) return BA_ERR_ALIGNMENT;
  return BA_OK;
}

ba_status run_attention(const AttnParams& ap, cudaStream_t s) {
  const int impl = g_impl.load();
  const bool tc_ok = attn_tc_supported(ap);
  if (impl == 2 && !tc_ok) return BA_ERR_UNSUPPORTED;
  const bool use_tc = (impl == 2) || (impl == 0 && tc_ok);
  const ba_status st = cuda_status(use_tc ? launch_attn_tc(ap, s) : launch_attn_simt(ap, s));
  if (st == BA_OK) tl_last_impl = use_tc ? 2 : 1;
  return st;
}

}  // namespace

extern "C" {

int ba_sign_words(int d) { return (d >= 1 && d <= 128) ? kSignWords : 0; }

int ba_v_row_bytes(int d) { return (d >= 1 && d <= 128) ? v_row_bytes(d) : 0; }

int ba_kv_block(void) { return kKvBlock; }

double ba_p_code_threshold(int k) { return p_code_threshold(k); }

int ba_prep_fused(int B, int H, int N, int d) {
  if (check_dims(B, H, N, d) != BA_OK || empty(B, H, N)) return 0;
  return use_slice_prep(dims(B, H, N, d)) ? 1 : 0;
}

size_t ba_pack_workspace_bytes(int B, int H, int N, int d) {
  if (check_dims(B, H, N, d) != BA_OK) return static_cast<size_t>(-1);
  return layout(B, H, N, d, kWsPack).total;
}

size_t ba_quant_workspace_bytes(int B, int H, int N, int d) {
  if (check_dims(B, H, N, d) != BA_OK) return static_cast<size_t>(-1);
  return layout(B, H, N, d, kWsQuant).total;
}

size_t ba_workspace_bytes(int B, int H, int N, int d) {
  if (check_dims(B, H, N, d) != BA_OK) return static_cast<size_t>(-1);
  return layout(B, H, N, d, kWsAll).total;
}

ba_status ba_pack_signs(const void* x, ba_dtype dt, int B, int H, int N, int d, uint32_t* bits,
                        float* mu, void* ws, size_t ws_bytes, void* stream) {
  ba_status st = check_dims(B, H, N, d);
  if (st != BA_OK) return st;
  if (dt != BA_F16 && dt != BA_BF16) return BA_ERR_INVALID_ARG;
  if (empty(B, H, N)) return BA_OK;
  if (!x || !bits || !mu) return BA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(bits) || !aligned16(mu)) return BA_ERR_ALIGNMENT;
  const WsLayout L = layout(B, H, N, d, kWsPack);
  if ((st = check_ws(ws, ws_bytes, L.total)) != BA_OK) return st;
  return run_pack(x, dt, dims(B, H, N, d), bits, mu, at<double>(ws, L.part_mu_q),
                  static_cast<cudaStream_t>(stream));
}

ba_status ba_quant_v(const void* v, ba_dtype dt, int B, int H, int N, int d, int8_t* vq,
                     float* v_scale, void* ws, size_t ws_bytes, void* stream) {
  ba_status st = check_dims(B, H, N, d);
  if (st != BA_OK) return st;
  if (dt != BA_F16 && dt != BA_BF16) return BA_ERR_INVALID_ARG;
  if (empty(B, H, N)) return BA_OK;
  if (!v || !vq || !v_scale) return BA_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(vq) || !aligned16(v_scale)) return BA_ERR_ALIGNMENT;
  const WsLayout L = layout(B, H, N, d, kWsQuant);
  if ((st = check_ws(ws, ws_bytes, L.total)) != BA_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const PrepDims g = dims(B, H, N, d);
  PrepParams pp{};
  pp.g = g;
  pp.job[0] = PrepJob{v, kJobAmax, nullptr, nullptr, at<float>(ws, L.part_amax)};
  pp.job[1] = pp.job[2] = pp.job[0];
  if ((st = cuda_status(launch_prep(pp, dt, 1, s))) != BA_OK) return st;
  QuantParams qp{};
  qp.g = g;
  qp.v = v;
  qp.part_amax = at<float>(ws, L.part_amax);
  qp.npart = amax_parts(g);
  qp.v_scale = v_scale;
  qp.vq = vq;
  qp.npack = 0;
  qp.tpc = quant_tokens_per_cta(g);
  return cuda_status(launch_quant(qp, dt, s));
}

ba_status ba_attention_fwd_packed(const uint32_t* bits_q, const float* mu_q, const uint32_t* bits_k,
                                  const float* mu_k, const int8_t* vq, const float* v_scale, int B,
                                  int H, int N, int d, const ba_bias* bias, float softmax_scale,
                                  void* o, ba_dtype o_dt, int32_t* dbg_logits, void* stream) {
  ba_status st = check_dims(B, H, N, d);
  if (st != BA_OK) return st;
  if (!std::isfinite(softmax_scale)) return BA_ERR_INVALID_ARG;
  if (empty(B, H, N)) return BA_OK;
  if ((st = validate_packed(bits_q, mu_q, bits_k, mu_k, vq, v_scale, o, o_dt, dbg_logits)) != BA_OK)
    return st;
  AttnParams ap{};
  if ((st = check_bias(bias, N, &ap.bias)) != BA_OK) return st;
  ap.bits_q = bits_q;
  ap.bits_k = bits_k;
  ap.mu_q = mu_q;
  ap.mu_k = mu_k;
  ap.vq = vq;
  ap.v_scale = v_scale;
  ap.B = B;
  ap.H = H;
  ap.N = N;
  ap.d = d;
  ap.dp = v_row_bytes(d);
  ap.softmax_scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  ap.o = o;
  ap.o_dt = o_dt;
  ap.dbg_logits = dbg_logits;
  return run_attention(ap, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

ba_status forward(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H, int N, int d,
                  const ba_bias* bias, float softmax_scale, void* o, ba_dtype o_dt, void* ws, size_t ws_bytes,
                  int32_t* dbg_logits, uint8_t* dbg_p, int p_check_all, void* stream) {
  ba_status st = check_dims(B, H, N, d);
  if (st != BA_OK) return st;
  if (dt != BA_F16 && dt != BA_BF16) return BA_ERR_INVALID_ARG;
  if (o_dt != BA_F16 && o_dt != BA_BF16 && o_dt != BA_F32) return BA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return BA_ERR_INVALID_ARG;
  if (empty(B, H, N)) return BA_OK;
  if (!q || !k || !v || !o) return BA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dbg_logits))
    return BA_ERR_ALIGNMENT;
  BiasParams bp;
  if ((st = check_bias(bias, N, &bp)) != BA_OK) return st;
  const WsLayout L = layout(B, H, N, d, kWsAll);
  if ((st = check_ws(ws, ws_bytes, L.total)) != BA_OK) return st;

  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const PrepDims g = dims(B, H, N, d);
  std::vector<cudaEvent_t> ev = timing_events();
  record(ev, 0, s);
  if (use_slice_prep(g)) {
    // Many slices of whole 16-byte rows: one launch prepares q, k and v slice by slice (the
    // finalize and quantise stages are empty).
    SliceParams sp{};
    sp.g = g;
    sp.q = q;
    sp.k = k;
    sp.v = v;
    sp.bits_q = at<uint32_t>(ws, L.bits_q);
    sp.bits_k = at<uint32_t>(ws, L.bits_k);
    sp.mu_q = at<float>(ws, L.mu_q);
    sp.mu_k = at<float>(ws, L.mu_k);
    sp.vq = at<int8_t>(ws, L.vq);
    sp.v_scale = at<float>(ws, L.v_scale);
    if ((st = cuda_status(launch_prep_slices(sp, dt, s))) != BA_OK) return keep(ev, false), st;
    record(ev, 1, s);
    record(ev, 2, s);
    record(ev, 3, s);
  } else {
    // One launch streams q, k and v: sign bits + |x| partial sums for q and k, partial channel
    // maxima for v.
    PrepParams pp{};
    pp.g = g;
    pp.job[0] = PrepJob{q, kJobPack, at<uint32_t>(ws, L.bits_q), at<double>(ws, L.part_mu_q), nullptr};
    pp.job[1] = PrepJob{k, kJobPack, at<uint32_t>(ws, L.bits_k), at<double>(ws, L.part_mu_k), nullptr};
    pp.job[2] = PrepJob{v, kJobAmax, nullptr, nullptr, at<float>(ws, L.part_amax)};
    if ((st = cuda_status(launch_prep(pp, dt, 3, s))) != BA_OK) return keep(ev, false), st;
    record(ev, 1, s);
    record(ev, 2, s);  // the finalize is folded into the quantiser
    // The quantiser reduces the V partials to scales and writes int8 V and mu of q and k.
    QuantParams qp{};
    qp.g = g;
    qp.v = v;
    qp.part_amax = at<float>(ws, L.part_amax);
    qp.npart = amax_parts(g);
    qp.v_scale = at<float>(ws, L.v_scale);
    qp.vq = at<int8_t>(ws, L.vq);
    qp.npack = 2;
    qp.tpc = quant_tokens_per_cta(g);
    qp.part_mu[0] = at<double>(ws, L.part_mu_q);
    qp.part_mu[1] = at<double>(ws, L.part_mu_k);
    qp.mu[0] = at<float>(ws, L.mu_q);
    qp.mu[1] = at<float>(ws, L.mu_k);
    if ((st = cuda_status(launch_quant(qp, dt, s))) != BA_OK) return keep(ev, false), st;
    record(ev, 3, s);
  }

  AttnParams ap{};
  ap.bias = bp;
  ap.bits_q = at<uint32_t>(ws, L.bits_q);
  ap.bits_k = at<uint32_t>(ws, L.bits_k);
  ap.mu_q = at<float>(ws, L.mu_q);
  ap.mu_k = at<float>(ws, L.mu_k);
  ap.vq = at<int8_t>(ws, L.vq);
  ap.v_scale = at<float>(ws, L.v_scale);
  ap.B = B;
  ap.H = H;
  ap.N = N;
  ap.d = d;
  ap.dp = g.dp;
  ap.softmax_scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  ap.o = o;
  ap.o_dt = o_dt;
  ap.dbg_logits = dbg_logits;
  ap.dbg_p = dbg_p;
  ap.p_check_all = p_check_all;
  st = run_attention(ap, s);
  record(ev, 4, s);
  keep(ev, st == BA_OK);
  return st;
}

}  // namespace

extern "C" {

ba_status ba_attention_fwd(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H,
                           int N, int d, const ba_bias* bias, float softmax_scale, void* o,
                           ba_dtype o_dt, void* ws, size_t ws_bytes, int32_t* dbg_logits,
                           void* stream) {
  return forward(q, k, v, dt, B, H, N, d, bias, softmax_scale, o, o_dt, ws, ws_bytes, dbg_logits, nullptr, 0,
                 stream);
}

ba_status ba_attention_fwd_debug(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H,
                                 int N, int d, const ba_bias* bias, float softmax_scale, void* o,
                                 ba_dtype o_dt, void* ws, size_t ws_bytes, int32_t* dbg_logits,
                                 uint8_t* dbg_p, int check_all_codes, void* stream) {
  if (check_all_codes != 0 && check_all_codes != 1) return BA_ERR_INVALID_ARG;
  if (!aligned16(dbg_p)) return BA_ERR_ALIGNMENT;
  return forward(q, k, v, dt, B, H, N, d, bias, softmax_scale, o, o_dt, ws, ws_bytes, dbg_logits, dbg_p,
                 check_all_codes, stream);
}

ba_status ba_stage_timing(int enable) {
  StageTimer& t = timer();
  std::lock_guard<std::mutex> lk(t.mu);
  t.enabled = enable != 0;
  return BA_OK;
}

ba_status ba_stage_times(float* ms, int n, int* calls) {
  if (ms == nullptr || calls == nullptr || n < 0 || n > kStages) return BA_ERR_INVALID_ARG;
  StageTimer& t = timer();
  std::lock_guard<std::mutex> lk(t.mu);
  double acc[kStages] = {0, 0, 0, 0};
  ba_status st = BA_OK;
  for (auto& ev : t.recorded) {
    for (int k = 0; k < kStages && st == BA_OK; ++k) {
      float e = 0.0f;
      cudaError_t err = cudaEventSynchronize(ev[k + 1]);
      if (err == cudaSuccess) err = cudaEventElapsedTime(&e, ev[k], ev[k + 1]);
      if (err != cudaSuccess) st = cuda_status(err);
      acc[k] += e;
    }
    for (cudaEvent_t x : ev) t.pool.push_back(x);
  }
  *calls = static_cast<int>(t.recorded.size());
  t.recorded.clear();
  for (int k = 0; k < n; ++k) ms[k] = static_cast<float>(acc[k]);
  return st;
}

ba_status ba_set_attention_impl(int impl) {
  if (impl < 0 || impl > 2) return BA_ERR_INVALID_ARG;
  g_impl.store(impl);
  return BA_OK;
}

int ba_get_attention_impl(void) { return g_impl.load(); }

int ba_last_attention_impl(void) { return tl_last_impl; }

ba_status ba_check_device_status(void* stream) {
  int v = 0;
  const ba_status st = cuda_status(read_and_clear_device_status(&v, static_cast<cudaStream_t>(stream)));
  if (st != BA_OK) return st;
  return v != 0 ? BA_ERR_TIMEOUT : BA_OK;
}

const char* ba_status_string(ba_status s) {
  switch (s) {
    case BA_OK: return "BA_OK";
    case BA_ERR_INVALID_ARG: return "BA_ERR_INVALID_ARG: invalid argument";
    case BA_ERR_UNSUPPORTED: return "BA_ERR_UNSUPPORTED: unsupported size";
    case BA_ERR_ALIGNMENT: return "BA_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case BA_ERR_WORKSPACE: return "BA_ERR_WORKSPACE: workspace missing or too small";
    case BA_ERR_CUDA: return "BA_ERR_CUDA: CUDA error";
    case BA_ERR_TIMEOUT: return "BA_ERR_TIMEOUT: a bounded device wait expired";
  }
  return "unknown status";
}

int ba_last_cuda_error(void) { return tl_last_cuda_error; }

}  // extern "C"
