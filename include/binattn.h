/*
 * binattn.h — C ABI of the BinaryAttention forward pass for NVIDIA B200 (sm_100a).
 *
 * The method (paper "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
 * Transformers", arXiv 2603.09582; cited below through its summary pages
 * gist.science/<lang>/paper/2603.09582):
 *   s_ij = alpha * x_ij + b_ij,     x_ij = d - 2 popc(sign bits of q_i XOR sign bits of k_j),
 *   alpha = softmax_scale * mu_q * mu_k,  mu = mean |x| of the (batch, head) slice,
 *   online softmax over key blocks of ba_kv_block() keys in ascending order,
 *   P_ij = rne(255 * exp(s_ij - m_t)) as uint8 (m_t = running row max after block t),
 *   V quantised per (batch, head, channel) to int8 with scale amax/127,
 *   O = (integer P.V accumulated per block, rescaled between blocks) * v_scale / (255 l).
 *
 * Conventions shared by every entry point:
 *   - Tensors are contiguous, row-major, [B][H][N][d] unless stated otherwise.
 *   - Every pointer argument is a DEVICE pointer owned by the caller, aligned to 16 bytes.
 *     The library never allocates, frees or keeps a pointer after the call returns.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *     stream). No call synchronises the host. Calls on different streams are independent
 *     provided each uses its own workspace.
 *   - Arguments are validated before anything is launched; on an error nothing is
 *     enqueued and a status code is returned. Launch failures return BA_ERR_CUDA
 *     (ba_last_cuda_error() gives the cudaError_t).
 *   - Supported sizes: 1 <= d <= 128, 0 <= B, H, N; B*H <= 65536; N <= 1048576. Empty
 *     problems (B, H or N = 0) return BA_OK and launch nothing.
 */
#ifndef BINATTN_H
#define BINATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BA_OK = 0,
  BA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum, inconsistent bias */
  BA_ERR_UNSUPPORTED = 2,   /* d outside [1,128], sizes beyond the limits above */
  BA_ERR_ALIGNMENT = 3,     /* a pointer not aligned to 16 bytes */
  BA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
  BA_ERR_CUDA = 5,          /* a CUDA launch or runtime call failed */
  BA_ERR_TIMEOUT = 6        /* a bounded device-side wait expired (see ba_check_device_status) */
} ba_status;

typedef enum { BA_F16 = 0, BA_BF16 = 1, BA_F32 = 2 } ba_dtype;  /* F32 is accepted for O only */

typedef enum { BA_BIAS_NONE = 0, BA_BIAS_DENSE = 1, BA_BIAS_RELPOS2D = 2 } ba_bias_kind;

/*
 * The additive logit bias b_ij ("bias enhancement": gist.science/zh, technical summary
 * 2.2(2); gist.science/it, sintesi tecnica 2B — dense or position-sensitive). It is
 * added after the alpha scaling and is not scaled. Values must be finite.
 *   BA_BIAS_DENSE:    data = fp32 [H][N][N] for batch 0; batch b reads data + b*batch_stride
 *                     (batch_stride = 0 broadcasts one tensor over the batch).
 *   BA_BIAS_RELPOS2D: data = fp32 [H][(2*table_h-1)*(2*table_w-1)]. Token t >= n_prefix sits
 *                     at (y, x) = ((t-n_prefix) / grid_w, (t-n_prefix) % grid_w) with
 *                     grid_h*grid_w = N - n_prefix; b_ij = data[h][(y_i-y_j+table_h-1)*(2*table_w-1)
 *                     + (x_i-x_j+table_w-1)]; rows and columns of prefix tokens get 0.
 *                     Requires table_h >= grid_h and table_w >= grid_w.
 */
typedef struct {
  ba_bias_kind kind;
  const float* data;
  int64_t batch_stride;
  int grid_h, grid_w;
  int table_h, table_w;
  int n_prefix;
} ba_bias;

/* Words per packed sign row: 4 (128 bits, one 16-byte row) for 1 <= d <= 128, else 0. */
int ba_sign_words(int d);

/* Bytes per quantised V row: d rounded up to a multiple of 16 (pad bytes are 0). */
int ba_v_row_bytes(int d);

/* Key block of the online softmax: the 8-bit P codes depend on it (128). */
int ba_kv_block(void);

/*
 * The exact-code thresholds the tcgen05 kernel uses near a rounding tie: for 0 <= k <= 254, the
 * least double d whose code min(255, rne(fl32(255 * fl32(exp(d))))) exceeds k (the code of a
 * logit s against the running max m, with d = (double)s - (double)m; gist.science/zh 2.2(3)).
 * NaN for any other k. Host-side; computed once per process.
 */
double ba_p_code_threshold(int k);

/*
 * Preparation path ba_attention_fwd takes for this shape: 1 = one launch (one CTA per (b, h)
 * slice and tensor writes the sign bits and mu of q and k and the scales and int8 rows of v;
 * taken for many short slices with d a multiple of 8 and d >= 32), 0 = three launches
 * (128-token chunks with partial sums, a finalize kernel, the V quantiser). A host query: it
 * launches nothing and reports the choice only; both paths compute the same values.
 */
int ba_prep_fused(int B, int H, int N, int d);

/* Workspace sizes in bytes (0 for empty problems; -1 cast to size_t for unsupported d). */
size_t ba_pack_workspace_bytes(int B, int H, int N, int d);
size_t ba_quant_workspace_bytes(int B, int H, int N, int d);
size_t ba_workspace_bytes(int B, int H, int N, int d);

/*
 * Sign binarisation and the scale factor mu (gist.science/zh 2.2(1): s_i = mu_q sign(q_i),
 * mu averaging |x| over every token and channel of the (b, h) slice; gist.science/nl
 * Methodologie 2).
 *   x:    [B][H][N][d] in dt (BA_F16 or BA_BF16).
 *   bits: [B][H][N][4] uint32 out. Bit (c % 32) of word c/32 is 1 iff x_c < 0 (IEEE: -0.0,
 *         +0.0 and NaN give 0); bits at c >= d are 0.
 *   mu:   [B][H] fp32 out, mean of |x| over the N*d entries of each (b, h) slice (x must be
 *         finite: mu of a slice holding inf or NaN is unspecified).
 *   ws:   at least ba_pack_workspace_bytes(B,H,N,d) bytes of device memory (partial sums).
 */
ba_status ba_pack_signs(const void* x, ba_dtype dt, int B, int H, int N, int d, uint32_t* bits,
                        float* mu, void* ws, size_t ws_bytes, void* stream);

/*
 * Channel-aware 8-bit V (gist.science/zh 2.2(3); gist.science/nl Methodologie 2: a
 * channel-specific scale). Per (b, h, c): amax = max_j |v_jc|, inv = 127/amax (fp32),
 * q = clamp(rne(v * inv), -127, 127), v_scale = amax/127; a zero channel gives q = 0 and
 * v_scale = 0. v must be finite (the codes of a channel holding inf or NaN are unspecified).
 *   v:       [B][H][N][d] in dt (BA_F16 or BA_BF16).
 *   vq:      [B][H][N][ba_v_row_bytes(d)] int8 out, pad columns 0.
 *   v_scale: [B][H][d] fp32 out.
 *   ws:      at least ba_quant_workspace_bytes(B,H,N,d) bytes (per-chunk maxima).
 */
ba_status ba_quant_v(const void* v, ba_dtype dt, int B, int H, int N, int d, int8_t* vq,
                     float* v_scale, void* ws, size_t ws_bytes, void* stream);

/*
 * The fused forward on pre-packed operands (gist.science/zh 2.3 and gist.science/it
 * sintesi tecnica 2C: a FlashAttention-2-style tiled kernel with binary QK and an
 * unsigned-8-bit x signed-8-bit P.V accumulated in 32-bit integers).
 *   bits_q, bits_k: [B][H][N][4] from ba_pack_signs; mu_q, mu_k: [B][H].
 *   vq, v_scale:    from ba_quant_v.
 *   bias:           NULL or kind BA_BIAS_NONE for no bias.
 *   softmax_scale:  <= 0 selects 1/sqrt(d); alpha = (softmax_scale * mu_q) * mu_k in fp32.
 *   o:              [B][H][N][d] out in o_dt (BA_F16, BA_BF16 or BA_F32).
 *   dbg_logits:     NULL, or [B][H][N][N] int32 out receiving x_ij (debug; large).
 */
ba_status ba_attention_fwd_packed(const uint32_t* bits_q, const float* mu_q, const uint32_t* bits_k,
                                  const float* mu_k, const int8_t* vq, const float* v_scale, int B,
                                  int H, int N, int d, const ba_bias* bias, float softmax_scale,
                                  void* o, ba_dtype o_dt, int32_t* dbg_logits, void* stream);

/*
 * The whole forward pass: the results of ba_pack_signs(q), ba_pack_signs(k) and ba_quant_v(v)
 * into the workspace (in one launch for the shapes ba_prep_fused reports, else three), then
 * the fused step of ba_attention_fwd_packed.
 *   q, k, v: [B][H][N][d] in dt (BA_F16 or BA_BF16).
 *   ws:      at least ba_workspace_bytes(B,H,N,d) bytes; its contents on return are the
 *            packed operands (layout private to the library).
 */
ba_status ba_attention_fwd(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H,
                           int N, int d, const ba_bias* bias, float softmax_scale, void* o,
                           ba_dtype o_dt, void* ws, size_t ws_bytes, int32_t* dbg_logits,
                           void* stream);

/*
 * ba_attention_fwd with debug outputs, for tests and diagnosis (slower; not for production use).
 *   dbg_logits:      NULL, or [B][H][N][N] int32 receiving x_ij.
 *   dbg_p:           NULL, or [B][H][N][N] uint8 receiving the 8-bit code P_ij of every key, taken
 *                    against the running maximum of the key's block (the codes the P.V product
 *                    uses; gist.science/zh 2.2(3)).
 *   check_all_codes: 0 = as ba_attention_fwd: the tensor-core kernel evaluates exp with the
 *                    hardware approximation and recomputes from the double-precision exponential
 *                    every code within its error band of a rounding tie in those blocks where a
 *                    changed code could move the output by more than a tenth of the 2e-3 error
 *                    bar (rows whose softmax sum is still small); 1 = in every block, so that every
 *                    code equals the definition's.  Other values: BA_ERR_INVALID_ARG.
 *   Other arguments and errors as ba_attention_fwd (dbg_p must be 16-byte aligned).
 */
ba_status ba_attention_fwd_debug(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H,
                                 int N, int d, const ba_bias* bias, float softmax_scale, void* o,
                                 ba_dtype o_dt, void* ws, size_t ws_bytes, int32_t* dbg_logits,
                                 uint8_t* dbg_p, int check_all_codes, void* stream);

/*
 * ba_attention_fwd without a caller-supplied workspace (the paper has no counterpart; this
 * is a deployment convenience). For callers that cannot allocate device memory: a plugin that
 * is handed only its input and output buffers, or a runtime that fixes all device memory at
 * start-up and forbids cudaMalloc afterwards (it can synchronize the device and bypasses the
 * host's allocator). The workspace comes from a fixed array of BA_NOALLOC_SCRATCH_BYTES in the
 * library's device memory, held by every GPU that loads the library until the process exits.
 *   - Arguments as ba_attention_fwd, minus ws / ws_bytes.
 *   - Problems with ba_workspace_bytes(B,H,N,d) > BA_NOALLOC_SCRATCH_BYTES return
 *     BA_ERR_WORKSPACE before anything is launched.
 *   - All calls share the array: calls that can overlap on the GPU (unordered streams) race
 *     and must be ordered by the caller. Its contents persist between calls; none of it needs
 *     to start at zero.
 *   - The first call on each device looks up the array's device address (and caches it);
 *     make that first call before any stream capture. The cache assumes the device's primary
 *     context lives as long as the process (no cudaDeviceReset between calls).
 *   - Allocates nothing: no cudaMalloc, cudaFree or other allocating routine.
 */
#define BA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
ba_status ba_attention_fwd_noalloc(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H,
                                   int N, int d, const ba_bias* bias, float softmax_scale, void* o,
                                   ba_dtype o_dt, int32_t* dbg_logits, void* stream);

/*
 * Kernel choice for the fused step, process-wide: 0 = automatic (the tcgen05 tensor-core
 * kernel where it supports the shape, else the CUDA-core kernel), 1 = the CUDA-core kernel,
 * 2 = the tcgen05 kernel (BA_ERR_UNSUPPORTED for shapes it does not take).
 */
ba_status ba_set_attention_impl(int impl);
int ba_get_attention_impl(void);

/* The kernel the last successful fused call on this thread ran: 1 CUDA-core, 2 tcgen05. */
int ba_last_attention_impl(void);

/*
 * Synchronises `stream` and reads (then clears) the device status word that kernels set
 * when a bounded wait expires. Returns BA_OK or BA_ERR_TIMEOUT (or BA_ERR_CUDA).
 */
ba_status ba_check_device_status(void* stream);

/*
 * Stage timing for measurement tools (off by default). While enabled, ba_attention_fwd
 * records a CUDA event on its stream before its first kernel and after each stage: the
 * q/k/v streaming pass, the finalize pass, the V quantiser and the fused attention kernel
 * (on the one-launch preparation path the finalize and quantiser stages are empty).
 * ba_stage_times synchronises on those events and writes the device time of each of the
 * four stages in milliseconds, summed over the calls since the last read, to ms[0..n-1]
 * (n <= 4), stores the number of calls in *calls, and forgets them.
 */
ba_status ba_stage_timing(int enable);
ba_status ba_stage_times(float* ms, int n, int* calls);

/* Human-readable status; the cudaError_t behind the last BA_ERR_CUDA on this thread. */
const char* ba_status_string(ba_status s);
int ba_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BINATTN_H */
