// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace binattn {

constexpr int kJobPack = 0;  // sign bits + sum |x| per chunk
constexpr int kJobAmax = 1;  // per-channel max |v| per group of chunks
constexpr int kQuantTokens = 1024;  // most tokens per CTA of the V quantiser

struct PrepDims {
  int64_t BH;
  int N, d, dp, nchunk;
};

struct PrepJob {
  const void* src;   // [BH][N][d] fp16/bf16
  int kind;
  uint32_t* bits;    // pack: [BH][N][4]
  double* part_sum;  // pack: [BH][nchunk] sums of |x|
  float* part;       // amax: [BH][amax_parts][dp] channel maxima
};

struct PrepParams {
  PrepJob job[3];
  PrepDims g;
};

// mu = sum |x| / (N d) per slice from the per-chunk partial sums (standalone sign packing).
struct FinalizeParams {
  PrepDims g;
  int npack;
  const double* part_mu[2];
  float* mu[2];
};

// V quantiser with the finalize folded in: each CTA reduces its slice's partial channel maxima
// (npart rows of dp floats), then writes int8 rows for tpc tokens; a slice's first CTA also
// writes the V scales and the mu of up to two packed tensors from their chunk sums.
struct QuantParams {
  PrepDims g;
  int tpc;  // tokens per CTA (quant_tokens_per_cta)
  const void* v;
  const float* part_amax;  // [BH][npart][dp]
  int npart;
  float* v_scale;  // [BH][d]
  int8_t* vq;      // [BH][N][dp]
  int npack;
  const double* part_mu[2];  // [BH][nchunk]
  float* mu[2];              // [BH]
};

// Whole-slice preparation (one warp per (b, h) and tensor; d % 8 == 0): sign bits and mu of q
// and k, channel scales and int8 rows of v, in one launch.
struct SliceParams {
  PrepDims g;
  const void* q;
  const void* k;
  const void* v;
  uint32_t* bits_q;
  uint32_t* bits_k;
  float* mu_q;
  float* mu_k;
  int8_t* vq;
  float* v_scale;
};

// Jobs [0, njobs): the sign-packing jobs first, then at most one channel-max job.
cudaError_t launch_prep(const PrepParams& p, int dt, int njobs, cudaStream_t s);
cudaError_t launch_prep_slices(const SliceParams& p, int dt, cudaStream_t s);
bool use_slice_prep(const PrepDims& g);
int amax_parts(const PrepDims& g);  // partial channel-max rows per slice written by launch_prep
cudaError_t launch_finalize(const FinalizeParams& p, cudaStream_t s);
cudaError_t launch_quant(const QuantParams& p, int dt, cudaStream_t s);
int quant_tokens_per_cta(const PrepDims& g);

// Fused attention on packed operands.
cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t s);
bool attn_tc_supported(const AttnParams& p);
double p_code_threshold(int k);  // the exact-code threshold table of the tcgen05 kernel
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s);

// Device status word of the kernels with bounded waits.
cudaError_t read_and_clear_device_status(int* value, cudaStream_t s);

}  // namespace binattn
