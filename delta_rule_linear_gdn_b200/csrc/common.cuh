// Internal declarations shared by the CUDA translation units of libgdn2.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn2.h"

namespace gdn2 {

// Conversions between the I/O dtypes and fp32.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// The epsilon of the fused L2 normalisation: x · (Σx² + eps)^(−1/2).
constexpr float kL2Eps = 1e-6f;

// Gate element i of a gate tensor: the fp32 value, or σ(x) of the bf16 logit
// x when the gates are given as logits (gdn2_params.gate_logits).
// (the fast exponential and division intrinsics: a few ulp, far inside what
// the gates feed, and a handful of instructions instead of a few dozen)
__device__ __forceinline__ float sigmoid_f32(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
// log σ(x) = −log(1 + e^(−x)), written as min(x, 0) − log1p(e^(−|x|)) so that
// it stays finite for every finite x (σ(x) itself underflows to 0 below
// x ≈ −87, where log would give −∞).
__device__ __forceinline__ float log_sigmoid_f32(float x) { return fminf(x, 0.f) - log1pf(expf(-fabsf(x))); }
__device__ __forceinline__ float gate_at(const float* g, size_t i, bool logits) {
  return logits ? sigmoid_f32(__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(g)[i])) : g[i];
}
template <bool LG> __device__ __forceinline__ float gate_at(const float* g, size_t i) {
  if (LG) return sigmoid_f32(__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(g)[i]));
  return g[i];
}

// Arguments of one launch, already validated by the host entry points.
struct ChunkArgs {
  int B, T, Hqk, Hv, dk, dv, chunk;
  float scale;
  int gate_mode;
  int l2norm;
  const float* conv_w;
  const void *q, *k, *v;
  const float *alpha, *b, *w, *S0;
  void* o;
  float* ST;
  void* workspace;
  size_t ws_bytes;
  int gate_logits;   // gates are bf16 logits (σ applied in the kernels)
  // Conv history [B, 3, 2·Hqk·dk + Hv·dv] in the input dtype (NULL = zeros)
  // and the buffer that receives the history after the last token (or NULL).
  const void* conv_in;
  void* conv_out;
  int Hg;            // heads of alpha and b: Hv, or Hqk when the value heads of a QK head share them
  // Sequences of different lengths packed along T (nseq > 0): B is then
  // nseq (states and conv histories per sequence), tokens are addressed in
  // the packed stream, sequence n is [cu_tok[n], cu_tok[n+1]) and owns the
  // 64-token chunks [cu_chk[n], cu_chk[n+1]) of the tensor-core prefill.
  int nseq;
  int cu_tok[GDN2_MAX_SEQS + 1];
  int cu_chk[GDN2_MAX_SEQS + 1];
  // Failure-path test hook (gdn2_debug_set_scan_stall): > 0 makes the scan
  // wait first, for at most this many polls, on a barrier nothing signals.
  unsigned stall_polls;
};

// First token (in the q, k, v, o buffers) and length of sequence bi.
__host__ __device__ __forceinline__ size_t seq_tok0(const ChunkArgs& a, int bi) {
  return a.nseq ? (size_t)a.cu_tok[bi] : (size_t)bi * a.T;
}
__host__ __device__ __forceinline__ int seq_len(const ChunkArgs& a, int bi) {
  return a.nseq ? a.cu_tok[bi + 1] - a.cu_tok[bi] : a.T;
}

struct DecodeArgs {
  int B, Hqk, Hv, d;
  float scale;
  int gate_mode;
  int l2norm;
  const void *q, *k, *v;
  const float *alpha, *b, *w;
  float* S;
  void* o;
  int gate_logits;   // gates are bf16 logits (σ applied in the kernels)
  const float* conv_w;   // conv taps [2·Hqk·d + Hv·d, 4] or NULL (no conv)
  const void* conv_in;   // conv history before this token, or NULL (zeros)
  void* conv_out;        // history after this token, or NULL
  int Hg;                // heads of alpha and b (Hv, or Hqk when shared per QK head)
};

// Arguments of the backward pass (gdn2_chunk_bwd), validated on the host.
struct BwdArgs {
  int B, T, Hqk, Hv, Hg, gate_mode, gate_logits;
  float scale;
  const void *q, *k, *v, *dO;          // q, k, v in the input dtype; dO in the output dtype
  const float *alpha, *b, *w, *S0, *dST;
  float *dq, *dk, *dv, *dalpha, *db, *dw, *dS0;
  float* ckpt;                         // workspace: every chunk's entry state
};

// Launchers (return cudaSuccess or the launch error).
cudaError_t launch_decode(const DecodeArgs& a, int qkv_bf16, int o_bf16, cudaStream_t s);
cudaError_t launch_chunk_simt(const ChunkArgs& a, int qkv_bf16, int o_bf16, cudaStream_t s);
bool chunk_tc_supported(const ChunkArgs& a, int qkv_bf16);
// Workspace of the tensor-core path for the whole sequence at once, and the
// least it can run with (one chunk slot per sequence-head, plus the carried
// state when S_T is NULL); in between, it runs the sequence in segments.
size_t chunk_tc_workspace(const ChunkArgs& a);
size_t chunk_tc_min_workspace(const ChunkArgs& a, bool carry_state);
cudaError_t launch_chunk_tc(const ChunkArgs& a, int o_bf16, cudaStream_t s);
// Writes a.conv_out: the three pre-conv inputs that end at token T−1 of each
// sequence (history from a.conv_in shifted in when T < 3).
cudaError_t launch_conv_state(const ChunkArgs& a, int qkv_bf16, cudaStream_t s);

// S_out = M · S_in + N for n states (M [n][dk][dk]; N, S_in, S_out [n][dk][dv];
// N or S_in NULL = zeros; S_out may be S_in).
cudaError_t launch_state_affine(int n, int dk, int dv, const float* M, const float* N, const float* S_in,
                                float* S_out, cudaStream_t s);

// Backward pass: workspace bytes and launcher.
size_t chunk_bwd_workspace(int n_states, int H_v, int T, int d);
cudaError_t launch_chunk_bwd(const BwdArgs& a, int d, int qkv_bf16, int do_bf16, cudaStream_t s);

// Shape, enum and offset checks shared by the prefill entry points.
gdn2_status check_chunk_params(const gdn2_params* p);

// The polls the scan's stall hook waits (0: off).
unsigned scan_stall_polls();

// GDN2_OK or GDN2_ERR_TIMEOUT from the status word a tensor-core prefill
// keeps at the start of its scratch, after the work on `stream` so far.
gdn2_status read_device_status(const void* scratch, cudaStream_t stream);

// gdn2_chunk_fwd after argument checks; `segmented_ok` accepts a workspace
// between the minimum and the full size.
gdn2_status chunk_fwd_checked(const gdn2_params* p, const void* q, const void* k, const void* v,
                              const float* alpha, const float* b, const float* w, const float* S0, void* o,
                              float* S_T, void* workspace, size_t ws_bytes, void* stream, bool segmented_ok);

}  // namespace gdn2
