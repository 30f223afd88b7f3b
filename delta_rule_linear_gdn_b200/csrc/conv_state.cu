// Conv history after a chunked prefill.
//
// The depthwise causal conv of kernel 4 ("Gated DeltaNet: o mixer em 48 das 64
// camadas", Conceito) reads the three inputs before each token. A prefill
// that continues an earlier one (or is followed by decode steps) needs those
// three inputs of the earlier call: this kernel writes them, per sequence and
// channel of q | k | v, as rows j = 0, 1, 2 holding the input of the
// sequence's token T − 3 + j (oldest first; T its length, also for sequences
// packed along one row). Rows before token 0 come from the incoming history
// (or are zero without one), which makes the chain of calls equal to one call
// over the concatenated tokens. The rows are copied bit for bit, in the input
// dtype.

#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kCsThreads = 256;

template <typename TIn>
__global__ void __launch_bounds__(kCsThreads) conv_state_kernel(ChunkArgs a) {
  const int D = a.dk;
  const size_t nq = (size_t)a.Hqk * D;                  // channels of q (= of k)
  const size_t ctot = 2 * nq + (size_t)a.Hv * a.dv;     // channels of q | k | v
  const size_t idx = (size_t)blockIdx.x * kCsThreads + threadIdx.x;
  if (idx >= (size_t)a.B * ctot) return;
  const int bi = (int)(idx / ctot);
  const size_t ch = idx % ctot;
  const TIn* src;
  size_t row, cw;                                       // elements per token, channel within the tensor
  if (ch < nq) {
    src = static_cast<const TIn*>(a.q); row = nq; cw = ch;
  } else if (ch < 2 * nq) {
    src = static_cast<const TIn*>(a.k); row = nq; cw = ch - nq;
  } else {
    src = static_cast<const TIn*>(a.v); row = (size_t)a.Hv * a.dv; cw = ch - 2 * nq;
  }
  const TIn* hin = static_cast<const TIn*>(a.conv_in);
  TIn* hout = static_cast<TIn*>(a.conv_out);
  // Read all three rows before writing any (rows of one channel only).
  const size_t tok0 = seq_tok0(a, bi);   // the sequence's first token in the q, k, v buffers
  const int len = seq_len(a, bi);
  TIn r[3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int t = len - 3 + j;           // token of the sequence
    if (t >= 0) {
      r[j] = src[(tok0 + t) * row + cw];
    } else if (hin) {
      r[j] = hin[((size_t)bi * 3 + 3 + t) * ctot + ch];
    } else {
      r[j] = from_f32<TIn>(0.f);
    }
  }
#pragma unroll
  for (int j = 0; j < 3; ++j) hout[((size_t)bi * 3 + j) * ctot + ch] = r[j];
}

}  // namespace

cudaError_t launch_conv_state(const ChunkArgs& a, int qkv_bf16, cudaStream_t s) {
  if (a.conv_out == nullptr || a.B == 0) return cudaSuccess;
  const size_t ctot = 2 * (size_t)a.Hqk * a.dk + (size_t)a.Hv * a.dv;
  const size_t n = (size_t)a.B * ctot;
  const unsigned grid = (unsigned)((n + kCsThreads - 1) / kCsThreads);
  if (qkv_bf16)
    conv_state_kernel<__nv_bfloat16><<<grid, kCsThreads, 0, s>>>(a);
  else
    conv_state_kernel<float><<<grid, kCsThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace gdn2
