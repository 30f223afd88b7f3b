// The affine map of a segment of the recurrence applied to a state:
//     S_out = M · S_in + N     per (sequence, value head)
// M is d_k × d_k, S and N are d_k × d_v. Over a segment of tokens the state
// update is affine in the entry state (each token's step is S ↦ A_t S + k_t
// z_tᵀ with A_t = (I − k_t e_tᵀ) Diag(α_t): "Resumo Técnico: Gated
// DeltaNet-2", Metodologia §1), so a sequence split into segments is carried
// from one segment to the next by composing these maps ("Uma análise das
// variantes de atenção linear da família DeltaNet", "Pipeline Triton da versão
// por chunks": the state sweep is the only sequential step). fp32 throughout.
//
// One CTA per (state, block of 32 value columns): the block of S_in is read
// into shared memory first, so S_out may be S_in (in place).

#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int AF_COLS = 32;
constexpr int AF_THREADS = 256;

__global__ void __launch_bounds__(AF_THREADS) state_affine_kernel(int dk, int dv, const float* __restrict__ M,
                                                                  const float* N, const float* S_in, float* S_out) {
  __shared__ float sS[128 * AF_COLS];
  const int blocks = dv / AF_COLS;
  const int i = blockIdx.x / blocks, c0 = (blockIdx.x % blocks) * AF_COLS;
  const size_t so = (size_t)i * dk * dv, mo = (size_t)i * dk * dk;
  for (int idx = threadIdx.x; idx < dk * AF_COLS; idx += AF_THREADS) {
    const int r = idx / AF_COLS, c = idx % AF_COLS;
    sS[idx] = S_in ? S_in[so + (size_t)r * dv + c0 + c] : 0.f;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < dk * AF_COLS; idx += AF_THREADS) {
    const int r = idx / AF_COLS, c = idx % AF_COLS;
    float acc = N ? N[so + (size_t)r * dv + c0 + c] : 0.f;
    const float* mr = M + mo + (size_t)r * dk;
    for (int kk = 0; kk < dk; ++kk) acc = fmaf(__ldg(mr + kk), sS[kk * AF_COLS + c], acc);
    S_out[so + (size_t)r * dv + c0 + c] = acc;
  }
}

}  // namespace

cudaError_t launch_state_affine(int n, int dk, int dv, const float* M, const float* N, const float* S_in,
                                float* S_out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (dk > 128 || dv % AF_COLS != 0 || dv < AF_COLS) return cudaErrorInvalidValue;
  state_affine_kernel<<<n * (dv / AF_COLS), AF_THREADS, 0, s>>>(dk, dv, M, N, S_in, S_out);
  return cudaGetLastError();
}

}  // namespace gdn2
