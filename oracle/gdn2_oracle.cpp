// Float64 CPU oracle for the Gated DeltaNet-2 forward recurrence.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
// this file; only the tests, the smoke check and the bench's CPU-baseline leg
// do. It shares no code, header or constant with the CUDA library.
//
// What it computes (one independent recurrence per (sequence, value head)):
//
//   "Resumo Técnico: Gated DeltaNet-2", Metodologia, §1 "Regra Delta Portão-2":
//     e_t = b_t ⊙ k_t           (erase gate on the key axis)
//     z_t = w_t ⊙ v_t           (write gate on the value axis)
//     S_t = (I − k_t e_tᵀ) Diag(α_t) S_{t−1} + k_t z_tᵀ        (S is d_k × d_v)
//   and the readout after the write ("Uma análise das variantes de atenção
//   linear da família DeltaNet", section "Kimi Delta Attention", step 5, read
//   after write): o_t = s · S_tᵀ q_t, with s = 1 unless the caller asks for
//   another scale.
//
// The only rearrangement is associativity of the matrix product:
//   (I − k eᵀ) S̄ = S̄ − k (eᵀ S̄),  S̄ = Diag(α) S_{t−1},
// which avoids forming the d_k × d_k matrix. Every step is a plain loop in
// double precision; there is no blocking, chunking or reordering beyond that.
//
// Grouped heads ("Gated DeltaNet: o mixer em 48 das 64 camadas", Conceito:
// each QK head serves three V heads): value head h reads the query/key head
// h / (H_v / H_qk) (contiguous grouping; the page gives no index map).
//
// Layouts (row-major, contiguous):
//   q, k      [B, T, H_qk, d_k]
//   v         [B, T, H_v,  d_v]
//   alpha, b  [B, T, H_v,  d_k]
//   w         [B, T, H_v,  d_v]
//   S0, S_T   [B, H_v, d_k, d_v]      (S0 may be NULL = zeros; S_T may be NULL)
//   o         [B, T, H_v, d_v]

#include <atomic>
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <thread>
#include <vector>

namespace {

struct Problem {
  int B, T, Hqk, Hv, dk, dv;
  double scale;
  const double *q, *k, *v, *alpha, *b, *w, *S0;
  double *o, *ST;
};

// One recurrence: sequence bi, value head hv.
void run_one(const Problem& p, int bi, int hv) {
  const int dk = p.dk, dv = p.dv;
  const int group = p.Hv / p.Hqk;
  const int hq = hv / group;
  std::vector<double> S((size_t)dk * dv, 0.0);
  std::vector<double> e(dk), z(dv), r(dv);
  const size_t sidx = ((size_t)bi * p.Hv + hv) * dk * dv;
  if (p.S0)
    for (size_t i = 0; i < (size_t)dk * dv; ++i) S[i] = p.S0[sidx + i];

  for (int t = 0; t < p.T; ++t) {
    const size_t tok = (size_t)bi * p.T + t;
    const double* qt = p.q + (tok * p.Hqk + hq) * dk;
    const double* kt = p.k + (tok * p.Hqk + hq) * dk;
    const double* vt = p.v + (tok * p.Hv + hv) * dv;
    const double* at = p.alpha + (tok * p.Hv + hv) * dk;
    const double* bt = p.b + (tok * p.Hv + hv) * dk;
    const double* wt = p.w + (tok * p.Hv + hv) * dv;
    double* ot = p.o + (tok * p.Hv + hv) * dv;

    // S̄ = Diag(α_t) S_{t−1}: row i of S (key channel i) scaled by α_t[i].
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= at[i];
    // e = b ⊙ k, z = w ⊙ v.
    for (int i = 0; i < dk; ++i) e[i] = bt[i] * kt[i];
    for (int j = 0; j < dv; ++j) z[j] = wt[j] * vt[j];
    // r = eᵀ S̄ (a d_v row vector).
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += e[i] * S[(size_t)i * dv + j];
      r[j] = acc;
    }
    // S_t = S̄ − k rᵀ + k zᵀ.
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j)
        S[(size_t)i * dv + j] += -kt[i] * r[j] + kt[i] * z[j];
    // o_t = s · S_tᵀ q_t.
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * qt[i];
      ot[j] = p.scale * acc;
    }
  }
  if (p.ST)
    for (size_t i = 0; i < (size_t)dk * dv; ++i) p.ST[sidx + i] = S[i];
}

}  // namespace

extern "C" {

// Returns 0 on success, -1 on bad arguments. n_threads <= 0 uses all cores.
int oracle_gdn2_forward(int B, int T, int H_qk, int H_v, int d_k, int d_v, double scale,
                        const double* q, const double* k, const double* v,
                        const double* alpha, const double* b, const double* w,
                        const double* S0, double* o, double* S_T, int n_threads) {
  if (B < 0 || T < 0 || H_qk <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0) return -1;
  if (H_v % H_qk != 0) return -1;
  if (T > 0 && (!q || !k || !v || !alpha || !b || !w || !o)) return -1;
  Problem p{B, T, H_qk, H_v, d_k, d_v, scale, q, k, v, alpha, b, w, S0, o, S_T};
  const int items = B * H_v;
  int nt = n_threads > 0 ? n_threads : (int)std::thread::hardware_concurrency();
  if (nt < 1) nt = 1;
  if (nt > items) nt = items > 0 ? items : 1;
  std::atomic<int> next{0};
  auto worker = [&]() {
    for (;;) {
      int it = next.fetch_add(1);
      if (it >= items) break;
      run_one(p, it / H_v, it % H_v);
    }
  };
  std::vector<std::thread> pool;
  for (int i = 1; i < nt; ++i) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
  return 0;
}

// Depthwise causal convolution, kernel 4, no bias, no activation, zero history
// ("Gated DeltaNet: o mixer em 48 das 64 camadas", Conceito: a short causal
// depthwise convolution with kernel 4 precedes the recurrence). Tap j of
// channel c multiplies the input 3 − j tokens back, so W[c][3] weights the
// current token:  y_t[c] = Σ_{j=0..3} W[c][j] · x_{t−3+j}[c].
//   x, y [B, T, C];  W [C, 4]
int oracle_causal_conv4(int B, int T, int C, const double* x, const double* W, double* y) {
  if (B < 0 || T < 0 || C <= 0) return -1;
  for (int bi = 0; bi < B; ++bi)
    for (int t = 0; t < T; ++t)
      for (int c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int j = 0; j < 4; ++j) {
          const int src = t - 3 + j;
          if (src < 0) continue;
          acc += W[(size_t)c * 4 + j] * x[((size_t)bi * T + src) * C + c];
        }
        y[((size_t)bi * T + t) * C + c] = acc;
      }
  return 0;
}

// Row-wise L2 normalisation: y = x · (Σ x² + eps)^(−1/2) over the last axis
// of length d, for n rows.
int oracle_l2norm(long long n, int d, double eps, const double* x, double* y) {
  if (n < 0 || d <= 0) return -1;
  for (long long r = 0; r < n; ++r) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[r * d + i] * x[r * d + i];
    const double inv = 1.0 / std::sqrt(ss + eps);
    for (int i = 0; i < d; ++i) y[r * d + i] = x[r * d + i] * inv;
  }
  return 0;
}

}  // extern "C"
