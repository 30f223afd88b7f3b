// Float64 CPU oracle for the gradients of the Gated DeltaNet-2 recurrence.
//
// TEST INFRASTRUCTURE ONLY, like gdn2_oracle.cpp: nothing in the product path
// may link, load or call this file. It shares no code with the CUDA library.
//
// The forward recurrence is the one of "Resumo Técnico: Gated DeltaNet-2",
// Metodologia §1 "Regra Delta Portão-2", per (sequence, value head):
//     S̄_t = Diag(α_t) S_{t−1},  e_t = b_t ⊙ k_t,  z_t = w_t ⊙ v_t
//     u_t = z_t − S̄_tᵀ e_t,     S_t = S̄_t + k_t u_tᵀ   (= (I − k eᵀ) S̄ + k zᵀ)
//     o_t = s · S_tᵀ q_t
// and the loss whose gradients are returned is L = <dO, o> + <dS_T, S_T> for
// given upstream gradients dO (like o) and dS_T (like S_T): the
// vector-Jacobian product that a training step's backward pass computes
// ("Resumo Técnico: Gated DeltaNet-2", Metodologia §3, "Passagem de
// Retropropagação Consciente de Portões": the gradient flows through the
// erase gate b and the write gate w per channel).
//
// It is reverse-mode differentiation of the token loop written out by hand,
// one step at a time in the reverse order of the forward operations, with
// the states recomputed from checkpoints taken every 64 tokens. For each
// token t, going backwards, with dS the gradient of S_t:
//     dq_t = s S_t do_t,             dS += s q_t do_tᵀ           (o_t = s S_tᵀ q_t)
//     dk_t += dS u_t,  du = dSᵀ k_t,  dS̄ = dS                    (S_t = S̄ + k uᵀ)
//     dz = du,  de = −S̄ du,  dS̄ −= e duᵀ                         (u = z − S̄ᵀ e)
//     dw_t = du ⊙ v_t,  dv_t = du ⊙ w_t                           (z = w ⊙ v)
//     db_t = de ⊙ k_t,  dk_t += de ⊙ b_t                          (e = b ⊙ k)
//     dα_t[i] = Σ_j dS̄[i][j] S_{t−1}[i][j],  dS_{t−1} = Diag(α_t) dS̄
// Value head h reads query/key head h / (H_v / H_qk), so dq and dk of a query/
// key head sum the contributions of its value heads; the work is split over
// (sequence, query/key head) so that no two threads write the same gradient.
//
// Layouts as in gdn2_oracle.cpp (gates per value head and per channel); the
// gradients have the shapes of their inputs. dS0 is the gradient of S0.

#include <algorithm>
#include <atomic>
#include <cstddef>
#include <thread>
#include <vector>

namespace {

struct BwdProblem {
  int B, T, Hqk, Hv, dk, dv;
  double scale;
  const double *q, *k, *v, *alpha, *b, *w, *S0, *dO, *dST;
  double *dq, *dk_, *dv_, *dalpha, *db, *dw, *dS0;
};

constexpr int kCkpt = 64;   // tokens between recomputation checkpoints

// Gradients of the recurrence of sequence bi, value head hv (accumulating
// into dq, dk of its query/key head).
void backward_one(const BwdProblem& p, int bi, int hv) {
  const int dk = p.dk, dv = p.dv;
  const size_t SS = (size_t)dk * dv;
  const int hq = hv / (p.Hv / p.Hqk);
  const size_t sidx = ((size_t)bi * p.Hv + hv) * SS;
  auto at = [&](const double* base, int t, int H, int h, int d) {
    return base + (((size_t)bi * p.T + t) * H + h) * d;
  };

  // One forward step from S (S_{t−1}) to S_t in place; also returns S̄ and u.
  std::vector<double> e(dk), z(dv), u(dv), Sbar(SS);
  auto step = [&](std::vector<double>& S, int t) {
    const double* kt = at(p.k, t, p.Hqk, hq, dk);
    const double* at_ = at(p.alpha, t, p.Hv, hv, dk);
    const double* bt = at(p.b, t, p.Hv, hv, dk);
    const double* vt = at(p.v, t, p.Hv, hv, dv);
    const double* wt = at(p.w, t, p.Hv, hv, dv);
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) Sbar[(size_t)i * dv + j] = at_[i] * S[(size_t)i * dv + j];
    for (int i = 0; i < dk; ++i) e[i] = bt[i] * kt[i];
    for (int j = 0; j < dv; ++j) z[j] = wt[j] * vt[j];
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += Sbar[(size_t)i * dv + j] * e[i];
      u[j] = z[j] - acc;
    }
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] = Sbar[(size_t)i * dv + j] + kt[i] * u[j];
  };

  // Checkpoints: the state before tokens 0, 64, 128, ...
  const int nblk = (p.T + kCkpt - 1) / kCkpt;
  std::vector<std::vector<double>> ckpt(nblk);
  std::vector<double> S(SS, 0.0);
  if (p.S0)
    for (size_t x = 0; x < SS; ++x) S[x] = p.S0[sidx + x];
  for (int blk = 0; blk < nblk; ++blk) {
    ckpt[blk] = S;
    for (int t = blk * kCkpt; t < std::min(p.T, (blk + 1) * kCkpt); ++t) step(S, t);
  }

  // dS: gradient of the state after the last token.
  std::vector<double> dS(SS, 0.0);
  if (p.dST)
    for (size_t x = 0; x < SS; ++x) dS[x] = p.dST[sidx + x];
  std::vector<std::vector<double>> states(kCkpt + 1, std::vector<double>(SS));
  std::vector<double> du(dv), de(dk);
  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * kCkpt, t1 = std::min(p.T, t0 + kCkpt);
    states[0] = ckpt[blk];
    for (int t = t0; t < t1; ++t) {
      states[t - t0 + 1] = states[t - t0];
      step(states[t - t0 + 1], t);
    }
    for (int t = t1 - 1; t >= t0; --t) {
      const std::vector<double>& Sprev = states[t - t0];
      const std::vector<double>& Scur = states[t - t0 + 1];
      // recompute S̄, e, z, u of token t (step() on a copy of S_{t−1})
      std::vector<double> tmp = Sprev;
      step(tmp, t);
      const double* qt = at(p.q, t, p.Hqk, hq, dk);
      const double* kt = at(p.k, t, p.Hqk, hq, dk);
      const double* at_ = at(p.alpha, t, p.Hv, hv, dk);
      const double* bt = at(p.b, t, p.Hv, hv, dk);
      const double* vt = at(p.v, t, p.Hv, hv, dv);
      const double* wt = at(p.w, t, p.Hv, hv, dv);
      const double* dot = at(p.dO, t, p.Hv, hv, dv);
      double* dqt = p.dq + (((size_t)bi * p.T + t) * p.Hqk + hq) * dk;
      double* dkt = p.dk_ + (((size_t)bi * p.T + t) * p.Hqk + hq) * dk;
      double* dat = p.dalpha + (((size_t)bi * p.T + t) * p.Hv + hv) * dk;
      double* dbt = p.db + (((size_t)bi * p.T + t) * p.Hv + hv) * dk;
      double* dvt = p.dv_ + (((size_t)bi * p.T + t) * p.Hv + hv) * dv;
      double* dwt = p.dw + (((size_t)bi * p.T + t) * p.Hv + hv) * dv;
      // o_t = s S_tᵀ q_t
      for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += Scur[(size_t)i * dv + j] * dot[j];
        dqt[i] += p.scale * acc;
      }
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += p.scale * qt[i] * dot[j];
      // S_t = S̄ + k uᵀ
      for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += dS[(size_t)i * dv + j] * u[j];
        dkt[i] += acc;
      }
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += dS[(size_t)i * dv + j] * kt[i];
        du[j] = acc;
      }
      // u = z − S̄ᵀ e
      for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += Sbar[(size_t)i * dv + j] * du[j];
        de[i] = -acc;
      }
      for (int j = 0; j < dv; ++j) {
        dwt[j] = du[j] * vt[j];
        dvt[j] = du[j] * wt[j];
      }
      for (int i = 0; i < dk; ++i) {
        dbt[i] = de[i] * kt[i];
        dkt[i] += de[i] * bt[i];
      }
      // dS̄ = dS − e duᵀ; S̄ = Diag(α) S_{t−1}
      for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) {
          const double dsb = dS[(size_t)i * dv + j] - e[i] * du[j];
          acc += dsb * Sprev[(size_t)i * dv + j];
          dS[(size_t)i * dv + j] = at_[i] * dsb;
        }
        dat[i] = acc;
      }
    }
  }
  if (p.dS0)
    for (size_t x = 0; x < SS; ++x) p.dS0[sidx + x] = dS[x];
}

}  // namespace

extern "C" {

// Gradients of L = <dO, o> + <dS_T, S_T> with respect to q, k, v, alpha, b,
// w and S0 (layouts of gdn2_oracle.cpp; S0 and dS_T may be NULL = zeros).
// dq and dk must be zero on entry (they accumulate over the value heads of a
// group). Returns 0 on success, -1 on bad arguments. n_threads <= 0: all cores.
int oracle_gdn2_backward(int B, int T, int H_qk, int H_v, int d_k, int d_v, double scale,
                         const double* q, const double* k, const double* v, const double* alpha,
                         const double* b, const double* w, const double* S0, const double* dO,
                         const double* dS_T, double* dq, double* dk, double* dv, double* dalpha,
                         double* db, double* dw, double* dS0, int n_threads) {
  if (B < 0 || T < 0 || H_qk <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0) return -1;
  if (H_v % H_qk != 0) return -1;
  if (T > 0 && (!q || !k || !v || !alpha || !b || !w || !dO || !dq || !dk || !dv || !dalpha || !db || !dw))
    return -1;
  BwdProblem p{B, T, H_qk, H_v, d_k, d_v, scale, q, k, v, alpha, b, w, S0, dO, dS_T,
               dq, dk, dv, dalpha, db, dw, dS0};
  const int group = H_v / H_qk;
  const int items = B * H_qk;   // (sequence, query/key head): owns dq, dk of that head
  int nt = n_threads > 0 ? n_threads : (int)std::thread::hardware_concurrency();
  if (nt < 1) nt = 1;
  if (nt > items) nt = items > 0 ? items : 1;
  std::atomic<int> next{0};
  auto worker = [&]() {
    for (;;) {
      const int it = next.fetch_add(1);
      if (it >= items) break;
      const int bi = it / H_qk, hq = it % H_qk;
      for (int g = 0; g < group; ++g) backward_one(p, bi, hq * group + g);
    }
  };
  std::vector<std::thread> pool;
  for (int i = 1; i < nt; ++i) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
  return 0;
}

}  // extern "C"
