// Backward pass of the chunked prefill, exact fp32 SIMT arithmetic.
//
// Gradients of L = <dO, o> + <dS_T, S_T> for the recurrence ("Resumo Técnico:
// Gated DeltaNet-2", Metodologia §1) with respect to q, k, v, the gates and S0,
// in the chunked form of the forward ("Uma análise das variantes de atenção
// linear da família DeltaNet", "Chunkwise KDA"; the decoupled gates of the
// GDN-2 summary, Metodologia §3, whose backward pass carries the per-channel
// erase and write gates through the gradients of the WY factors). Per chunk
// of C tokens with entry state S, cumulative decays γ_i = Π_{s≤i} α_s, and the
// pairwise decay D_ij = Π_{j<s≤i} α_s (per key channel):
//     T_ij = Σ_c e_ic k_jc D_ijc (j < i),  Aqk_ij = Σ_c q_ic k_jc D_ijc (j ≤ i)
//     A = (I + T)⁻¹,  R = Z − Ē S,  U = A R,  O = s (Q̄ S + Aqk U),
//     S' = Γ S + K_endᵀ U,  Ē = γ ⊙ e, Q̄ = γ ⊙ q, K_end,j = k_j ⊙ Π_{j<s≤C} α_s.
// Going back through the chunk with dO and dS' (the gradient of S'):
//     dU = s Aqkᵀ dO + K_end dS',   dR = Aᵀ dU  (= dZ),
//     dS = s Q̄ᵀ dO + Γ dS' − Ēᵀ dR  (carried to the previous chunk),
//     dT_ij = −Σ_v dR_iv U_jv (j < i),   dAqk_ij = s Σ_v dO_iv U_jv (j ≤ i),
//     dQ̄ = s dO Sᵀ,  dĒ = −dR Sᵀ,  dK_end = U dS'ᵀ,  dΓ_c = Σ_v dS'_cv S_cv,
// then through the decays in log space (G_i = Σ_{s≤i} log α_s): every factor
// is exp of a difference of G, so its gradient lands on the G of both ends,
// and dlog α_s = Σ_{i≥s} dG_i. The Gram gradients use the running products
// of α (no reciprocal, no logarithm), as the forward's exact kernel does, so
// every α ∈ (0, 1] is taken.
//
// One CTA per (sequence, value head, tile of DVT value columns): the state's
// columns evolve independently, so each CTA first runs the forward over all
// chunks, writing its columns of each chunk's entry state to a checkpoint
// buffer, then walks the chunks in reverse carrying its columns of dS. The
// gradients of v and w are per column and written once; those of q, k, α and
// b are sums over all columns (and over the value heads of a query/key head)
// and are added with atomics into buffers the launcher zeroes.

#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int BC = 16;        // chunk of the backward pass
constexpr int BT = 512;       // threads (16 warps: one CTA per SM for its shared memory)

template <int D>
struct BwdSmem {
  static constexpr int DVT = D < 64 ? D : 64;   // value columns per CTA
  static constexpr int DP = D + 4;              // key rows: 16-byte multiples (broadcast rows load as float4)
  static constexpr int CP = BC + 1;
  static constexpr int VP = DVT + 1;            // (odd: column walks across lanes are conflict-free)
  // [BC][DP] ×11: q, k, b, α, e, γ, bk (Π_{i<s<BC} α), and the gradients of q, k, e, G
  // [BC][CP] ×5:  T, A = (I+T)⁻¹, Aqk, dT, dAqk
  // [BC][VP] ×6:  Z (then R, then dR), U, dO, dU, v, w
  // [D][VP] ×3:   S, dS', dS
  // [D]:          γ_C
  static constexpr size_t floats = 11 * BC * DP + 5 * BC * CP + 6 * BC * VP + 3 * D * VP + D;
  static constexpr size_t bytes = floats * sizeof(float);
};
static_assert(BwdSmem<128>::bytes <= 232448, "backward shared memory");

template <int D, typename TIn, typename TdO>
__global__ void __launch_bounds__(BT, 1) chunk_bwd_kernel(BwdArgs a) {
  using L = BwdSmem<D>;
  constexpr int DVT = L::DVT, DP = L::DP, CP = L::CP, VP = L::VP;
  constexpr int TILES = D / DVT;
  constexpr int CPT = (D + 31) / 32;   // channels per lane of the pairwise passes (one warp per row)
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sK = sQ + BC * DP;
  float* sB = sK + BC * DP;
  float* sAl = sB + BC * DP;
  float* sE = sAl + BC * DP;
  float* sGm = sE + BC * DP;
  float* sBk = sGm + BC * DP;
  float* gQ = sBk + BC * DP;
  float* gK = gQ + BC * DP;
  float* gE = gK + BC * DP;
  float* gG = gE + BC * DP;
  float* sT = gG + BC * DP;
  float* sA = sT + BC * CP;
  float* sAq = sA + BC * CP;
  float* sdT = sAq + BC * CP;
  float* sdAq = sdT + BC * CP;
  float* tZ = sdAq + BC * CP;
  float* tU = tZ + BC * VP;
  float* tdO = tU + BC * VP;
  float* tdU = tdO + BC * VP;
  float* tV = tdU + BC * VP;
  float* tW = tV + BC * VP;
  float* sS = tW + BC * VP;
  float* sdS = sS + D * VP;
  float* sdSn = sdS + D * VP;
  float* sgC = sdSn + D * VP;

  const int tile = blockIdx.x % TILES, bh = blockIdx.x / TILES;
  const int h = bh % a.Hv, bi = bh / a.Hv;
  const int hq = h / (a.Hv / a.Hqk);
  const int hg = a.Hg == a.Hv ? h : hq;
  const int col0 = tile * DVT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool full = a.gate_mode == GDN2_GATES_FULL, alpha_pc = a.gate_mode != GDN2_GATES_GDN;
  const bool lg = a.gate_logits != 0;
  const int T = a.T, N = (T + BC - 1) / BC;
  const float s = a.scale;
  const TIn* qg = static_cast<const TIn*>(a.q);
  const TIn* kg = static_cast<const TIn*>(a.k);
  const TIn* vg = static_cast<const TIn*>(a.v);
  const TdO* og = static_cast<const TdO*>(a.dO);
  float* ckpt = a.ckpt + (size_t)bh * N * D * D;   // [N][D][D]; this CTA owns columns col0 ..

  // ---- one chunk's inputs: key side [BC][D], value side of the tile [BC][DVT]
  auto load_chunk = [&](int c, bool grads) {
    const int t0 = c * BC, Lc = min(BC, T - t0);
    for (int idx = tid; idx < BC * D; idx += BT) {
      const int i = idx / D, cc = idx % D;
      float q = 0.f, k = 0.f, al = 1.f, bb = 0.f;
      if (i < Lc) {
        const size_t t = (size_t)bi * T + t0 + i;
        const size_t qk = (t * a.Hqk + hq) * D + cc;
        q = to_f32(qg[qk]);
        k = to_f32(kg[qk]);
        const size_t gr = t * a.Hg + hg;
        al = gate_at(a.alpha, alpha_pc ? gr * D + cc : gr, lg);
        bb = gate_at(a.b, full ? gr * D + cc : gr, lg);
      }
      sQ[i * DP + cc] = q;
      sK[i * DP + cc] = k;
      sAl[i * DP + cc] = al;
      sB[i * DP + cc] = bb;
      sE[i * DP + cc] = bb * k;
    }
    for (int idx = tid; idx < BC * DVT; idx += BT) {
      const int i = idx / DVT, v = idx % DVT;
      float vv = 0.f, ww = 0.f, d = 0.f;
      if (i < Lc) {
        const size_t t = (size_t)bi * T + t0 + i;
        const size_t vi = (t * a.Hv + h) * D + col0 + v;
        vv = to_f32(vg[vi]);
        ww = full ? gate_at(a.w, vi, lg) : gate_at(a.b, t * a.Hg + hg, lg);
        if (grads) d = to_f32(og[vi]);
      }
      tV[i * VP + v] = vv;
      tW[i * VP + v] = ww;
      tZ[i * VP + v] = ww * vv;
      tdO[i * VP + v] = d;
    }
  };

  // ---- γ (forward products), bk (backward products), γ_C; then T, Aqk by
  // running products per (column j, 16-channel part). Warp w owns columns
  // 2w, 2w + 1 and runs its rows from 2w.
  auto decays_and_gram = [&]() {
    if (tid < D) {
      const int c = tid;
      float g = 1.f;
      for (int i = 0; i < BC; ++i) {
        g *= sAl[i * DP + c];
        sGm[i * DP + c] = g;
      }
      sgC[c] = g;
      float p = 1.f;
      for (int i = BC - 1; i >= 0; --i) {
        sBk[i * DP + c] = p;
        p *= sAl[i * DP + c];
      }
    }
    // warp j takes key row j, lane l its channels l + 32 m
    const int j = warp, part = lane;
    float kj[CPT], dd[CPT];
#pragma unroll
    for (int m = 0; m < CPT; ++m) {
      kj[m] = part + 32 * m < D ? sK[j * DP + part + 32 * m] : 0.f;
      dd[m] = 1.f;
    }
    for (int i = j; i < BC; ++i) {
      float at = 0.f, aa = 0.f;
#pragma unroll
      for (int m = 0; m < CPT; ++m) {
        const int c = part + 32 * m;
        if (c < D) {
          dd[m] *= i > j ? sAl[i * DP + c] : 1.f;
          const float kd = kj[m] * dd[m];
          at = fmaf(sE[i * DP + c], kd, at);
          aa = fmaf(sQ[i * DP + c], kd, aa);
        }
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        at += __shfl_xor_sync(0xffffffffu, at, off);
        aa += __shfl_xor_sync(0xffffffffu, aa, off);
      }
      if (part == 0) {
        sT[i * CP + j] = i > j ? at : 0.f;
        sAq[i * CP + j] = aa;
      }
    }
  };

  // Register tiles of the products below. A BC-row result: warp w takes rows
  // 2(w mod 8), 2(w mod 8) + 1 and, with lane l, the value columns
  // l + 32(w/8 + 2n) (NVH of them) or key columns l + 32(w/8 + 2n) (NKH). A
  // D-row result: warp w takes rows RW·w .. RW·w + RW − 1 and lane l the value
  // columns l + 32n (NV).
  constexpr int NW = BT / 32;
  constexpr int NV = (DVT + 31) / 32, NK = (D + 31) / 32;
  constexpr int NVH = (NV + 1) / 2, NKH = (NK + 1) / 2;
  constexpr int RW = D / NW > 0 ? D / NW : 1;
  static_assert(BC == 16 && NW == 16, "row tiles assume 16 rows and 16 warps");
  const int r2 = 2 * (warp & 7), wh = warp >> 3;
  auto vcol = [&](int n) { return lane + 32 * (wh + 2 * n); };
  auto kcol = [&](int n) { return lane + 32 * (wh + 2 * n); };
  // Ē = γ ⊙ e, Q̄ = γ ⊙ q and K_end = k ⊙ bk, into the gradient arrays, which
  // the backward sweep rewrites only after their last use.
  auto absorbed = [&]() {
    for (int idx = tid; idx < BC * D; idx += BT) {
      const int i = idx / D, c = idx % D;
      const float g = sGm[i * DP + c];
      gE[i * DP + c] = g * sE[i * DP + c];
      gQ[i * DP + c] = g * sQ[i * DP + c];
      gK[i * DP + c] = sK[i * DP + c] * sBk[i * DP + c];
    }
  };
  // A = (I + T)⁻¹ by forward substitution, one column per thread; R = Z − Ē S.
  auto inverse_and_R = [&]() {
    if (tid < BC) {
      const int j = tid;
      for (int i = 0; i < BC; ++i) {
        float x = i == j ? 1.f : 0.f;
        if (i > j) {
          float acc = 0.f;
          for (int l = j; l < i; ++l) acc = fmaf(sT[i * CP + l], sA[l * CP + j], acc);
          x = -acc;
        }
        sA[i * CP + j] = x;
      }
    }
    {
      float acc[2][NVH] = {};
#pragma unroll 2
      for (int c4 = 0; c4 < D; c4 += 4) {
        const float4 e0 = *reinterpret_cast<const float4*>(gE + r2 * DP + c4);
        const float4 e1 = *reinterpret_cast<const float4*>(gE + (r2 + 1) * DP + c4);
        const float a0[4] = {e0.x, e0.y, e0.z, e0.w}, a1[4] = {e1.x, e1.y, e1.z, e1.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int n = 0; n < NVH; ++n) {
            const int v = vcol(n);
            const float sv = v < DVT ? sS[(c4 + t) * VP + v] : 0.f;
            acc[0][n] = fmaf(a0[t], sv, acc[0][n]);
            acc[1][n] = fmaf(a1[t], sv, acc[1][n]);
          }
      }
#pragma unroll
      for (int n = 0; n < NVH; ++n) {
        const int v = vcol(n);
        if (v < DVT) {
          tZ[r2 * VP + v] -= acc[0][n];
          tZ[(r2 + 1) * VP + v] -= acc[1][n];
        }
      }
    }
  };
  // U = A R
  auto solve_U = [&]() {
    for (int idx = tid; idx < BC * DVT; idx += BT) {
      const int i = idx / DVT, v = idx % DVT;
      float acc = 0.f;
      for (int j = 0; j <= i; ++j) acc = fmaf(sA[i * CP + j], tZ[j * VP + v], acc);
      tU[i * VP + v] = acc;
    }
  };

  // ------------------------------------------------------------------ forward
  for (int idx = tid; idx < D * DVT; idx += BT) {
    const int r = idx / DVT, v = idx % DVT;
    sS[r * VP + v] = a.S0 ? a.S0[((size_t)bh * D + r) * D + col0 + v] : 0.f;
  }
  for (int c = 0; c < N; ++c) {
    __syncthreads();
    for (int idx = tid; idx < D * DVT; idx += BT) {
      const int r = idx / DVT, v = idx % DVT;
      ckpt[((size_t)c * D + r) * D + col0 + v] = sS[r * VP + v];
    }
    load_chunk(c, false);
    __syncthreads();
    decays_and_gram();
    __syncthreads();
    absorbed();
    __syncthreads();
    inverse_and_R();
    __syncthreads();
    solve_U();
    __syncthreads();
    // S ← Γ S + K_endᵀ U (each thread updates its own entries in place)
    for (int r0 = RW * warp; r0 < D; r0 += RW * NW) {
      float acc[RW][NV];
#pragma unroll
      for (int m = 0; m < RW; ++m)
#pragma unroll
        for (int n = 0; n < NV; ++n) {
          const int v = lane + 32 * n;
          acc[m][n] = v < DVT ? sgC[r0 + m] * sS[(r0 + m) * VP + v] : 0.f;
        }
#pragma unroll 4
      for (int j = 0; j < BC; ++j) {
        float u[NV];
#pragma unroll
        for (int n = 0; n < NV; ++n) u[n] = lane + 32 * n < DVT ? tU[j * VP + lane + 32 * n] : 0.f;
#pragma unroll
        for (int m = 0; m < RW; ++m) {
          const float ke = gK[j * DP + r0 + m];
#pragma unroll
          for (int n = 0; n < NV; ++n) acc[m][n] = fmaf(ke, u[n], acc[m][n]);
        }
      }
#pragma unroll
      for (int m = 0; m < RW; ++m)
#pragma unroll
        for (int n = 0; n < NV; ++n)
          if (lane + 32 * n < DVT) sS[(r0 + m) * VP + lane + 32 * n] = acc[m][n];
    }
  }

  // ------------------------------------------------------------------ backward
  float* dSp = sdS;     // dS' (gradient of the chunk's exit state)
  float* dSn = sdSn;    // dS of its entry state
  __syncthreads();
  for (int idx = tid; idx < D * DVT; idx += BT) {
    const int r = idx / DVT, v = idx % DVT;
    dSp[r * VP + v] = a.dST ? a.dST[((size_t)bh * D + r) * D + col0 + v] : 0.f;
  }
  for (int c = N - 1; c >= 0; --c) {
    const int t0 = c * BC, Lc = min(BC, T - t0);
    __syncthreads();
    for (int idx = tid; idx < D * DVT; idx += BT) {
      const int r = idx / DVT, v = idx % DVT;
      sS[r * VP + v] = ckpt[((size_t)c * D + r) * D + col0 + v];
    }
    load_chunk(c, true);
    __syncthreads();
    decays_and_gram();
    __syncthreads();
    absorbed();
    __syncthreads();
    inverse_and_R();
    __syncthreads();
    solve_U();
    __syncthreads();
    // dU = s Aqkᵀ dO + K_end dS'
    {
      float aq[2][NVH] = {}, ak[2][NVH] = {};
      for (int i = r2; i < BC; ++i) {
        const float a0 = sAq[i * CP + r2], a1 = i > r2 ? sAq[i * CP + r2 + 1] : 0.f;
#pragma unroll
        for (int n = 0; n < NVH; ++n) {
          const int v = vcol(n);
          const float d = v < DVT ? tdO[i * VP + v] : 0.f;
          aq[0][n] = fmaf(a0, d, aq[0][n]);
          aq[1][n] = fmaf(a1, d, aq[1][n]);
        }
      }
#pragma unroll 2
      for (int c4 = 0; c4 < D; c4 += 4) {
        const float4 q0 = *reinterpret_cast<const float4*>(gK + r2 * DP + c4);
        const float4 q1 = *reinterpret_cast<const float4*>(gK + (r2 + 1) * DP + c4);
        const float k0[4] = {q0.x, q0.y, q0.z, q0.w}, k1[4] = {q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int n = 0; n < NVH; ++n) {
            const int v = vcol(n);
            const float p = v < DVT ? dSp[(c4 + t) * VP + v] : 0.f;
            ak[0][n] = fmaf(k0[t], p, ak[0][n]);
            ak[1][n] = fmaf(k1[t], p, ak[1][n]);
          }
      }
#pragma unroll
      for (int n = 0; n < NVH; ++n) {
        const int v = vcol(n);
        if (v < DVT) {
          tdU[r2 * VP + v] = fmaf(s, aq[0][n], ak[0][n]);
          tdU[(r2 + 1) * VP + v] = fmaf(s, aq[1][n], ak[1][n]);
        }
      }
    }
    __syncthreads();
    // dR = Aᵀ dU, into the R array
    for (int idx = tid; idx < BC * DVT; idx += BT) {
      const int i = idx / DVT, v = idx % DVT;
      float acc = 0.f;
      for (int j = i; j < BC; ++j) acc = fmaf(sA[j * CP + i], tdU[j * VP + v], acc);
      tZ[i * VP + v] = acc;
    }
    __syncthreads();
    float* tdR = tZ;
    // dS of the entry state: Γ dS' + s Q̄ᵀ dO − Ēᵀ dR
    for (int r0 = RW * warp; r0 < D; r0 += RW * NW) {
      float acc[RW][NV];
#pragma unroll
      for (int m = 0; m < RW; ++m)
#pragma unroll
        for (int n = 0; n < NV; ++n) {
          const int v = lane + 32 * n;
          acc[m][n] = v < DVT ? sgC[r0 + m] * dSp[(r0 + m) * VP + v] : 0.f;
        }
#pragma unroll 2
      for (int i = 0; i < BC; ++i) {
        float od[NV], rd[NV];
#pragma unroll
        for (int n = 0; n < NV; ++n) {
          const int v = lane + 32 * n;
          od[n] = v < DVT ? s * tdO[i * VP + v] : 0.f;
          rd[n] = v < DVT ? tdR[i * VP + v] : 0.f;
        }
#pragma unroll
        for (int m = 0; m < RW; ++m) {
          const float qb = gQ[i * DP + r0 + m], eb = gE[i * DP + r0 + m];
#pragma unroll
          for (int n = 0; n < NV; ++n) acc[m][n] = fmaf(qb, od[n], fmaf(-eb, rd[n], acc[m][n]));
        }
      }
#pragma unroll
      for (int m = 0; m < RW; ++m)
#pragma unroll
        for (int n = 0; n < NV; ++n)
          if (lane + 32 * n < DVT) dSn[(r0 + m) * VP + lane + 32 * n] = acc[m][n];
    }
    // dv = dR ⊙ w; dw = dR ⊙ v (per channel), or its sum into dβ (tied gates)
    for (int idx = tid; idx < BC * DVT; idx += BT) {
      const int i = idx / DVT, v = idx % DVT;
      if (i >= Lc) continue;
      const size_t t = (size_t)bi * T + t0 + i;
      const size_t vi = (t * a.Hv + h) * D + col0 + v;
      const float dr = tdR[i * VP + v], ww = tW[i * VP + v];
      a.dv[vi] = dr * ww;
      if (full) a.dw[vi] = dr * tV[i * VP + v] * (lg ? ww * (1.f - ww) : 1.f);
    }
    if (!full) {
      // Σ_v dR ⊙ v per token, one warp per token
      for (int i = warp; i < Lc; i += BT / 32) {
        float acc = 0.f;
        for (int v = lane; v < DVT; v += 32) acc = fmaf(tdR[i * VP + v], tV[i * VP + v], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
          const float beta = tW[i * VP];
          atomicAdd(a.db + ((size_t)bi * T + t0 + i) * a.Hg + hg, acc * (lg ? beta * (1.f - beta) : 1.f));
        }
      }
    }
    // dT, dAqk
    if (tid < BC * BC) {
      const int i = tid >> 4, j = tid & 15;
      float x = 0.f, y = 0.f;
      if (j <= i) {
        for (int v = 0; v < DVT; ++v) {
          const float u = tU[j * VP + v];
          x = fmaf(tdR[i * VP + v], u, x);
          y = fmaf(tdO[i * VP + v], u, y);
        }
      }
      sdT[i * CP + j] = j < i ? -x : 0.f;
      sdAq[i * CP + j] = j <= i ? s * y : 0.f;
    }
    // per (i, c): dQ̄ = s dO Sᵀ, dĒ = −dR Sᵀ, dK_end = U dS'ᵀ, and what they give
    // q, e, k and G directly (after every thread's last read of Q̄, Ē, K_end)
    __syncthreads();
    {
      float aq[2][NKH] = {}, ae[2][NKH] = {}, ak[2][NKH] = {};
#pragma unroll 2
      for (int v = 0; v < DVT; ++v) {
        const float o0 = tdO[r2 * VP + v], o1 = tdO[(r2 + 1) * VP + v];
        const float d0 = tdR[r2 * VP + v], d1 = tdR[(r2 + 1) * VP + v];
        const float u0 = tU[r2 * VP + v], u1 = tU[(r2 + 1) * VP + v];
#pragma unroll
        for (int n = 0; n < NKH; ++n) {
          const int cc = kcol(n);
          const float sv = cc < D ? sS[cc * VP + v] : 0.f, pv = cc < D ? dSp[cc * VP + v] : 0.f;
          aq[0][n] = fmaf(o0, sv, aq[0][n]);
          aq[1][n] = fmaf(o1, sv, aq[1][n]);
          ae[0][n] = fmaf(d0, sv, ae[0][n]);
          ae[1][n] = fmaf(d1, sv, ae[1][n]);
          ak[0][n] = fmaf(u0, pv, ak[0][n]);
          ak[1][n] = fmaf(u1, pv, ak[1][n]);
        }
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int n = 0; n < NKH; ++n) {
          const int i = r2 + h2, cc = kcol(n);
          if (cc >= D) continue;
          const float dq_ = s * aq[h2][n], de_ = -ae[h2][n], dke = ak[h2][n];
          const float g = sGm[i * DP + cc], bk = sBk[i * DP + cc];
          gQ[i * DP + cc] = g * dq_;
          gE[i * DP + cc] = g * de_;
          gK[i * DP + cc] = bk * dke;
          gG[i * DP + cc] = g * (sQ[i * DP + cc] * dq_ + sE[i * DP + cc] * de_) - sK[i * DP + cc] * bk * dke;
        }
    }
    __syncthreads();
    // G at the chunk's last token: from K_end (Σ_j K_end,j ⊙ dK_end,j) and Γ
    if (tid < D) {
      const int cc = tid;
      float acc = 0.f;
      for (int j = 0; j < BC; ++j) acc = fmaf(sK[j * DP + cc], gK[j * DP + cc], acc);
      float dg = 0.f;
      for (int v = 0; v < DVT; ++v) dg = fmaf(dSp[cc * VP + v], sS[cc * VP + v], dg);
      gG[(BC - 1) * DP + cc] += fmaf(sgC[cc], dg, acc);
    }
    __syncthreads();
    // Gram gradients, key side: thread (j, part) runs i up from j with D_ij
    {
      const int j = warp, part = lane;   // warp j: key row j, lane l: channels l + 32 m
      float dd[CPT], ak[CPT], ag[CPT], kj[CPT];
#pragma unroll
      for (int m = 0; m < CPT; ++m) {
        dd[m] = 1.f;
        ak[m] = 0.f;
        ag[m] = 0.f;
        kj[m] = part + 32 * m < D ? sK[j * DP + part + 32 * m] : 0.f;
      }
      for (int i = j; i < BC; ++i) {
        const float ct = sdT[i * CP + j], ca = sdAq[i * CP + j];
#pragma unroll
        for (int m = 0; m < CPT; ++m) {
          const int cc = part + 32 * m;
          if (cc < D) {
            dd[m] *= i > j ? sAl[i * DP + cc] : 1.f;
            const float x = fmaf(ct, sE[i * DP + cc], ca * sQ[i * DP + cc]) * dd[m];
            ak[m] += x;
            ag[m] = fmaf(x, kj[m], ag[m]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < CPT; ++m) {
        const int cc = part + 32 * m;
        if (cc < D) {
          gK[j * DP + cc] += ak[m];
          gG[j * DP + cc] -= ag[m];
        }
      }
    }
    __syncthreads();
    // query / erase side: thread (i, part) runs j down from i with D_ij
    {
      const int i = warp, part = lane;   // warp i: row i, lane l: channels l + 32 m
      float dd[CPT], ae[CPT], aq[CPT], ag[CPT];
#pragma unroll
      for (int m = 0; m < CPT; ++m) {
        dd[m] = 1.f;
        ae[m] = 0.f;
        aq[m] = 0.f;
        ag[m] = 0.f;
      }
      for (int j = i; j >= 0; --j) {
        const float ct = sdT[i * CP + j], ca = sdAq[i * CP + j];
#pragma unroll
        for (int m = 0; m < CPT; ++m) {
          const int cc = part + 32 * m;
          if (cc < D) {
            if (j < i) dd[m] *= sAl[(j + 1) * DP + cc];
            const float kd = sK[j * DP + cc] * dd[m];
            ae[m] = fmaf(ct, kd, ae[m]);
            aq[m] = fmaf(ca, kd, aq[m]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < CPT; ++m) {
        const int cc = part + 32 * m;
        if (cc >= D) continue;
        ag[m] = fmaf(ae[m], sE[i * DP + cc], aq[m] * sQ[i * DP + cc]);
        gE[i * DP + cc] += ae[m];
        gQ[i * DP + cc] += aq[m];
        gG[i * DP + cc] += ag[m];
      }
    }
    __syncthreads();
    // dlog α_s = Σ_{i≥s} dG_i per channel (into gG)
    if (tid < D) {
      const int cc = tid;
      float acc = 0.f;
      for (int i = BC - 1; i >= 0; --i) {
        acc += gG[i * DP + cc];
        gG[i * DP + cc] = acc;
      }
    }
    __syncthreads();
    // gradients of this tile's columns into q, k, α, b (per channel) by
    // atomics; scalar gates (tied β, scalar α) as per-token sums
    for (int i = warp; i < Lc; i += BT / 32) {
      const size_t t = (size_t)bi * T + t0 + i;
      const size_t qk = (t * a.Hqk + hq) * D;
      const size_t gr = t * a.Hg + hg;
      float sa = 0.f, sb = 0.f;
      for (int cc = lane; cc < D; cc += 32) {
        const float k = sK[i * DP + cc], ge = gE[i * DP + cc], al = sAl[i * DP + cc], bb = sB[i * DP + cc];
        atomicAdd(a.dq + qk + cc, gQ[i * DP + cc]);
        atomicAdd(a.dk + qk + cc, fmaf(ge, bb, gK[i * DP + cc]));
        const float dlog = gG[i * DP + cc];
        const float da = lg ? dlog * (1.f - al) : dlog / al;   // d/dα of log α = 1/α; d/dx of log σ(x) = 1 − σ
        const float db_ = ge * k;
        if (alpha_pc) atomicAdd(a.dalpha + gr * D + cc, da);
        else sa += dlog;
        if (full) atomicAdd(a.db + gr * D + cc, db_ * (lg ? bb * (1.f - bb) : 1.f));
        else sb += db_;
      }
      if (!alpha_pc || !full) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          sa += __shfl_xor_sync(0xffffffffu, sa, off);
          sb += __shfl_xor_sync(0xffffffffu, sb, off);
        }
        if (lane == 0) {
          if (!alpha_pc) {
            const float al = sAl[i * DP];
            atomicAdd(a.dalpha + gr, lg ? sa * (1.f - al) : sa / al);
          }
          if (!full) {
            const float beta = sB[i * DP];
            atomicAdd(a.db + gr, sb * (lg ? beta * (1.f - beta) : 1.f));
          }
        }
      }
    }
    float* tmp = dSp;
    dSp = dSn;
    dSn = tmp;
  }
  __syncthreads();
  if (a.dS0) {
    for (int idx = tid; idx < D * DVT; idx += BT) {
      const int r = idx / DVT, v = idx % DVT;
      a.dS0[((size_t)bh * D + r) * D + col0 + v] = dSp[r * VP + v];
    }
  }
}

template <int D, typename TIn, typename TdO>
cudaError_t launch_bwd_t(const BwdArgs& a, cudaStream_t st) {
  using L = BwdSmem<D>;
  const int grid = a.B * a.Hv * (D / L::DVT);
  if (grid == 0) return cudaSuccess;
  auto kfn = chunk_bwd_kernel<D, TIn, TdO>;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
  if (e != cudaSuccess) return e;
  kfn<<<grid, BT, L::bytes, st>>>(a);
  return cudaGetLastError();
}

template <typename TIn, typename TdO>
cudaError_t launch_bwd_d(const BwdArgs& a, int d, cudaStream_t st) {
  switch (d) {
    case 16: return launch_bwd_t<16, TIn, TdO>(a, st);
    case 32: return launch_bwd_t<32, TIn, TdO>(a, st);
    case 64: return launch_bwd_t<64, TIn, TdO>(a, st);
    case 128: return launch_bwd_t<128, TIn, TdO>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t chunk_bwd_workspace(int n_states, int H_v, int T, int d) {
  return (size_t)n_states * H_v * (size_t)((T + BC - 1) / BC) * d * d * sizeof(float);
}

cudaError_t launch_chunk_bwd(const BwdArgs& a, int d, int qkv_bf16, int do_bf16, cudaStream_t st) {
  if (qkv_bf16)
    return do_bf16 ? launch_bwd_d<__nv_bfloat16, __nv_bfloat16>(a, d, st) : launch_bwd_d<__nv_bfloat16, float>(a, d, st);
  return do_bf16 ? launch_bwd_d<float, __nv_bfloat16>(a, d, st) : launch_bwd_d<float, float>(a, d, st);
}

}  // namespace gdn2
