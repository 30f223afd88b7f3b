// Chunked prefill in fp32 SIMT arithmetic (the precise path).
//
// Chunk algebra ("Uma análise das variantes de atenção linear da família
// DeltaNet", section "Chunkwise KDA", generalised to the decoupled gates of
// "Resumo Técnico: Gated DeltaNet-2", Metodologia §3). Inside a chunk of C
// tokens with entry state S, let G_i = Σ_{j≤i} log α_j (per key channel,
// from the chunk start) and γ_i = exp(G_i). Unrolling the token loop gives
//     u_i = z_i − S̄_iᵀ e_i
//         = z_i − Sᵀ(γ_i ⊙ e_i) − Σ_{j<i} T_ij u_j,
//     T_ij = Σ_c e_ic k_jc exp(G_ic − G_jc)                    (j < i)
// so (I + T) U = Z − Ē S with Ē_i = γ_i ⊙ e_i: a unit-lower-triangular solve.
// Then
//     O = s (Q̄ S + A_qk U),  Q̄_i = γ_i ⊙ q_i,
//         A_qk,ij = Σ_c q_ic k_jc exp(G_ic − G_jc)             (j ≤ i)
//     S ← Diag(γ_C) S + K_endᵀ U,  K_end,j = k_j ⊙ exp(G_C − G_j).
// This kernel evaluates every exp(G_i − G_j) pairwise (exponent ≤ 0, so no
// overflow for any α ∈ (0,1]) and keeps everything in fp32.
//
// One CTA per (sequence, value head, tile of DVT value columns): the value
// columns of S evolve independently once T and A_qk are known, so tiles of
// the same head run in parallel and recompute only the C×C matrices.

#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kCMax = 64;
constexpr int kThreads = 256;

template <int D, int DVT>
struct SimtSmem {
  static constexpr int DP = D + 1;        // padded row stride of [C][D] arrays
  static constexpr int CP = kCMax + 1;    // padded row stride of [C][C] arrays
  static constexpr size_t floats =
      5 * (size_t)kCMax * DP + (size_t)D * DVT + 2 * (size_t)kCMax * CP + 2 * (size_t)kCMax * DVT + D;
  static constexpr size_t bytes = floats * sizeof(float);
};

template <typename TIn>
__device__ __forceinline__ float load_conv(const TIn* base, size_t tok_stride, int t, const float* wrow,
                                           bool conv, const TIn* hist, size_t hist_stride) {
  // base points at token 0 of this channel; tok_stride is the element stride
  // between consecutive tokens. hist (or NULL: zeros) points at row 0 of the
  // channel's history, whose row 3 + t holds the input of token t < 0.
  if (!conv) return to_f32(base[(size_t)t * tok_stride]);
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int src = t - 3 + j;
    if (src >= 0) acc += wrow[j] * to_f32(base[(size_t)src * tok_stride]);
    else if (hist) acc += wrow[j] * to_f32(hist[(size_t)(3 + src) * hist_stride]);
  }
  return acc;
}

template <int D, int DVT, typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads) chunk_simt_kernel(ChunkArgs a) {
  using L = SimtSmem<D, DVT>;
  constexpr int DP = L::DP, CP = L::CP;
  constexpr int TILES = D / DVT;
  constexpr int NWARP = kThreads / 32;
  constexpr int CPW = DVT / NWARP;        // solve: columns per warp
  constexpr int JG = 32 / CPW;            // solve: lanes sharing one column
  static_assert(DVT % NWARP == 0 && 32 % CPW == 0, "bad solve tiling");

  extern __shared__ float smem[];
  float* sk = smem;                        // [C][DP] k, later K_end
  float* sq = sk + kCMax * DP;             // [C][DP] q, later Q̄
  float* se = sq + kCMax * DP;             // [C][DP] b, then e, later Ē
  float* sG = se + kCMax * DP;             // [C][DP] log α, then cumulative G
  float* sS = sG + kCMax * DP;             // [D][DVT] state tile
  float* sT = sS + D * DVT;                // [C][CP] strict lower T
  float* sA = sT + kCMax * CP;             // [C][CP] lower-incl A_qk
  float* sz = sA + kCMax * CP;             // [C][DVT] z, then W, then U
  float* sP = sz + kCMax * DVT;            // [C][DVT] Q̄ S
  float* sgC = sP + kCMax * DVT;           // [D] γ_C
  float* sGl = sgC + D;                    // [C][DP] low part of G (G = sG + sGl)

  const int tile = blockIdx.x % TILES;
  const int bh = blockIdx.x / TILES;
  const int h = bh % a.Hv;
  const int bi = bh / a.Hv;
  const int hq = h / (a.Hv / a.Hqk);
  const int hg = a.Hg == a.Hv ? h : hq;     // head of alpha and b
  const int col0 = tile * DVT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = a.chunk;
  const bool conv = a.conv_w != nullptr;
  const int mode = a.gate_mode;

  const TIn* qg = static_cast<const TIn*>(a.q);
  const TIn* kg = static_cast<const TIn*>(a.k);
  const TIn* vg = static_cast<const TIn*>(a.v);
  TOut* og = static_cast<TOut*>(a.o);
  const size_t qk_tok = (size_t)a.Hqk * D;   // element stride between tokens of q/k
  const size_t v_tok = (size_t)a.Hv * D;
  const float* wq = conv ? a.conv_w + (size_t)(hq * D) * 4 : nullptr;
  const float* wk = conv ? a.conv_w + (size_t)(a.Hqk * D + hq * D) * 4 : nullptr;
  const float* wv = conv ? a.conv_w + (size_t)(2 * a.Hqk * D + h * D) * 4 : nullptr;
  const size_t hstride = 2 * qk_tok + v_tok;   // channels of the conv history rows
  const TIn* hist = static_cast<const TIn*>(a.conv_in);
  const TIn* hq_ = hist ? hist + (size_t)bi * 3 * hstride + (size_t)hq * D : nullptr;
  const TIn* hk_ = hist ? hist + (size_t)bi * 3 * hstride + qk_tok + (size_t)hq * D : nullptr;
  const TIn* hv_ = hist ? hist + (size_t)bi * 3 * hstride + 2 * qk_tok + (size_t)h * D + col0 : nullptr;

  // Entry state tile.
  for (int idx = tid; idx < D * DVT; idx += kThreads) {
    const int r = idx / DVT, c = idx % DVT;
    sS[idx] = a.S0 ? a.S0[((size_t)bh * D + r) * D + col0 + c] : 0.f;
  }

  const size_t tok0 = seq_tok0(a, bi);     // first token of the sequence in the buffers
  const int Tn = seq_len(a, bi);
  const int nchunks = (Tn + C - 1) / C;
  for (int ck = 0; ck < nchunks; ++ck) {
    const int t0 = ck * C;
    const int Lc = min(C, Tn - t0);
    __syncthreads();

    // 1. Load q, k, log α, b (key side) and z = w ⊙ v (value tile).
    for (int idx = tid; idx < C * D; idx += kThreads) {
      const int i = idx / D, c = idx % D;
      float qv = 0.f, kv = 0.f, gv = 0.f, bv = 0.f;
      if (i < Lc) {
        const int t = t0 + i;
        const size_t qk0 = tok0 * qk_tok + (size_t)hq * D + c;
        qv = load_conv(qg + qk0, qk_tok, t, conv ? wq + c * 4 : nullptr, conv, hq_ ? hq_ + c : nullptr, hstride);
        kv = load_conv(kg + qk0, qk_tok, t, conv ? wk + c * 4 : nullptr, conv, hk_ ? hk_ + c : nullptr, hstride);
        const size_t gt = (tok0 + t) * a.Hg + hg;   // row of alpha, b
        const size_t ai = mode == GDN2_GATES_GDN ? gt : gt * D + c;
        gv = a.gate_logits ? log_sigmoid_f32(__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.alpha)[ai]))
                           : logf(a.alpha[ai]);
        bv = gate_at(a.b, (mode == GDN2_GATES_FULL) ? gt * D + c : gt, a.gate_logits);
      }
      sq[i * DP + c] = qv;
      sk[i * DP + c] = kv;
      sG[i * DP + c] = gv;
      se[i * DP + c] = bv;
    }
    for (int idx = tid; idx < C * DVT; idx += kThreads) {
      const int i = idx / DVT, c = idx % DVT;
      float zv = 0.f;
      if (i < Lc) {
        const int t = t0 + i;
        const size_t gt = (tok0 + t) * a.Hv + h;     // row of w
        const size_t gtb = (tok0 + t) * a.Hg + hg;   // row of b (= β, tied modes)
        const float vv = load_conv(vg + tok0 * v_tok + (size_t)h * D + col0 + c, v_tok, t,
                                   conv ? wv + (col0 + c) * 4 : nullptr, conv, hv_ ? hv_ + c : nullptr, hstride);
        const float wv_ = (mode == GDN2_GATES_FULL) ? gate_at(a.w, gt * D + col0 + c, a.gate_logits)
                                                    : gate_at(a.b, gtb, a.gate_logits);
        zv = wv_ * vv;
      }
      sz[i * DVT + c] = zv;
    }
    __syncthreads();

    // 2. Optional L2 norm of q, k (after the conv); e = b ⊙ k.
    for (int i = warp; i < C; i += NWARP) {
      float iq = 1.f, ik = 1.f;
      if (a.l2norm) {
        float ssq = 0.f, ssk = 0.f;
        for (int c = lane; c < D; c += 32) {
          ssq += sq[i * DP + c] * sq[i * DP + c];
          ssk += sk[i * DP + c] * sk[i * DP + c];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
          ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
        }
        iq = rsqrtf(ssq + kL2Eps);
        ik = rsqrtf(ssk + kL2Eps);
      }
      for (int c = lane; c < D; c += 32) {
        const float kk = sk[i * DP + c] * ik;
        sk[i * DP + c] = kk;
        sq[i * DP + c] *= iq;
        se[i * DP + c] *= kk;
      }
    }
    // 3. Cumulative log decay per key channel, summed in double and kept as
    // a float pair (hi + lo): after a run of strong decay |G| is large, and a
    // difference G_i − G_j of two single floats would lose the small
    // exponent that tokens after that run need.
    if (tid < D) {
      double acc = 0.0;
      for (int i = 0; i < C; ++i) {
        acc += (double)sG[i * DP + tid];
        const float hi = (float)acc;
        sG[i * DP + tid] = hi;
        sGl[i * DP + tid] = (float)(acc - (double)hi);
      }
    }
    __syncthreads();

    // 4. T (strict lower) and A_qk (lower incl. diagonal), pairwise decays.
    for (int i = warp; i < C; i += NWARP) {
      for (int j = lane; j < C; j += 32) {
        float tv = 0.f, av = 0.f;
        if (j <= i) {
          for (int c = 0; c < D; ++c) {
            const float dec = expf((sG[i * DP + c] - sG[j * DP + c]) + (sGl[i * DP + c] - sGl[j * DP + c]));
            const float kd = sk[j * DP + c] * dec;
            tv += se[i * DP + c] * kd;
            av += sq[i * DP + c] * kd;
          }
        }
        sT[i * CP + j] = (j < i) ? tv : 0.f;
        sA[i * CP + j] = av;
      }
    }
    __syncthreads();
    // 4b. Absorb the decay: Ē = γ ⊙ e, Q̄ = γ ⊙ q, K_end = k ⊙ exp(G_C − G), γ_C.
    for (int idx = tid; idx < C * D; idx += kThreads) {
      const int i = idx / D, c = idx % D;
      const float G = sG[i * DP + c], Gl = sGl[i * DP + c];
      const float Gc = sG[(C - 1) * DP + c], Gcl = sGl[(C - 1) * DP + c];
      const float g = expf(G + Gl);
      se[i * DP + c] *= g;
      sq[i * DP + c] *= g;
      sk[i * DP + c] *= expf((Gc - G) + (Gcl - Gl));
    }
    if (tid < D) sgC[tid] = expf(sG[(C - 1) * DP + tid] + sGl[(C - 1) * DP + tid]);
    __syncthreads();

    // 5. W = Z − Ē S and P = Q̄ S for the tile.
    for (int idx = tid; idx < C * DVT; idx += kThreads) {
      const int i = idx / DVT, c = idx % DVT;
      float ws = 0.f, ps = 0.f;
      for (int r = 0; r < D; ++r) {
        const float s = sS[r * DVT + c];
        ws += se[i * DP + r] * s;
        ps += sq[i * DP + r] * s;
      }
      sz[i * DVT + c] -= ws;
      sP[i * DVT + c] = ps;
    }
    __syncthreads();

    // 6. Forward substitution (I + T) U = W, each warp owning CPW columns.
    {
      const int c = warp * CPW + lane / JG;
      const int jg = lane % JG;
      for (int i = 1; i < C; ++i) {
        float acc = 0.f;
        for (int j = jg; j < i; j += JG) acc += sT[i * CP + j] * sz[j * DVT + c];
#pragma unroll
        for (int off = 1; off < JG; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (jg == 0) sz[i * DVT + c] -= acc;
        __syncwarp();
      }
    }
    __syncthreads();

    // 7. Outputs O = s (P + A_qk U).
    for (int idx = tid; idx < C * DVT; idx += kThreads) {
      const int i = idx / DVT, c = idx % DVT;
      if (i >= Lc) continue;
      float acc = sP[i * DVT + c];
      for (int j = 0; j <= i; ++j) acc += sA[i * CP + j] * sz[j * DVT + c];
      og[((tok0 + t0 + i) * a.Hv + h) * D + col0 + c] = from_f32<TOut>(a.scale * acc);
    }
    // 8. State S ← Diag(γ_C) S + K_endᵀ U.
    for (int idx = tid; idx < D * DVT; idx += kThreads) {
      const int r = idx / DVT, c = idx % DVT;
      float acc = sgC[r] * sS[idx];
      for (int j = 0; j < C; ++j) acc += sk[j * DP + r] * sz[j * DVT + c];
      sS[idx] = acc;
    }
  }
  __syncthreads();
  if (a.ST) {
    for (int idx = tid; idx < D * DVT; idx += kThreads) {
      const int r = idx / DVT, c = idx % DVT;
      a.ST[((size_t)bh * D + r) * D + col0 + c] = sS[idx];
    }
  }
}

template <int D, int DVT, typename TIn, typename TOut>
cudaError_t launch_t(const ChunkArgs& a, cudaStream_t s) {
  using L = SimtSmem<D, DVT>;
  const int grid = a.B * a.Hv * (D / DVT);
  if (grid == 0) return cudaSuccess;
  auto kfn = chunk_simt_kernel<D, DVT, TIn, TOut>;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
  if (e != cudaSuccess) return e;
  kfn<<<grid, kThreads, L::bytes, s>>>(a);
  return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_d(const ChunkArgs& a, cudaStream_t s) {
  switch (a.dk) {
    case 16: return launch_t<16, 16, TIn, TOut>(a, s);
    case 32: return launch_t<32, 32, TIn, TOut>(a, s);
    case 64: return launch_t<64, 32, TIn, TOut>(a, s);
    case 128: return launch_t<128, 32, TIn, TOut>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs& a, int qkv_bf16, int o_bf16, cudaStream_t s) {
  if (qkv_bf16) {
    return o_bf16 ? launch_d<__nv_bfloat16, __nv_bfloat16>(a, s) : launch_d<__nv_bfloat16, float>(a, s);
  }
  return o_bf16 ? launch_d<float, __nv_bfloat16>(a, s) : launch_d<float, float>(a, s);
}

}  // namespace gdn2
