// Fused recurrent decode step of the Gated DeltaNet-2 recurrence (one token).
//
// Per (sequence, value head) — "Resumo Técnico: Gated DeltaNet-2", Metodologia
// §1, and the fused recurrent schedule of "Uma análise das variantes de
// atenção linear da família DeltaNet", section "Kernel Triton recorrente
// fundido para decode":
//     S̄ = Diag(α) S                 (decay)
//     r = S̄ᵀ e,  p = S̄ᵀ q            (key-read and query-read reductions)
//     u = z − r                     (residual)
//     S ← S̄ + k uᵀ                  (outer-product write)
//     o = s (p + (kᵀq) u)           (= s·Sᵀq after the write)
// with e = b ⊙ k, z = w ⊙ v. Both reductions run on the decayed state in the
// same register pass, so the state is read from HBM once and written once.
//
// With the depthwise causal conv (kernel 4, "Gated DeltaNet: o mixer em 48
// das 64 camadas", Conceito) the step convolves its q, k, v channels with the
// three previous inputs held in the caller's conv history, normalises q, k
// after the conv when asked, and writes the shifted history to a second
// buffer (never the one it reads, since several CTAs read each q, k channel).
// The q, k channels of a QK head are written by the CTA of its first value
// head and first column tile; each CTA writes its own v channels.
//
// Work split: one CTA per (sequence, value head, tile of COLS value columns).
// Thread (cg, rg) owns 4 consecutive columns (one float4) of rows
// rg, rg+16, rg+32, ...: a warp instruction covers whole 4·COLS-byte row
// segments, so every state access is a coalesced 128-bit load/store. The
// state is streamed (evict-first) because it is far larger than L2.

#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kRowGroups = 16;

template <int D, int COLS, typename TIn, typename TOut, bool LG, bool CONV>
__global__ void __launch_bounds__((COLS / 4) * kRowGroups, 4)
decode_kernel(DecodeArgs a) {
  constexpr int CG = COLS / 4;            // column groups (float4 each)
  constexpr int NT = CG * kRowGroups;     // threads
  constexpr int RPT = D / kRowGroups;     // rows per thread
  constexpr int NW = NT / 32;             // warps
  constexpr int TILES = D / COLS;
  static_assert(NT % 32 == 0 && RPT >= 1, "bad decode tiling");

  const int tile = blockIdx.x % TILES;
  const int bh = blockIdx.x / TILES;      // b * Hv + h
  const int h = bh % a.Hv;
  const int bi = bh / a.Hv;
  const int hq = h / (a.Hv / a.Hqk);
  const size_t bg = (size_t)bi * a.Hg + (a.Hg == a.Hv ? h : hq);   // row of alpha, b
  const int tid = threadIdx.x;
  const int cg = tid % CG;
  const int rg = tid / CG;
  const int col0 = tile * COLS;

  __shared__ float s_q[D], s_k[D], s_a[D], s_e[D];
  __shared__ float s_z[COLS];
  __shared__ float s_red[2][NW][COLS];
  __shared__ float s_u[COLS];
  __shared__ float s_scalar[4];           // |q|⁻¹, |k|⁻¹, kᵀq

  float4* Sg = reinterpret_cast<float4*>(a.S + (size_t)bh * D * D + col0) + cg;
  float4 st[RPT];

  // Per-token vectors into shared memory (fp32). Every small load of the
  // step (q, k, v, their conv taps and history, the gates) is issued before
  // the state loads, so that none of them waits behind the state stream and
  // no load depends on another.
  const TIn* qg = static_cast<const TIn*>(a.q) + ((size_t)bi * a.Hqk + hq) * D;
  const TIn* kg = static_cast<const TIn*>(a.k) + ((size_t)bi * a.Hqk + hq) * D;
  const TIn* vg = static_cast<const TIn*>(a.v) + (size_t)bh * D + col0;
  // Conv history rows [B, 3, channels]; channel offsets of q, k and v.
  const size_t ctot = (size_t)(2 * a.Hqk + a.Hv) * D;
  const size_t hbase = (size_t)bi * 3 * ctot;
  const size_t cq = (size_t)hq * D, ck = (size_t)(a.Hqk + hq) * D, cv = (size_t)2 * a.Hqk * D + (size_t)h * D + col0;
  const TIn* hin = static_cast<const TIn*>(a.conv_in);
  const TIn zero = from_f32<TIn>(0.f);
  // y = Σ_j W[ch][j] x_{t−3+j}; the channel's history rows 1, 2 and its input
  // are kept (in `keep`) for the shifted history written at the end
  // (loads of conv1: the taps, the history rows, the input)
  struct ConvIn {
    float4 wt;
    TIn h0, h1, h2, x;
  };
  auto conv_load = [&](const TIn* xp, size_t ch) -> ConvIn {
    ConvIn c;
    c.x = *xp;
    c.wt = __ldg(reinterpret_cast<const float4*>(a.conv_w) + ch);
    c.h0 = c.h1 = c.h2 = zero;
    if (hin) {
      const TIn* hp = hin + hbase + ch;
      c.h0 = hp[0];
      c.h1 = hp[ctot];
      c.h2 = hp[2 * ctot];
    }
    return c;
  };
  auto conv1 = [&](const ConvIn& c, TIn* keep) -> float {
    keep[0] = c.h1;
    keep[1] = c.h2;
    keep[2] = c.x;
    return c.wt.x * to_f32(c.h0) + c.wt.y * to_f32(c.h1) + c.wt.z * to_f32(c.h2) + c.wt.w * to_f32(c.x);
  };
  // the shifted history of the channels this thread convolved (written after
  // the state: nothing in the step waits for it)
  constexpr int KQ = (2 * D + NT - 1) / NT;        // q, k channels per thread
  TIn keep_qk[KQ][3], keep_v[3];
  // this thread's channels: q/k channel tid + m·NT of the 2·D (q first;
  // warp-uniform halves, so each thread waits for one channel's loads),
  // α and b channels tid, tid + NT, ..., v channel tid < COLS
  static_assert(COLS <= NT, "one v channel per thread at most");
  ConvIn cin_qk[KQ], cin_v;
  float xqk[KQ], av[(D + NT - 1) / NT], bv[(D + NT - 1) / NT];
#pragma unroll
  for (int m = 0; m < KQ; ++m) {
    const int i = tid + m * NT;
    if (i < 2 * D) {
      const bool isq = i < D;
      const int c = isq ? i : i - D;
      if (CONV) cin_qk[m] = conv_load((isq ? qg : kg) + c, (isq ? cq : ck) + c);
      else xqk[m] = to_f32((isq ? qg : kg)[c]);
    }
  }
  const bool full = a.gate_mode == GDN2_GATES_FULL;
#pragma unroll
  for (int m = 0; m * NT < D; ++m) {
    const int i = tid + m * NT;
    if (i < D) {
      av[m] = gate_at<LG>(a.alpha, (a.gate_mode == GDN2_GATES_GDN) ? bg : bg * D + i);
      bv[m] = full ? gate_at<LG>(a.b, bg * D + i) : 0.f;
    }
  }
  const float beta = full ? 0.f : gate_at<LG>(a.b, bg);
  float wj = 0.f, vx = 0.f;
  if (tid < COLS) {
    wj = full ? gate_at<LG>(a.w, (size_t)bh * D + col0 + tid) : beta;
    if (CONV) cin_v = conv_load(vg + tid, cv + tid);
    else vx = to_f32(vg[tid]);
  }
  // The state loads: the HBM-heavy traffic.
#pragma unroll
  for (int i = 0; i < RPT; ++i) st[i] = __ldcs(Sg + (size_t)(rg + kRowGroups * i) * (D / 4));

#pragma unroll
  for (int m = 0; m < KQ; ++m) {
    const int i = tid + m * NT;
    if (i < 2 * D) (i < D ? s_q : s_k)[i < D ? i : i - D] = CONV ? conv1(cin_qk[m], keep_qk[m]) : xqk[m];
  }
#pragma unroll
  for (int m = 0; m * NT < D; ++m) {
    const int i = tid + m * NT;
    if (i < D) s_a[i] = av[m];
  }
  if (tid < COLS) s_z[tid] = wj * (CONV ? conv1(cin_v, keep_v) : vx);
  __syncthreads();
  if (tid < 32) {
    float sq = 0.f, sk = 0.f, kq = 0.f;
    for (int i = tid; i < D; i += 32) {
      sq += s_q[i] * s_q[i];
      sk += s_k[i] * s_k[i];
      kq += s_k[i] * s_q[i];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      sq += __shfl_xor_sync(0xffffffffu, sq, off);
      sk += __shfl_xor_sync(0xffffffffu, sk, off);
      kq += __shfl_xor_sync(0xffffffffu, kq, off);
    }
    if (tid == 0) {
      float iq = 1.f, ik = 1.f;
      if (a.l2norm) {
        iq = rsqrtf(sq + kL2Eps);
        ik = rsqrtf(sk + kL2Eps);
      }
      s_scalar[0] = iq;
      s_scalar[1] = ik;
      s_scalar[2] = kq * iq * ik;
    }
  }
  __syncthreads();
  const float iq = s_scalar[0], ik = s_scalar[1], kq = s_scalar[2];
#pragma unroll
  for (int m = 0; m * NT < D; ++m) {
    const int i = tid + m * NT;
    if (i < D) s_e[i] = (full ? bv[m] : beta) * (s_k[i] * ik);
  }
  __syncthreads();

  // Decay and both reductions over the thread's rows.
  float r[4] = {0.f, 0.f, 0.f, 0.f}, p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int row = rg + kRowGroups * i;
    const float al = s_a[row];
    st[i].x *= al; st[i].y *= al; st[i].z *= al; st[i].w *= al;
    const float er = s_e[row], qr = s_q[row] * iq;
    r[0] += st[i].x * er; r[1] += st[i].y * er; r[2] += st[i].z * er; r[3] += st[i].w * er;
    p[0] += st[i].x * qr; p[1] += st[i].y * qr; p[2] += st[i].z * qr; p[3] += st[i].w * qr;
  }
  // Reduce across the row groups that share a warp (lanes cg + CG·m).
#pragma unroll
  for (int off = CG; off < 32; off <<= 1) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      r[c] += __shfl_xor_sync(0xffffffffu, r[c], off);
      p[c] += __shfl_xor_sync(0xffffffffu, p[c], off);
    }
  }
  const int lane = tid & 31, warp = tid >> 5;
  if (lane < CG) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      s_red[0][warp][cg * 4 + c] = r[c];
      s_red[1][warp][cg * 4 + c] = p[c];
    }
  }
  __syncthreads();
  if (tid < COLS) {
    float rr = 0.f, pp = 0.f;
#pragma unroll
    for (int w_ = 0; w_ < NW; ++w_) {
      rr += s_red[0][w_][tid];
      pp += s_red[1][w_][tid];
    }
    const float u = s_z[tid] - rr;
    s_u[tid] = u;
    TOut* og = static_cast<TOut*>(a.o) + (size_t)bh * D + col0;
    og[tid] = from_f32<TOut>(a.scale * (pp + kq * u));
  }
  __syncthreads();

  // Write S ← S̄ + k uᵀ.
  const float u0 = s_u[cg * 4 + 0], u1 = s_u[cg * 4 + 1], u2 = s_u[cg * 4 + 2], u3 = s_u[cg * 4 + 3];
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int row = rg + kRowGroups * i;
    const float kr = s_k[row] * ik;
    float4 x = st[i];
    x.x += kr * u0; x.y += kr * u1; x.z += kr * u2; x.w += kr * u3;
    __stcs(Sg + (size_t)row * (D / 4), x);
  }
  if (CONV && a.conv_out) {
    // Shifted history: rows 1, 2 of the incoming history, then this token.
    // The q, k channels of a QK head are written by the CTA of its first
    // value head and first column tile; every CTA writes its v channels.
    TIn* hout = static_cast<TIn*>(a.conv_out);
    auto shift = [&](size_t ch, const TIn* kp) {
      hout[hbase + ch] = kp[0];
      hout[hbase + ctot + ch] = kp[1];
      hout[hbase + 2 * ctot + ch] = kp[2];
    };
    if (tile == 0 && h % (a.Hv / a.Hqk) == 0) {
#pragma unroll
      for (int m = 0; m < KQ; ++m) {
        const int i = tid + m * NT;
        if (i < 2 * D) shift(i < D ? cq + i : ck + (i - D), keep_qk[m]);
      }
    }
    if (tid < COLS) shift(cv + tid, keep_v);
  }
}

template <int D, int COLS, typename TIn, typename TOut>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t s) {
  const int grid = a.B * a.Hv * (D / COLS);
  if (grid == 0) return cudaSuccess;
  constexpr int NT = (COLS / 4) * kRowGroups;
  const bool conv = a.conv_w != nullptr;
  if (a.gate_logits)
    (conv ? decode_kernel<D, COLS, TIn, TOut, true, true> : decode_kernel<D, COLS, TIn, TOut, true, false>)
        <<<grid, NT, 0, s>>>(a);
  else
    (conv ? decode_kernel<D, COLS, TIn, TOut, false, true> : decode_kernel<D, COLS, TIn, TOut, false, false>)
        <<<grid, NT, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t s) {
  switch (a.d) {
    case 16: return launch_t<16, 16, TIn, TOut>(a, s);
    case 32: return launch_t<32, 32, TIn, TOut>(a, s);
    case 64: return launch_t<64, 64, TIn, TOut>(a, s);
    case 128: return launch_t<128, 64, TIn, TOut>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, int qkv_bf16, int o_bf16, cudaStream_t s) {
  if (qkv_bf16) {
    return o_bf16 ? launch_d<__nv_bfloat16, __nv_bfloat16>(a, s) : launch_d<__nv_bfloat16, float>(a, s);
  }
  return o_bf16 ? launch_d<float, __nv_bfloat16>(a, s) : launch_d<float, float>(a, s);
}

}  // namespace gdn2
