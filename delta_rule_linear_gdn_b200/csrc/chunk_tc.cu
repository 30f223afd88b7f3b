// Chunked prefill on the sm_100a tensor cores (tcgen05 + TMEM), 16-bit operands,
// fp32 accumulation and fp32 state. d_k = d_v = 128, chunk C = 64.
//
// Algebra ("Uma análise das variantes de atenção linear da família DeltaNet",
// section "Chunkwise KDA", with the decoupled erase/write gates of "Resumo
// Técnico: Gated DeltaNet-2", Metodologia §3: the per-channel decay is
// absorbed into the erase factor Ē and the write side Z = w ⊙ v, and the
// chunk is resolved by a unit-lower-triangular (I + T)⁻¹). For a chunk with
// entry state S (d_k × d_v) and γ_i = Π_{s≤i} α_s (per key channel, from the
// chunk start):
//     T_ij  = Σ_c e_ic k_jc Π_{j<s≤i} α_sc      (j < i),   e = b ⊙ k
//     Aqk_ij = Σ_c q_ic k_jc Π_{j<s≤i} α_sc     (j ≤ i)
//     A     = (I + T)⁻¹
//     Y = A Ē (Ē_i = γ_i ⊙ e_i),   U_w = A Z
//     U = U_w − Y S
//     O = s (Q̄ S + Aqk U),        Q̄_i = γ_i ⊙ q_i
//     S ← Diag(γ_C) S + K_endᵀ U,  K_end,j = k_j ⊙ Π_{j<s≤C} α_s
//
// Two kernels, following the pages' split between the parallel intra-chunk
// work and the single inter-chunk sweep ("Pipeline Triton da versão por
// chunks"):
//   * prep: one CTA per (chunk, sequence, value head), all in parallel. It
//     builds T and Aqk (tensor cores), inverts I + T (fp32), forms Yᵀ and U_wᵀ
//     (tensor cores) and writes the chunk's scan operands — Yᵀ, U_wᵀ, Q̄, K_end,
//     Aqk as fp16 tiles already in the MMA shared-memory layout, and γ_C — to
//     one 73 KB workspace slot.
//   * scan: one CTA per (sequence, value head) walks the chunks in order. It
//     streams the slots into shared memory with bulk copies (double-buffered,
//     chunk c+1 in flight while c computes) and runs
//         (Y S)ᵀ = Sᵀ Yᵀ,  Oᵀ = Sᵀ Q̄ᵀ,  Uᵀ = U_wᵀ − (Y S)ᵀ,
//         Sᵀ ← Sᵀ Γ + Uᵀ K_end,  Oᵀ += Uᵀ Aqkᵀ,
//     with the fp32 state Sᵀ resident in TMEM and an fp16 copy in shared
//     memory feeding the next chunk's MMAs.
// Everything is computed transposed so that every MMA has M = 128. All MMA
// operand tiles use the 128-byte-swizzled layout (see tc_prims.cuh), so that
// a warp writing or reading whole rows is free of bank conflicts.
//
// Decay factors of the Gram matrices. Π_{j<s≤i} α is split into two factors
// about a reference token so that one factor multiplies row i and the other
// row j (each product stays a GEMM):
//   * i, j in the same 32-token half: reference at the boundary of the half's
//     two 16-token quarters (factors are products over at most 16 tokens);
//   * i in the second half, j in the first: reference at the half boundary
//     (both factors ≤ 1).
// All factors are cumulative products of α (no exp/log); each element needs
// one reciprocal. This requires the product of α over any 16-token aligned
// quarter to stay above ~1e-37 per channel (α averaging ≥ 0.005); the fp32
// SIMT kernel has no such restriction.
//
// Operand precision. Every operand after the Gram step (Ē, Z, Q̄, K_end, A,
// Aqk, Y, U_w, U and the copy of S) is bounded in magnitude and is stored as
// fp16 (11-bit significand), eight times finer than bf16 at the same
// tensor-core rate; this keeps the chunked result within 2e-2 of the float64
// token loop. The Gram factors contain reciprocals of decay products and use
// fp16 when every quarter product of α exceeds 2^-14, bf16 (fp32 range)
// otherwise, chosen per chunk. The fp16 operands require |S| and |v| < 6e4.

#include <algorithm>

#include "common.cuh"
#include "tc_prims.cuh"

namespace gdn2 {
namespace {

using namespace tc;

constexpr int D = 128;            // d_k = d_v
constexpr int C = 64;             // chunk
constexpr int NT = 256;           // threads per CTA (8 warps)

// ------------------------------------------------------------------ workspace
// Word 0 of the workspace is the device status (nonzero: a wait gave up).
// Slots follow, one per (sequence, value head, chunk of the segment). Tiles
// are swizzled; "BS" is the byte stride between 64-column blocks.
constexpr size_t WS_HEAD = 256;
constexpr int SL_YT = 0;              // Yᵀ   fp16 [128 key][64 tok]   (MN-major B of (YS)ᵀ)
constexpr int SL_UW = 16384;          // U_wᵀ fp16 [128 dv][64 tok]
constexpr int SL_QB = 32768;          // Q̄    fp16 [64 tok][128 key]  BS 8192 (K-major B of Oᵀ)
constexpr int SL_KE = 49152;          // K_end fp16 [64 tok][128 key] BS 8192 (MN-major B of Sᵀ)
constexpr int SL_AQ = 65536;          // Aqk  fp16 [64 i][64 j]        (K-major B of Oᵀ)
constexpr int SL_GC = 73728;          // γ_C  fp32 [128]
constexpr int SLOT_USED = 74240;      // bytes copied per chunk
constexpr int SLOT = 74752;           // slot stride (1 KB multiple)
constexpr int BS_ROW128 = 16384;      // block stride of a 128-row tile
constexpr int BS_ROW64 = 8192;        // block stride of a 64-row tile

// ------------------------------------------------------------------ prep smem
// [0, 32K)   Gb: Gram boundary operand [Ē_bnd ; Q̄_bnd], 128 rows (32..63 and
//            96..127 used), BS 16K. Its rows 0..31 hold K̃_bnd (the Kb tile,
//            BS 16K) and its block-0 rows 64..95 ([8K, 12K)) hold the quarter
//            products; the MMA reads those rows as don't-care.
// [32K, 64K) Gm: [Ē_mid ; Q̄_mid], 128 rows, BS 16K
// [64K, 80K) Km: K̃_mid, 64 rows, BS 8K
// [80K, 96K) Ē (64 tok × 128 key, BS 8K)   [96K, 112K) Z (64 tok × 128 dv)
// Before pass 2, [32K, 66K) stages α for the cumulative products; after the
// Gram MMAs, [32K, 71K) holds the fp32 arrays of the inverse and [0, 8K) the
// fp16 A = (I+T)⁻¹ (64 × 64).
constexpr int P_GB = 0;
constexpr int P_KB = 0;
constexpr int P_PQ = 8192;            // quarter products [4][128] fp32
constexpr int P_RED = P_PQ + 4 * D * 4;
static_assert(P_RED + 64 <= 12288, "quarter products must stay in the unused Gram rows");
constexpr int P_GM = 32768;
constexpr int P_KM = 65536;
constexpr int P_EB = 81920;
constexpr int P_Z = 98304;
constexpr int P_END = 114688;
constexpr int SS = 132;               // α staging row stride (floats)
constexpr int P_STG = P_GM;
static_assert(P_STG + C * SS * 4 <= P_EB, "staging overlap");
constexpr int P_AINV = 0;
constexpr int TS = 68;                // fp32 row stride of T and its inverse
constexpr int P_T = P_GM;             // T   [64][68]
constexpr int P_I = P_T + C * TS * 4; // inv [64][68]
constexpr int P_X = P_I + C * TS * 4; // tmp [32][36]
static_assert(P_X + 32 * 36 * 4 <= P_EB, "prep smem overlap");
constexpr int P_BAR = P_END;
constexpr int P_TMEMP = P_BAR + 16;
constexpr int P_FLAG = P_TMEMP + 16;
constexpr int P_SMEM = P_FLAG + 16;
// prep TMEM columns
constexpr uint32_t PT_GM = 0, PT_GB = 64, PT_YT = 128, PT_UW = 192, PT_COLS = 256;

// ------------------------------------------------------------------ scan smem
constexpr int S_STAGE0 = 0;
constexpr int S_STAGE1 = SLOT;
constexpr int S_ST = 2 * SLOT;        // Sᵀ fp16 [128 dv][128 key], BS 16K
constexpr int S_UT = S_ST + D * D * 2;// Uᵀ fp16 [128 dv][64 tok]
constexpr int S_OS = S_UT + D * C * 2;// output staging, 16 KB of [rows][128] TOut
constexpr int S_BAR = S_OS + 16384;   // full[2], ys, st, o
constexpr int S_TMEMP = S_BAR + 48;
constexpr int S_FLAG = S_TMEMP + 16;
constexpr int S_SMEM = S_FLAG + 16;
constexpr uint32_t ST_S = 0, ST_YS = 128, ST_O = 192, ST_COLS = 512;   // Oᵀ double-buffered: 192, 256

__device__ __forceinline__ void st16(uint8_t* base, uint32_t off, uint4 v) {
  *reinterpret_cast<uint4*>(base + off) = v;
}
__device__ __forceinline__ void st8(uint8_t* base, uint32_t off, uint2 v) {
  *reinterpret_cast<uint2*>(base + off) = v;
}

__device__ __forceinline__ void unpack4_bf16(uint2 u, float* x) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
  const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
  x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
__device__ __forceinline__ void unpack8_f16(uint4 u, float* x) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// Key-side inputs of one token for 4 channels (coalesced: a warp reads whole
// rows), and the pointers and sizes needed to load them, passed by value.
struct KeyIn {
  uint2 k, q;              // bf16 × 4
  float4 b;                // fp32 × 4 (tied gates: β broadcast)
};
struct RowSrc {
  const __nv_bfloat16 *k, *q;
  const float* b;
  int T, Hqk, Hv, full_gates;
};

__device__ __forceinline__ void load_key_row(RowSrc r_, int bi, int t, int h, int hq, int c4, bool valid, KeyIn& r) {
  if (valid) {
    const size_t tq = ((size_t)bi * r_.T + t) * r_.Hqk + hq;
    const size_t gt = ((size_t)bi * r_.T + t) * r_.Hv + h;
    r.k = __ldg(reinterpret_cast<const uint2*>(r_.k + tq * D + c4));
    r.q = __ldg(reinterpret_cast<const uint2*>(r_.q + tq * D + c4));
    if (r_.full_gates) {
      r.b = __ldg(reinterpret_cast<const float4*>(r_.b + gt * D + c4));
    } else {
      const float beta = __ldg(r_.b + gt);
      r.b = make_float4(beta, beta, beta, beta);
    }
  } else {
    r.k = r.q = make_uint2(0, 0);
    r.b = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

__device__ __forceinline__ void wait_mma(uint64_t* bar, uint32_t& phase, int* sflag) {
  if (!mbar_wait(bar, phase)) atomicOr(sflag, 1);
  phase ^= 1u;
  fence_after_sync();
}

__device__ __forceinline__ void sync_for_mma() {
  fence_async_smem();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
}

// =============================================================================
// prep kernel: persistent, one 512-thread CTA per SM looping over the work
// items (chunk of the segment, sequence, value head). Each item's inputs are
// loaded in one round into registers; the next item's loads are issued as
// soon as the current item's elementwise pass has consumed its registers, so
// they arrive while the Gram, inverse and Yᵀ/U_wᵀ phases run.
// =============================================================================
constexpr int NP = 512;               // prep threads (16 warps)

// Inputs of one token for 4 channels (a warp reads whole rows).
struct TokIn {
  float4 al, b, w;
  uint2 k, q, v;
};
struct PrepSrc {
  const float *alpha, *b, *w;
  const __nv_bfloat16 *k, *q, *v;
  int T, Hqk, Hv, mode;
};

__device__ __forceinline__ void load_token(const PrepSrc& p, int bi, int t, int h, int hq, int c4, bool valid,
                                           TokIn& r) {
  if (valid) {
    const size_t gt = ((size_t)bi * p.T + t) * p.Hv + h;
    const size_t tq = ((size_t)bi * p.T + t) * p.Hqk + hq;
    if (p.mode == GDN2_GATES_GDN) {
      const float sa = __ldg(p.alpha + gt);
      r.al = make_float4(sa, sa, sa, sa);
    } else {
      r.al = __ldg(reinterpret_cast<const float4*>(p.alpha + gt * D + c4));
    }
    if (p.mode == GDN2_GATES_FULL) {
      r.b = __ldg(reinterpret_cast<const float4*>(p.b + gt * D + c4));
      r.w = __ldg(reinterpret_cast<const float4*>(p.w + gt * D + c4));
    } else {
      const float beta = __ldg(p.b + gt);
      r.b = r.w = make_float4(beta, beta, beta, beta);
    }
    r.k = __ldg(reinterpret_cast<const uint2*>(p.k + tq * D + c4));
    r.q = __ldg(reinterpret_cast<const uint2*>(p.q + tq * D + c4));
    r.v = __ldg(reinterpret_cast<const uint2*>(p.v + gt * D + c4));
  } else {
    r.al = make_float4(1.f, 1.f, 1.f, 1.f);
    r.b = r.w = make_float4(0.f, 0.f, 0.f, 0.f);
    r.k = r.q = r.v = make_uint2(0, 0);
  }
}

struct Item {
  int bh, cl, h, bi, hq, t0, Lc;
};
__device__ __forceinline__ Item decode_item(const ChunkArgs& a, int c_begin, int item) {
  Item it;
  it.bh = item % (a.B * a.Hv);      // value head fastest: heads sharing q, k run together
  it.cl = item / (a.B * a.Hv);
  it.h = it.bh % a.Hv;
  it.bi = it.bh / a.Hv;
  it.hq = it.h / (a.Hv / a.Hqk);
  it.t0 = (c_begin + it.cl) * C;
  it.Lc = min(C, a.T - it.t0);
  return it;
}

__global__ void __launch_bounds__(NP, 1) chunk_prep_kernel(ChunkArgs a, int c_begin, int n_seg) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + P_BAR);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + P_TMEMP);
  int* sflag = reinterpret_cast<int*>(smem + P_FLAG);
  float* sPq = reinterpret_cast<float*>(smem + P_PQ);
  float* sred = reinterpret_cast<float*>(smem + P_RED);
  float* stage = reinterpret_cast<float*>(smem + P_STG);
  float* sT = reinterpret_cast<float*>(smem + P_T);
  float* sI = reinterpret_cast<float*>(smem + P_I);
  float* sX = reinterpret_cast<float*>(smem + P_X);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = a.B * a.Hv * n_seg;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    *sflag = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, PT_COLS);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_ptr;
  const int lq = warp & 3;                       // TMEM lane quarter of this warp
  const uint32_t t_lane = tmem + ((uint32_t)(lq * 32) << 16);
  const int row = lq * 32 + lane;
  const int cgp = warp >> 2;                     // column group (0..3) among warps of a lane quarter

  // Element mapping: lane → 4 channels c4..c4+3 (a warp covers a whole row),
  // warp w → token w + 16 j of quarter j (j = 0..3).
  const int c4 = lane * 4;
  // Swizzled offsets of this thread's 4-channel piece: every token it handles
  // has row ≡ warp (mod 8), so only a multiple of 128 bytes depends on the row.
  const uint32_t col64 = sw_off(warp & 7, c4, BS_ROW64) - (uint32_t)((warp & 7) * 128);
  const uint32_t col128 = sw_off(warp & 7, c4, BS_ROW128) - (uint32_t)((warp & 7) * 128);
  const PrepSrc src{a.alpha, a.b, a.w, static_cast<const __nv_bfloat16*>(a.k),
                    static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.v),
                    a.T, a.Hqk, a.Hv, a.gate_mode};
  TokIn in[4];
  int item = blockIdx.x;
  if (item < n_items) {
    const Item it = decode_item(a, c_begin, item);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = warp + 16 * j;
      load_token(src, it.bi, it.t0 + i, it.h, it.hq, c4, i < it.Lc, in[j]);
    }
  }
  uint32_t phase = 0;
  for (; item < n_items; item += gridDim.x) {
    const Item it = decode_item(a, c_begin, item);
    uint8_t* slot = static_cast<uint8_t*>(a.workspace) + WS_HEAD + ((size_t)it.bh * n_seg + it.cl) * SLOT;

    // -------- pass 1: α rows into the staging tile; the write side Z = w ⊙ v
    // (which needs no decay) goes straight to its tile
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = warp + 16 * j;
      *reinterpret_cast<float4*>(stage + i * SS + c4) = in[j].al;
      float vx[4];
      unpack4_bf16(in[j].v, vx);
      st8(smem, P_Z + col64 + i * 128,
          pack4_f16(in[j].w.x * vx[0], in[j].w.y * vx[1], in[j].w.z * vx[2], in[j].w.w * vx[3]));
    }
    __syncthreads();
    // forward cumulative products down each channel within each quarter
    {
      const int c = tid & 127, q = tid >> 7;
      float acc = 1.f;
#pragma unroll
      for (int s_ = 0; s_ < 16; ++s_) {
        float* pp = stage + (16 * q + s_) * SS + c;
        acc *= *pp;
        *pp = acc;
      }
      sPq[q * D + c] = acc;
      float mn = acc;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      if (lane == 0) sred[warp] = mn;
    }
    __syncthreads();
    bool gram_bf16;
    {
      float mall = sred[0];
#pragma unroll
      for (int w_ = 1; w_ < NP / 32; ++w_) mall = fminf(mall, sred[w_]);
      // every in-quarter forward/backward product is ≥ the quarter product
      gram_bf16 = !(mall > 6.103515625e-05f);   // 2^-14
    }
    if (tid < D) {
      const float g = sPq[tid] * sPq[D + tid] * sPq[2 * D + tid] * sPq[3 * D + tid];
      reinterpret_cast<float*>(slot + SL_GC)[tid] = g;
    }
    float fw[4][4], Pq[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = *reinterpret_cast<const float4*>(stage + (warp + 16 * j) * SS + c4);
      fw[j][0] = v.x; fw[j][1] = v.y; fw[j][2] = v.z; fw[j][3] = v.w;
      const float4 pq = *reinterpret_cast<const float4*>(sPq + j * D + c4);
      Pq[j][0] = pq.x; Pq[j][1] = pq.y; Pq[j][2] = pq.z; Pq[j][3] = pq.w;
    }
    __syncthreads();   // the staging tile is free from here on

    // -------- pass 2: key-side operand tiles (token i = warp + 16 m is in quarter m)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int i = warp + 16 * m;
      float kx[4], qx[4], ex[4];
      unpack4_bf16(in[m].k, kx);
      unpack4_bf16(in[m].q, qx);
      ex[0] = in[m].b.x * kx[0]; ex[1] = in[m].b.y * kx[1]; ex[2] = in[m].b.z * kx[2]; ex[3] = in[m].b.w * kx[3];
      float o_eb[4], o_qb[4], o_ke[4], o_em[4], o_qm[4], o_km[4], o_x1[4], o_x2[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float P = Pq[m][c];
        float pre = 1.f, suf = 1.f;
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
          if (mm < m) pre *= Pq[mm][c];
          if (mm > m) suf *= Pq[mm][c];
        }
        const float f = fw[m][c];               // Π_{quarter start ≤ s ≤ i} α
        const float rf = __fdividef(1.f, f);
        const float bw = P * rf;                // Π_{i < s ≤ quarter end} α
        const float g = pre * f;                // γ_i
        const float bk = bw * suf;              // Π_{i < s ≤ 63} α
        o_eb[c] = ex[c] * g;
        o_qb[c] = qx[c] * g;
        o_ke[c] = kx[c] * bk;
        float fe, fk;
        if ((m & 1) == 0) {
          fe = f * __fdividef(1.f, P);          // 1 / bw
          fk = bw;
        } else {
          fe = f;
          fk = rf;
        }
        o_em[c] = ex[c] * fe;
        o_qm[c] = qx[c] * fe;
        o_km[c] = kx[c] * fk;
        if (m >= 2) {
          const float fq = (m == 3 ? Pq[2][c] : 1.f) * f;
          o_x1[c] = ex[c] * fq;
          o_x2[c] = qx[c] * fq;
        } else {
          const float fb = bw * (m == 0 ? Pq[1][c] : 1.f);
          o_x1[c] = kx[c] * fb;
          o_x2[c] = 0.f;
        }
      }
      st8(slot, SL_QB + col64 + i * 128, pack4(o_qb, false));
      st8(slot, SL_KE + col64 + i * 128, pack4(o_ke, false));
      st8(smem, P_EB + col64 + i * 128, pack4(o_eb, false));
      st8(smem, P_GM + col128 + i * 128, pack4(o_em, gram_bf16));
      st8(smem, P_GM + col128 + (64 + i) * 128, pack4(o_qm, gram_bf16));
      st8(smem, P_KM + col64 + i * 128, pack4(o_km, gram_bf16));
      if (m >= 2) {
        st8(smem, P_GB + col128 + i * 128, pack4(o_x1, gram_bf16));
        st8(smem, P_GB + col128 + (64 + i) * 128, pack4(o_x2, gram_bf16));
      } else {
        st8(smem, P_KB + col128 + i * 128, pack4(o_x1, gram_bf16));
      }
    }
    // the next item's inputs: issued now, consumed at the top of the next pass
    {
      const int nxt = item + (int)gridDim.x;
      if (nxt < n_items) {
        const Item in_ = decode_item(a, c_begin, nxt);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = warp + 16 * j;
          load_token(src, in_.bi, in_.t0 + i, in_.h, in_.hq, c4, i < in_.Lc, in[j]);
        }
      }
    }
    sync_for_mma();

    // -------- Gram MMAs: [T; Aqk] candidates
    if (tid == 0) {
      const uint64_t gm = desc_k_sw(smem_u32(smem + P_GM), 0, BS_ROW128);
      const uint64_t km = desc_k_sw(smem_u32(smem + P_KM), 0, BS_ROW64);
      const uint64_t gb = desc_k_sw(smem_u32(smem + P_GB), 0, BS_ROW128);
      const uint64_t kb = desc_k_sw(smem_u32(smem + P_KB), 0, BS_ROW128);
      const uint32_t id_m = idesc_16(128, 64, false, false, gram_bf16);
      const uint32_t id_b = idesc_16(128, 32, false, false, gram_bf16);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma16(tmem + PT_GM, gm + k_step_sw(ks, BS_ROW128), km + k_step_sw(ks, BS_ROW64), id_m, ks > 0);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma16(tmem + PT_GB, gb + k_step_sw(ks, BS_ROW128), kb + k_step_sw(ks, BS_ROW128), id_b, ks > 0);
      mma_commit(bar);
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);

    // -------- T (fp32, shared) and Aqk (fp16, workspace) from TMEM. Lanes
    // 0..63 hold rows of T, lanes 64..127 rows of Aqk; the four warps of a
    // lane quarter take 16 columns each.
    {
      const bool is_t = row < 64;
      const int i = row & 63;
      const int j0 = 16 * cgp;
      float dm[16], db[16];
      tmem_ld16(t_lane + PT_GM + j0, dm);
      tmem_ld16(t_lane + PT_GB + (j0 & 31), db);
      tmem_wait_ld();
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = j0 + u;
        const bool keep = is_t ? (j < i) : (j <= i);
        const bool same = (j >> 5) == (i >> 5);
        const float x = same ? dm[u] : (j0 < 32 ? db[u] : 0.f);
        v[u] = keep ? x : 0.f;
      }
      if (is_t) {
#pragma unroll
        for (int u = 0; u < 16; u += 4)
          *reinterpret_cast<float4*>(sT + i * TS + j0 + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
      } else {
        st16(slot, SL_AQ + sw_off(i, j0, BS_ROW64), pack8_f16(v));
        st16(slot, SL_AQ + sw_off(i, j0 + 8, BS_ROW64), pack8_f16(v + 8));
      }
    }
    __syncthreads();

    // -------- A = (I + T)⁻¹, blocked
    // level 0: the four 16 × 16 diagonal blocks by forward substitution, one
    // column per thread; the others zero the upper-right 16 × 16 block of each
    // 32-half (read by the level-2 products).
    if (tid < 64) {
      const int blk = tid >> 4, j = tid & 15, base = blk * 16;
      float x[16];
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        float acc = (ii == j) ? 1.f : 0.f;
#pragma unroll
        for (int l = 0; l < ii; ++l)
          if (l >= j) acc -= sT[(base + ii) * TS + base + l] * x[l];
        x[ii] = (ii >= j) ? acc : 0.f;
      }
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) sI[(base + ii) * TS + base + j] = x[ii];
    } else {
      for (int o = tid - 64; o < 512; o += NP - 64) {
        const int hf = o >> 8, ii = (o >> 4) & 15, jj = o & 15;
        sI[(hf * 32 + ii) * TS + hf * 32 + 16 + jj] = 0.f;
      }
    }
    __syncthreads();
    // level 1: X21 = −I22 T21 I11 in each 32-half (one entry per thread)
    {
      const int hf = tid >> 8, ii = (tid >> 4) & 15, jj = tid & 15;
      const int r0 = hf * 32 + 16, c0 = hf * 32;
      float acc = 0.f;
#pragma unroll
      for (int l = 0; l < 16; ++l) acc += sT[(r0 + ii) * TS + c0 + l] * sI[(c0 + l) * TS + c0 + jj];
      sX[(hf * 16 + ii) * 36 + jj] = acc;
    }
    __syncthreads();
    {
      const int hf = tid >> 8, ii = (tid >> 4) & 15, jj = tid & 15;
      const int r0 = hf * 32 + 16, c0 = hf * 32;
      float acc = 0.f;
#pragma unroll
      for (int l = 0; l < 16; ++l) acc += sI[(r0 + ii) * TS + r0 + l] * sX[(hf * 16 + l) * 36 + jj];
      sI[(r0 + ii) * TS + c0 + jj] = -acc;
    }
    __syncthreads();
    // level 2: X_QP = −I_QQ T_QP I_PP (thread: row ii, 2 columns)
    {
      const int ii = tid >> 4, jp = (tid & 15) * 2;
      float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
      for (int l = 0; l < 32; ++l) {
        const float t = sT[(32 + ii) * TS + l];
        const float2 iv = *reinterpret_cast<const float2*>(sI + l * TS + jp);
        a0 += t * iv.x; a1 += t * iv.y;
      }
      *reinterpret_cast<float2*>(sX + ii * 36 + jp) = make_float2(a0, a1);
    }
    __syncthreads();
    {
      const int ii = tid >> 4, jp = (tid & 15) * 2;
      float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
      for (int l = 0; l < 32; ++l) {
        const float t = sI[(32 + ii) * TS + 32 + l];
        const float2 xv = *reinterpret_cast<const float2*>(sX + l * 36 + jp);
        a0 += t * xv.x; a1 += t * xv.y;
      }
      *reinterpret_cast<float2*>(sI + (32 + ii) * TS + jp) = make_float2(-a0, -a1);
    }
    __syncthreads();
    // pack A (lower triangle; zeros above the diagonal), one 8-wide piece per thread
    {
      const int i = tid >> 3, j0 = (tid & 7) * 8;
      float x[8];
      const float4 p0 = *reinterpret_cast<const float4*>(sI + i * TS + j0);
      const float4 p1 = *reinterpret_cast<const float4*>(sI + i * TS + j0 + 4);
      x[0] = p0.x; x[1] = p0.y; x[2] = p0.z; x[3] = p0.w; x[4] = p1.x; x[5] = p1.y; x[6] = p1.z; x[7] = p1.w;
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = (j0 + u <= i) ? x[u] : 0.f;
      st16(smem, P_AINV + sw_off(i, j0, BS_ROW64), pack8_f16(x));
    }
    sync_for_mma();

    // -------- Yᵀ = Ēᵀ Aᵀ, U_wᵀ = Zᵀ Aᵀ
    if (tid == 0) {
      const uint64_t eb = desc_mn_sw(smem_u32(smem + P_EB), 0, BS_ROW64);
      const uint64_t z = desc_mn_sw(smem_u32(smem + P_Z), 0, BS_ROW64);
      const uint64_t ai = desc_k_sw(smem_u32(smem + P_AINV), 0, BS_ROW64);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        mma16(tmem + PT_YT, eb + mn_step_sw(ks), ai + k_step_sw(ks, BS_ROW64), idesc_f16(128, 64, true, false),
              ks > 0);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        mma16(tmem + PT_UW, z + mn_step_sw(ks), ai + k_step_sw(ks, BS_ROW64), idesc_f16(128, 64, true, false),
              ks > 0);
      mma_commit(bar);
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);
    {
      // column groups 0, 1: Yᵀ rows (key lanes); 2, 3: U_wᵀ rows (dv lanes)
      const uint32_t col = (cgp < 2 ? PT_YT : PT_UW) + 32u * (uint32_t)(cgp & 1);
      const int dst = cgp < 2 ? SL_YT : SL_UW;
      const int cb0 = 32 * (cgp & 1);
      float v[32];
      tmem_ld16(t_lane + col, v);
      tmem_ld16(t_lane + col + 16, v + 16);
      tmem_wait_ld();
#pragma unroll
      for (int cb = 0; cb < 32; cb += 8) st16(slot, dst + sw_off(row, cb0 + cb, BS_ROW128), pack8_f16(v + cb));
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
  }
  if (*sflag && tid == 0) atomicOr(static_cast<int*>(a.workspace), 1);
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, PT_COLS);
}

// =============================================================================
// scan kernel: one CTA per (sequence, value head), chunks of the segment in order
// =============================================================================
template <typename TOut>
__global__ void __launch_bounds__(NT, 1) chunk_scan_kernel(ChunkArgs a, int c_begin, int n_seg, const float* S_in,
                                                           float* S_out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S_BAR);
  uint64_t* bar_ys = full + 2;          // (Y S)ᵀ done
  uint64_t* bar_st = full + 3;          // state update done
  uint64_t* bar_o = full + 4;           // all MMAs of the chunk done
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + S_TMEMP);
  int* sflag = reinterpret_cast<int*>(smem + S_FLAG);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int h = bh % a.Hv, bi = bh / a.Hv;
  const uint8_t* slots = static_cast<const uint8_t*>(a.workspace) + WS_HEAD + (size_t)bh * n_seg * SLOT;
  TOut* og = static_cast<TOut*>(a.o);

  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(bar_ys, 1);
    mbar_init(bar_st, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
    *sflag = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, ST_COLS);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_ptr;
  if (tid == 0) {
    mbar_arrive_expect_tx(&full[0], SLOT_USED);
    bulk_g2s(smem + S_STAGE0, slots, SLOT_USED, &full[0]);
  }

  const int lq = warp & 3;
  const uint32_t t_lane = tmem + ((uint32_t)(lq * 32) << 16);
  const int row = lq * 32 + lane;       // dv index j of Sᵀ[j][*]
  const bool lo = warp < 4;

  // Entry state: Sᵀ[j][c] = S[c][j]. The fp16 copy (operand of the first
  // chunk's MMAs) is the state itself; TMEM holds it already multiplied by the
  // first chunk's decay Γ, ready for the first update Sᵀ ← Sᵀ Γ + Uᵀ K_end.
  if (!mbar_wait(&full[0], 0)) atomicOr(sflag, 1);
  {
    const float* gC = reinterpret_cast<const float*>(smem + S_STAGE0 + SL_GC);
    const int c0 = lo ? 0 : 64;
    const float* S0 = S_in ? S_in + (size_t)bh * D * D : nullptr;
    for (int cb = c0; cb < c0 + 64; cb += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = S0 ? __ldg(S0 + (size_t)(cb + u) * D + row) : 0.f;
      st16(smem, S_ST + sw_off(row, cb, BS_ROW128), pack8_f16(v));
      st16(smem, S_ST + sw_off(row, cb + 8, BS_ROW128), pack8_f16(v + 8));
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] *= gC[cb + u];
      tmem_st16(t_lane + ST_S + cb, v);
    }
    tmem_wait_st();
  }
  sync_for_mma();

  // Output epilogue of a chunk: Oᵀ (TMEM buffer `ob`) → staging tile
  // [rows][128] of TOut → contiguous 16-byte stores to o, O_ROWS tokens at a
  // time. It runs while the next chunk's first MMAs execute.
  constexpr int O_ROWS = 16384 / (D * (int)sizeof(TOut));   // 64 (bf16) or 32 (fp32)
  auto out_epilogue = [&](uint32_t ob, int t0o, int Lco) {
    TOut* so = reinterpret_cast<TOut*>(smem + S_OS);
    const int c0 = lo ? 0 : 32;
    float v[32];
    tmem_ld16(t_lane + ob + c0, v);
    tmem_ld16(t_lane + ob + c0 + 16, v + 16);
    tmem_wait_ld();
    constexpr int VEC = 16 / (int)sizeof(TOut);             // elements per 16 bytes
    for (int r0 = 0; r0 < C; r0 += O_ROWS) {
      if (r0 > 0) __syncthreads();
      if (c0 >= r0 && c0 < r0 + O_ROWS) {
#pragma unroll
        for (int u = 0; u < 32; ++u) so[(c0 - r0 + u) * D + row] = from_f32<TOut>(a.scale * v[u]);
      }
      __syncthreads();
      const int nvec = O_ROWS * D / VEC;
      for (int e = tid; e < nvec; e += NT) {
        const int rr = e / (D / VEC), cc = (e % (D / VEC)) * VEC;
        const int i = r0 + rr;
        if (i < Lco)
          *reinterpret_cast<uint4*>(og + (((size_t)bi * a.T + t0o + i) * a.Hv + h) * D + cc) =
              *reinterpret_cast<const uint4*>(so + rr * D + cc);
      }
    }
  };

  uint32_t mphase = 0;
  int issued = 1;                       // bulk copies issued (for the error path)
  int waited = 1;
  int prev_t0 = 0, prev_L = 0;          // chunk whose outputs are still in TMEM
  for (int cl = 0; cl < n_seg; ++cl) {
    const int s = cl & 1;
    uint8_t* stg = smem + (s ? S_STAGE1 : S_STAGE0);
    uint8_t* nstg = smem + (s ? S_STAGE0 : S_STAGE1);
    const int t0 = (c_begin + cl) * C;
    const int Lc = min(C, a.T - t0);
    const uint32_t ob = ST_O + 64u * (uint32_t)s;           // this chunk's Oᵀ buffer
    // prefetch the next chunk into the other stage (free: its MMAs and reads
    // finished before the barrier that closed the previous iteration)
    if (cl + 1 < n_seg) {
      if (tid == 0) {
        mbar_arrive_expect_tx(&full[s ^ 1], SLOT_USED);
        bulk_g2s(nstg, slots + (size_t)(cl + 1) * SLOT, SLOT_USED, &full[s ^ 1]);
      }
      ++issued;
    }
    // (Y S)ᵀ = Sᵀ Yᵀ (waited for right away), then Oᵀ = Sᵀ Q̄ᵀ
    if (tid == 0) {
      const uint64_t a0 = desc_k_sw(smem_u32(smem + S_ST), 0, BS_ROW128);
      const uint64_t y0 = desc_mn_sw(smem_u32(stg + SL_YT), 0, BS_ROW128);
      const uint64_t q0 = desc_k_sw(smem_u32(stg + SL_QB), 0, BS_ROW64);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma16(tmem + ST_YS, a0 + k_step_sw(ks, BS_ROW128), y0 + mn_step_sw(ks), idesc_f16(128, 64, false, true),
              ks > 0);
      mma_commit(bar_ys);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma16(tmem + ob, a0 + k_step_sw(ks, BS_ROW128), q0 + k_step_sw(ks, BS_ROW64),
              idesc_f16(128, 64, false, false), ks > 0);
    }
    // meanwhile: the previous chunk's outputs (its MMAs completed before the
    // barrier that closed the previous iteration)
    if (cl > 0) out_epilogue(ST_O + 64u * (uint32_t)(s ^ 1), prev_t0, prev_L);
    __syncwarp();
    {
      uint32_t ph = mphase;
      wait_mma(bar_ys, ph, sflag);
    }
    // Uᵀ = U_wᵀ − (Y S)ᵀ
    {
      const int c0 = lo ? 0 : 32;
      float ys[32], uw[32];
      tmem_ld16(t_lane + ST_YS + c0, ys);
      tmem_ld16(t_lane + ST_YS + c0 + 16, ys + 16);
#pragma unroll
      for (int cb = 0; cb < 32; cb += 8)
        unpack8_f16(*reinterpret_cast<const uint4*>(stg + SL_UW + sw_off(row, c0 + cb, BS_ROW128)), uw + cb);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 32; ++u) uw[u] -= ys[u];
#pragma unroll
      for (int cb = 0; cb < 32; cb += 8) st16(smem, S_UT + sw_off(row, c0 + cb, BS_ROW128), pack8_f16(uw + cb));
    }
    sync_for_mma();
    // Sᵀ += Uᵀ K_end (waited for by the state copy), then Oᵀ += Uᵀ Aqkᵀ
    if (tid == 0) {
      const uint64_t u0 = desc_k_sw(smem_u32(smem + S_UT), 0, BS_ROW128);
      const uint64_t k0 = desc_mn_sw(smem_u32(stg + SL_KE), 0, BS_ROW64);
      const uint64_t q0 = desc_k_sw(smem_u32(stg + SL_AQ), 0, BS_ROW64);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        mma16(tmem + ST_S, u0 + k_step_sw(ks, BS_ROW128), k0 + mn_step_sw(ks), idesc_f16(128, 128, false, true), 1);
      mma_commit(bar_st);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        mma16(tmem + ob, u0 + k_step_sw(ks, BS_ROW128), q0 + k_step_sw(ks, BS_ROW64), idesc_f16(128, 64, false, false),
              1);
      mma_commit(bar_o);
    }
    __syncwarp();
    {
      uint32_t ph = mphase;
      wait_mma(bar_st, ph, sflag);
    }
    // Next chunk's fp16 Sᵀ operand, then Sᵀ ← Sᵀ Γ_next in TMEM (the next
    // slot's γ_C; its copy was issued at the top of this iteration).
    const bool more = cl + 1 < n_seg;
    if (more) {
      if (!mbar_wait(&full[s ^ 1], ((cl + 1) >> 1) & 1)) atomicOr(sflag, 1);
      ++waited;
    }
    {
      const float* gN = reinterpret_cast<const float*>(nstg + SL_GC);
      const int c0 = lo ? 0 : 64;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tmem_ld16(t_lane + ST_S + c0 + half * 32, v);
        tmem_ld16(t_lane + ST_S + c0 + half * 32 + 16, v + 16);
        tmem_wait_ld();
#pragma unroll
        for (int cb = 0; cb < 32; cb += 8)
          st16(smem, S_ST + sw_off(row, c0 + half * 32 + cb, BS_ROW128), pack8_f16(v + cb));
        if (more) {
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] *= gN[c0 + half * 32 + u];
          tmem_st16(t_lane + ST_S + c0 + half * 32, v);
          tmem_st16(t_lane + ST_S + c0 + half * 32 + 16, v + 16);
        }
      }
      if (more) tmem_wait_st();
    }
    {
      uint32_t ph = mphase;
      wait_mma(bar_o, ph, sflag);
      mphase ^= 1u;                   // the three MMA barriers advance together
    }
    prev_t0 = t0;
    prev_L = Lc;
    sync_for_mma();
    if (*sflag) break;
  }
  // the last chunk's outputs
  if (!*sflag && n_seg > 0) out_epilogue(ST_O + 64u * (uint32_t)((n_seg - 1) & 1), prev_t0, prev_L);

  if (S_out && !*sflag) {
    const int c0 = lo ? 0 : 64;
    float* ST = S_out + (size_t)bh * D * D;
    for (int cb = c0; cb < c0 + 64; cb += 16) {
      float v[16];
      tmem_ld16(t_lane + ST_S + cb, v);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 16; ++u) ST[(size_t)(cb + u) * D + row] = v[u];
    }
  }
  if (*sflag && tid == 0) {
    atomicOr(static_cast<int*>(a.workspace), 1);
    // after an early exit a prefetched bulk copy may still be in flight:
    // wait for it (bounded) before this CTA's shared memory is released
    if (issued > waited) mbar_wait(&full[waited & 1], (waited >> 1) & 1, 1u << 16);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ST_COLS);
}

size_t state_bytes(const ChunkArgs& a) { return (size_t)a.B * a.Hv * D * D * sizeof(float); }

}  // namespace

bool chunk_tc_supported(const ChunkArgs& a, int qkv_bf16) {
  return qkv_bf16 && a.dk == D && a.dv == D && a.chunk == C && a.conv_w == nullptr && !a.l2norm;
}

// Workspace for the whole sequence in one segment.
size_t chunk_tc_workspace(const ChunkArgs& a) {
  const size_t nchunks = (a.T + C - 1) / C;
  return WS_HEAD + (size_t)a.B * a.Hv * nchunks * SLOT;
}

size_t chunk_tc_min_workspace(const ChunkArgs& a, bool carry_state) {
  return WS_HEAD + (size_t)a.B * a.Hv * SLOT + (carry_state ? state_bytes(a) : 0);
}

// Runs the chunks in segments when the workspace holds fewer chunk slots than
// the sequence has; the state is carried between segments through S_T (or,
// when S_T is NULL, through the end of the workspace).
cudaError_t launch_chunk_tc(const ChunkArgs& a, int o_bf16, cudaStream_t s) {
  const int BH = a.B * a.Hv;
  const int nchunks = (a.T + C - 1) / C;
  if (a.ws_bytes < WS_HEAD) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(a.workspace, 0, sizeof(int), s);
  if (e != cudaSuccess || BH == 0 || nchunks == 0) return e;
  size_t slot_bytes = a.ws_bytes - WS_HEAD;
  int seg = (int)std::min<size_t>(nchunks, slot_bytes / ((size_t)BH * SLOT));
  float* carry = a.ST;
  if (seg < nchunks && carry == nullptr) {
    const size_t sb = state_bytes(a);
    slot_bytes = slot_bytes > sb ? slot_bytes - sb : 0;
    seg = (int)std::min<size_t>(nchunks, slot_bytes / ((size_t)BH * SLOT));
    carry = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + WS_HEAD + (size_t)BH * seg * SLOT);
  }
  if (seg < 1) return cudaErrorInvalidValue;

  if ((e = cudaFuncSetAttribute(chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM)) !=
      cudaSuccess)
    return e;
  auto scan = o_bf16 ? chunk_scan_kernel<__nv_bfloat16> : chunk_scan_kernel<float>;
  if ((e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize, S_SMEM)) != cudaSuccess) return e;

  int dev = 0, sms = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const float* s_in = a.S0;
  for (int c0 = 0; c0 < nchunks; c0 += seg) {
    const int n = std::min(seg, nchunks - c0);
    const bool last = c0 + n >= nchunks;
    float* s_out = last ? a.ST : carry;
    chunk_prep_kernel<<<std::min(BH * n, sms), NP, P_SMEM, s>>>(a, c0, n);
    scan<<<BH, NT, S_SMEM, s>>>(a, c0, n, s_in, s_out);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    s_in = carry;
  }
  return cudaSuccess;
}

}  // namespace gdn2
