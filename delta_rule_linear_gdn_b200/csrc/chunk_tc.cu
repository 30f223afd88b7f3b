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
#include <type_traits>

#include "common.cuh"
#include "tc_prims.cuh"

namespace gdn2 {
namespace {

using namespace tc;

constexpr int D = 128;            // d_k = d_v
constexpr int C = 64;             // chunk

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
// After the Gram MMAs, [32K, 71K) holds the fp32 arrays of the inverse and
// [0, 8K) the fp16 A = (I+T)⁻¹ (64 × 64). Two CTAs of this layout fit one SM.
constexpr int P_GB = 0;
constexpr int P_KB = 0;
constexpr int P_PQ = 8192;            // quarter products [4][128] fp32
constexpr int P_RED = P_PQ + 4 * D * 4;
static_assert(P_RED + 32 <= 12288, "quarter products must stay in the unused Gram rows");
constexpr int P_GM = 32768;
constexpr int P_KM = 65536;
constexpr int P_EB = 81920;
constexpr int P_Z = 98304;
constexpr int P_END = 114688;
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
constexpr int S_BAR = S_OS + 16384;   // 13 mbarriers (see the scan kernel)
constexpr int S_TMEMP = S_BAR + 128;
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
// prep kernel: persistent, two 256-thread CTAs per SM, each looping over the
// work items (chunk of the segment, sequence, value head). While one CTA waits
// for its tensor-core products or runs the serial steps of the inverse, the
// other CTA on the SM runs its elementwise passes.
// =============================================================================
constexpr int NP = 256;               // prep threads (8 warps)

struct PrepSrc {
  const float *alpha, *b, *w;
  const __nv_bfloat16 *k, *q, *v;
};

// fp32 gate of one token for 4 channels, or the token's scalar gate broadcast.
__device__ __forceinline__ float4 gate4(const float* g, size_t gt, int c0, bool per_channel) {
  if (per_channel) return __ldg(reinterpret_cast<const float4*>(g + gt * D + c0));
  const float s = __ldg(g + gt);
  return make_float4(s, s, s, s);
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

__global__ void __launch_bounds__(NP, 2) chunk_prep_kernel(ChunkArgs a, int c_begin, int n_seg) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + P_BAR);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + P_TMEMP);
  int* sflag = reinterpret_cast<int*>(smem + P_FLAG);
  float* sPq = reinterpret_cast<float*>(smem + P_PQ);
  float* sred = reinterpret_cast<float*>(smem + P_RED);
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
  const int hc = warp >> 2;                      // which of the two warps of a lane quarter

  // Element mapping of the elementwise passes: warp w takes quarter qt = w/2
  // (tokens 16 qt .. 16 qt + 15) and channel half w%2; a lane takes 4 channels
  // c0..c0+3 of the 8 tokens i0 + u (u = 0..7). Each memory access of a warp
  // covers whole rows of 64 channels.
  const int qt = warp >> 1, cg = lane & 15, tg = lane >> 4;
  const int c0 = (warp & 1) * 64 + cg * 4;
  const int i0 = 16 * qt + 8 * tg;
  // Offset of this thread's 8-byte piece in row i0 + u of a swizzled tile,
  // less the row's i·128 ((i0 + u) mod 8 = u); `blk` is the tile's block stride.
  auto piece = [&](int u, int blk) -> uint32_t {
    return (uint32_t)((warp & 1) * blk + ((((cg >> 1) ^ u) << 4) | ((cg & 1) << 3)));
  };
  const bool full = a.gate_mode == GDN2_GATES_FULL;
  const bool alpha_pc = a.gate_mode != GDN2_GATES_GDN;
  const PrepSrc src{a.alpha, a.b, full ? a.w : a.b, static_cast<const __nv_bfloat16*>(a.k),
                    static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.v)};

  uint32_t phase = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const Item it = decode_item(a, c_begin, item);
    uint8_t* slot = static_cast<uint8_t*>(a.workspace) + WS_HEAD + ((size_t)it.bh * n_seg + it.cl) * SLOT;
    const size_t tok0 = (size_t)it.bi * a.T + it.t0 + i0;    // token of u = 0

    // -------- pass 1: the write side Z = w ⊙ v (no decay) straight to its
    // tile; α's forward products within the quarter. The key-side inputs of
    // tokens u = 0..3 are requested here, those of u = 4..7 in pass 2.
    float f[8][4];
    float4 bq[4];
    uint2 kk[4], qq[4];
    const bool whole = it.Lc == C;              // every chunk but a sequence's last
    auto load_key = [&](int u0) {
      if (whole) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const size_t gt = (tok0 + u0 + u) * a.Hv + it.h;
          const size_t tq = (tok0 + u0 + u) * a.Hqk + it.hq;
          bq[u] = gate4(src.b, gt, c0, full);
          kk[u] = __ldg(reinterpret_cast<const uint2*>(src.k + tq * D + c0));
          qq[u] = __ldg(reinterpret_cast<const uint2*>(src.q + tq * D + c0));
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const bool ok = i0 + u0 + u < it.Lc;
          const size_t gt = (tok0 + u0 + u) * a.Hv + it.h;
          const size_t tq = (tok0 + u0 + u) * a.Hqk + it.hq;
          bq[u] = ok ? gate4(src.b, gt, c0, full) : make_float4(0.f, 0.f, 0.f, 0.f);
          kk[u] = ok ? __ldg(reinterpret_cast<const uint2*>(src.k + tq * D + c0)) : make_uint2(0, 0);
          qq[u] = ok ? __ldg(reinterpret_cast<const uint2*>(src.q + tq * D + c0)) : make_uint2(0, 0);
        }
      }
    };
    {
      float4 wv[8];
      uint2 vv[8];
      if (whole) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const size_t gt = (tok0 + u) * a.Hv + it.h;
          const float4 al = gate4(src.alpha, gt, c0, alpha_pc);
          f[u][0] = al.x; f[u][1] = al.y; f[u][2] = al.z; f[u][3] = al.w;
          wv[u] = gate4(src.w, gt, c0, full);
          vv[u] = __ldg(reinterpret_cast<const uint2*>(src.v + gt * D + c0));
        }
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const bool ok = i0 + u < it.Lc;
          const size_t gt = (tok0 + u) * a.Hv + it.h;
          const float4 al = ok ? gate4(src.alpha, gt, c0, alpha_pc) : make_float4(1.f, 1.f, 1.f, 1.f);
          f[u][0] = al.x; f[u][1] = al.y; f[u][2] = al.z; f[u][3] = al.w;
          wv[u] = ok ? gate4(src.w, gt, c0, full) : make_float4(0.f, 0.f, 0.f, 0.f);
          vv[u] = ok ? __ldg(reinterpret_cast<const uint2*>(src.v + gt * D + c0)) : make_uint2(0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float vx[4];
        unpack4_bf16(vv[u], vx);
        st8(smem, P_Z + (uint32_t)(i0 + u) * 128 + piece(u, BS_ROW64),
            pack4_f16(wv[u].x * vx[0], wv[u].y * vx[1], wv[u].z * vx[2], wv[u].w * vx[3]));
      }
    }
    load_key(0);
    {
      // within the thread's 8 tokens, then across the two token groups of the
      // quarter (lanes l and l + 16)
      float pq[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int u = 1; u < 8; ++u) f[u][c] *= f[u - 1][c];
        const float y = __shfl_up_sync(0xffffffffu, f[7][c], 16);
        const float ex = tg ? y : 1.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u][c] *= ex;
        pq[c] = __shfl_sync(0xffffffffu, f[7][c], cg + 16);    // product over the quarter
      }
      if (tg == 0) *reinterpret_cast<float4*>(sPq + qt * D + c0) = make_float4(pq[0], pq[1], pq[2], pq[3]);
      float mn = fminf(fminf(pq[0], pq[1]), fminf(pq[2], pq[3]));
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
    // Per-channel factors of quarter qt from the quarter products P_m:
    //   γ_i = pre · f_i,                      pre = Π_{m<qt} P_m
    //   Π_{i<s≤63} α = (P_qt · suf) / f_i,      suf = Π_{m>qt} P_m
    //   mid-reference factors: f_i / P_qt and P_qt / f_i (first quarter of a
    //   half), f_i and 1 / f_i (second quarter);
    //   half-boundary factors: P_2 f_i (quarter 3), f_i (quarter 2) for rows
    //   of the second half; P_qt P_1 / f_i (quarter 0), P_qt / f_i (quarter 1)
    //   for keys of the first half.
    float pre[4], ps[4], se[4], sk[4], sx[4];
    {
      float P[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 v = *reinterpret_cast<const float4*>(sPq + m * D + c0);
        P[m][0] = v.x; P[m][1] = v.y; P[m][2] = v.z; P[m][3] = v.w;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float pr = 1.f, su = 1.f, own = P[0][c];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          if (m < qt) pr *= P[m][c];
          if (m > qt) su *= P[m][c];
          if (m == qt) own = P[m][c];
        }
        pre[c] = pr;
        ps[c] = own * su;
        const bool even = (qt & 1) == 0;
        se[c] = even ? rcp_approx(own) : 1.f;
        sk[c] = even ? own : 1.f;
        sx[c] = qt == 3 ? P[2][c] : (qt == 2 ? 1.f : (qt == 0 ? own * P[1][c] : own));
      }
    }

    // -------- pass 2: key-side operand tiles, tile by tile per token
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (u == 4) load_key(4);
      const int uk = u & 3;
      const uint32_t i128 = (uint32_t)(i0 + u) * 128;
      const uint32_t p64 = i128 + piece(u, BS_ROW64), p128 = i128 + piece(u, BS_ROW128);
      float kx[4], qx[4], e[4], rf[4], g[4], fe[4];
      unpack4_bf16(kk[uk], kx);
      unpack4_bf16(qq[uk], qx);
      e[0] = bq[uk].x * kx[0]; e[1] = bq[uk].y * kx[1]; e[2] = bq[uk].z * kx[2]; e[3] = bq[uk].w * kx[3];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        rf[c] = rcp_approx(f[u][c]);
        g[c] = pre[c] * f[u][c];
        fe[c] = se[c] * f[u][c];
      }
      float o[4];
#define GDN2_TILE(dst, off, expr)                                             \
  {                                                                           \
    _Pragma("unroll") for (int c = 0; c < 4; ++c) o[c] = (expr);              \
    st8(dst, off, pack4_f16(o[0], o[1], o[2], o[3]));                         \
  }
#define GDN2_GRAM_TILE(dst, off, expr)                                        \
  {                                                                           \
    _Pragma("unroll") for (int c = 0; c < 4; ++c) o[c] = (expr);              \
    if (gram_bf16)                                                            \
      st8(dst, off, pack4_bf16(o[0], o[1], o[2], o[3]));                      \
    else                                                                      \
      st8(dst, off, pack4_f16(o[0], o[1], o[2], o[3]));                       \
  }
      GDN2_TILE(slot, SL_QB + p64, qx[c] * g[c])
      GDN2_TILE(slot, SL_KE + p64, kx[c] * (ps[c] * rf[c]))
      GDN2_TILE(smem, P_EB + p64, e[c] * g[c])
      GDN2_GRAM_TILE(smem, P_GM + p128, e[c] * fe[c])
      GDN2_GRAM_TILE(smem, P_GM + 64 * 128 + p128, qx[c] * fe[c])
      GDN2_GRAM_TILE(smem, P_KM + p64, kx[c] * (sk[c] * rf[c]))
      if (qt >= 2) {
        GDN2_GRAM_TILE(smem, P_GB + p128, e[c] * (sx[c] * f[u][c]))
        GDN2_GRAM_TILE(smem, P_GB + 64 * 128 + p128, qx[c] * (sx[c] * f[u][c]))
      } else {
        GDN2_GRAM_TILE(smem, P_KB + p128, kx[c] * (sx[c] * rf[c]))
      }
#undef GDN2_TILE
#undef GDN2_GRAM_TILE
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
    // 0..63 hold rows of T, lanes 64..127 rows of Aqk; the two warps of a lane
    // quarter take 32 columns each (only columns < 32 need the half-boundary
    // product: a row i ≥ 32 against a key j < 32).
    {
      const bool is_t = row < 64;
      const int i = row & 63;
      const int j0 = 32 * hc;
      float dm[32], db[32];
      tmem_ld16(t_lane + PT_GM + j0, dm);
      tmem_ld16(t_lane + PT_GM + j0 + 16, dm + 16);
      if (hc == 0) {
        tmem_ld16(t_lane + PT_GB, db);
        tmem_ld16(t_lane + PT_GB + 16, db + 16);
      }
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int j = j0 + u;
        const bool keep = is_t ? (j < i) : (j <= i);
        const bool same = (j >> 5) == (i >> 5);
        const float x = same ? dm[u] : (hc == 0 ? db[u] : 0.f);
        dm[u] = keep ? x : 0.f;
      }
      if (is_t) {
#pragma unroll
        for (int u = 0; u < 32; u += 4)
          *reinterpret_cast<float4*>(sT + i * TS + j0 + u) = make_float4(dm[u], dm[u + 1], dm[u + 2], dm[u + 3]);
      } else {
#pragma unroll
        for (int cb = 0; cb < 32; cb += 8) st16(slot, SL_AQ + sw_off(i, j0 + cb, BS_ROW64), pack8_f16(dm + cb));
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
    // level 1: X21 = −I22 T21 I11 in each 32-half (two entries per thread)
    {
      const int hf = tid >> 7, ii = (tid >> 3) & 15, jj = (tid & 7) * 2;
      const int r0 = hf * 32 + 16, cc = hf * 32;
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int l = 0; l < 16; ++l) {
        const float t = sT[(r0 + ii) * TS + cc + l];
        const float2 iv = *reinterpret_cast<const float2*>(sI + (cc + l) * TS + cc + jj);
        a0 += t * iv.x;
        a1 += t * iv.y;
      }
      *reinterpret_cast<float2*>(sX + (hf * 16 + ii) * 36 + jj) = make_float2(a0, a1);
    }
    __syncthreads();
    {
      const int hf = tid >> 7, ii = (tid >> 3) & 15, jj = (tid & 7) * 2;
      const int r0 = hf * 32 + 16, cc = hf * 32;
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int l = 0; l < 16; ++l) {
        const float t = sI[(r0 + ii) * TS + r0 + l];
        const float2 xv = *reinterpret_cast<const float2*>(sX + (hf * 16 + l) * 36 + jj);
        a0 += t * xv.x;
        a1 += t * xv.y;
      }
      *reinterpret_cast<float2*>(sI + (r0 + ii) * TS + cc + jj) = make_float2(-a0, -a1);
    }
    __syncthreads();
    // level 2: X_QP = −I_QQ T_QP I_PP (thread: row ii, 4 columns)
    {
      const int ii = tid >> 3, jp = (tid & 7) * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
      for (int l = 0; l < 32; ++l) {
        const float t = sT[(32 + ii) * TS + l];
        const float4 iv = *reinterpret_cast<const float4*>(sI + l * TS + jp);
        acc.x += t * iv.x; acc.y += t * iv.y; acc.z += t * iv.z; acc.w += t * iv.w;
      }
      *reinterpret_cast<float4*>(sX + ii * 36 + jp) = acc;
    }
    __syncthreads();
    {
      const int ii = tid >> 3, jp = (tid & 7) * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
      for (int l = 0; l < 32; ++l) {
        const float t = sI[(32 + ii) * TS + 32 + l];
        const float4 xv = *reinterpret_cast<const float4*>(sX + l * 36 + jp);
        acc.x += t * xv.x; acc.y += t * xv.y; acc.z += t * xv.z; acc.w += t * xv.w;
      }
      *reinterpret_cast<float4*>(sI + (32 + ii) * TS + jp) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    __syncthreads();
    // pack A (lower triangle; zeros above the diagonal), 16 entries per thread
    {
      const int i = tid >> 2, j0 = (tid & 3) * 16;
#pragma unroll
      for (int h8 = 0; h8 < 16; h8 += 8) {
        float x[8];
        const float4 p0 = *reinterpret_cast<const float4*>(sI + i * TS + j0 + h8);
        const float4 p1 = *reinterpret_cast<const float4*>(sI + i * TS + j0 + h8 + 4);
        x[0] = p0.x; x[1] = p0.y; x[2] = p0.z; x[3] = p0.w; x[4] = p1.x; x[5] = p1.y; x[6] = p1.z; x[7] = p1.w;
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = (j0 + h8 + u <= i) ? x[u] : 0.f;
        st16(smem, P_AINV + sw_off(i, j0 + h8, BS_ROW64), pack8_f16(x));
      }
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
      // warps 0..3: Yᵀ rows (key lanes); warps 4..7: U_wᵀ rows (dv lanes)
      const uint32_t col = hc == 0 ? PT_YT : PT_UW;
      const int dst = hc == 0 ? SL_YT : SL_UW;
#pragma unroll
      for (int cb0 = 0; cb0 < 64; cb0 += 32) {
        float v[32];
        tmem_ld16(t_lane + col + cb0, v);
        tmem_ld16(t_lane + col + cb0 + 16, v + 16);
        tmem_wait_ld();
#pragma unroll
        for (int cb = 0; cb < 32; cb += 8) st16(slot, dst + sw_off(row, cb0 + cb, BS_ROW128), pack8_f16(v + cb));
      }
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
// scan kernel: one CTA per (sequence, value head), chunks of the segment in
// order. Warp 12 issues the tensor-core products and the slot copies (one
// thread); warps 0..7 run the state chain, warps 8..11 write the outputs.
// They hand over through mbarriers:
//   MMA thread, chunk c:  (Y S)ᵀ [after each half of the fp16 Sᵀ copy] → Oᵀ =
//     Sᵀ Q̄ᵀ → [after Uᵀ] Sᵀ += Uᵀ K_end in two 64-key halves → Oᵀ += Uᵀ Aqkᵀ →
//     [when chunk c's products are done] copy of chunk c + 2's slot;
//   chain warps, chunk c:  Uᵀ = U_wᵀ − (Y S)ᵀ → per key half: fp16 Sᵀ copy for
//     chunk c + 1 and Sᵀ ← Sᵀ Γ_{c+1} in TMEM;
//   output warps, chunk c:  Oᵀ (double-buffered in TMEM) → o.
// =============================================================================
constexpr int NS = 416;               // scan threads: 8 chain warps, 4 output warps, 1 MMA warp
constexpr int NO = 128;               // output threads

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }
__device__ __forceinline__ void out_sync() { asm volatile("bar.sync 2, 128;\n" ::: "memory"); }

template <typename TOut>
__global__ void __launch_bounds__(NS, 1) chunk_scan_kernel(ChunkArgs a, int c_begin, int n_seg, const float* S_in,
                                                           float* S_out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S_BAR);
  uint64_t* full = bars;                // [2] slot copy landed in stage s
  uint64_t* b_ys = bars + 2;            // (Y S)ᵀ done
  uint64_t* b_sa = bars + 3;            // state update, keys 0..63, done
  uint64_t* b_sb = bars + 4;            // state update, keys 64..127, done
  uint64_t* b_o = bars + 5;             // every product of the chunk done
  uint64_t* b_u = bars + 6;             // Uᵀ written
  uint64_t* b_slo = bars + 7;           // fp16 Sᵀ keys 0..63 written (and TMEM scaled)
  uint64_t* b_shi = bars + 8;           // keys 64..127
  uint64_t* b_of = bars + 9;            // [2] Oᵀ buffer read out
  uint64_t* b_ob = bars + 11;           // [2] Oᵀ buffer complete (one phase per use)
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + S_TMEMP);
  int* sflag = reinterpret_cast<int*>(smem + S_FLAG);
  int* estop = sflag + 1;               // the chain warps' sample of the flag
  int* ostop = sflag + 2;               // the output warps' sample
  const volatile int* vflag = sflag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int h = bh % a.Hv, bi = bh / a.Hv;
  const uint8_t* slots = static_cast<const uint8_t*>(a.workspace) + WS_HEAD + (size_t)bh * n_seg * SLOT;
  TOut* og = static_cast<TOut*>(a.o);

  if (tid == 0) {
    for (int i = 0; i < 13; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    sflag[0] = 0;
    sflag[1] = 0;
    sflag[2] = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, ST_COLS);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_ptr;

  if (warp == 12) {
    // ------------------------------------------------------------ MMA thread
    if (lane == 0) {
      int issued = 0, landed = 0;       // slot copies issued / seen complete
      for (int c = 0; c < n_seg && c < 2; ++c) {
        mbar_arrive_expect_tx(&full[c], SLOT_USED);
        bulk_g2s(smem + (c ? S_STAGE1 : S_STAGE0), slots + (size_t)c * SLOT, SLOT_USED, &full[c]);
        ++issued;
      }
      const uint32_t id64 = idesc_f16(128, 64, false, false);
      const uint32_t id64n = idesc_f16(128, 64, false, true);
      const uint64_t sdesc0 = desc_k_sw(smem_u32(smem + S_ST), 0, BS_ROW128);
      const uint64_t udesc0 = desc_k_sw(smem_u32(smem + S_UT), 0, BS_ROW128);
      bool ok = true;
      for (int c = 0; c < n_seg && ok; ++c) {
        const int s = c & 1;
        const uint32_t ph = (uint32_t)(c & 1);
        uint8_t* stg = smem + (s ? S_STAGE1 : S_STAGE0);
        const uint32_t ob = ST_O + 64u * (uint32_t)s;
        ok = mbar_wait_or_stop(&full[s], (uint32_t)((c >> 1) & 1), vflag);
        if (!ok) break;
        ++landed;
        const uint64_t y0 = desc_mn_sw(smem_u32(stg + SL_YT), 0, BS_ROW128);
        // (Y S)ᵀ = Sᵀ Yᵀ, keys 0..63 then 64..127 as the fp16 copy lands
        ok = mbar_wait_or_stop(b_slo, ph, vflag);
        if (!ok) break;
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma16(tmem + ST_YS, sdesc0 + k_step_sw(ks, BS_ROW128), y0 + mn_step_sw(ks), id64n, ks > 0);
        ok = mbar_wait_or_stop(b_shi, ph, vflag);
        if (!ok) break;
        fence_after_sync();
#pragma unroll
        for (int ks = 4; ks < 8; ++ks)
          mma16(tmem + ST_YS, sdesc0 + k_step_sw(ks, BS_ROW128), y0 + mn_step_sw(ks), id64n, 1);
        mma_commit(b_ys);
        // Oᵀ = Sᵀ Q̄ᵀ into this chunk's buffer, once chunk c − 2 has left it
        if (c >= 2) {
          ok = mbar_wait_or_stop(&b_of[s], (uint32_t)(((c - 2) >> 1) & 1), vflag);
          if (!ok) break;
          fence_after_sync();
        }
        const uint64_t q0 = desc_k_sw(smem_u32(stg + SL_QB), 0, BS_ROW64);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma16(tmem + ob, sdesc0 + k_step_sw(ks, BS_ROW128), q0 + k_step_sw(ks, BS_ROW64), id64, ks > 0);
        // Sᵀ += Uᵀ K_end (two key halves), then Oᵀ += Uᵀ Aqkᵀ
        ok = mbar_wait_or_stop(b_u, ph, vflag);
        if (!ok) break;
        fence_after_sync();
        const uint64_t ke0 = desc_mn_sw(smem_u32(stg + SL_KE), 0, BS_ROW64);
        const uint64_t ke1 = desc_mn_sw(smem_u32(stg + SL_KE + BS_ROW64), 0, BS_ROW64);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma16(tmem + ST_S, udesc0 + k_step_sw(ks, BS_ROW128), ke0 + mn_step_sw(ks), id64n, 1);
        mma_commit(b_sa);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma16(tmem + ST_S + 64, udesc0 + k_step_sw(ks, BS_ROW128), ke1 + mn_step_sw(ks), id64n, 1);
        mma_commit(b_sb);
        const uint64_t aq0 = desc_k_sw(smem_u32(stg + SL_AQ), 0, BS_ROW64);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma16(tmem + ob, udesc0 + k_step_sw(ks, BS_ROW128), aq0 + k_step_sw(ks, BS_ROW64), id64, 1);
        mma_commit(b_o);
        mma_commit(&b_ob[s]);
        // stage s is free once this chunk's products are done: chunk c + 2
        if (c + 2 < n_seg) {
          ok = mbar_wait_or_stop(b_o, ph, vflag);
          if (!ok) break;
          mbar_arrive_expect_tx(&full[s], SLOT_USED);
          bulk_g2s(stg, slots + (size_t)(c + 2) * SLOT, SLOT_USED, &full[s]);
          ++issued;
        }
      }
      if (!ok) {
        atomicOr(sflag, 1);
        // copies still in flight complete (bounded) before shared memory is released
        for (int k = landed; k < issued; ++k) mbar_wait(&full[k & 1], (uint32_t)((k >> 1) & 1), 1u << 16);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ chain warps
    const int lq = warp & 3;
    const uint32_t t_lane = tmem + ((uint32_t)(lq * 32) << 16);
    const int row = lq * 32 + lane;     // dv index j of Sᵀ[j][*], Oᵀ[j][*]
    const int hw = warp >> 2;           // which of the two warps of a lane quarter
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok && !mbar_wait_or_stop(bar, parity, vflag)) {
        ok = false;
        atomicOr(sflag, 1);
      }
      fence_after_sync();
    };
    // Publish this thread's fp16 operand writes and TMEM stores, then one
    // arrival for all 256 epilogue threads.
    auto publish = [&](uint64_t* bar) {
      fence_async_smem();
      fence_before_sync();
      epi_sync();
      if (tid == 0) mbar_arrive(bar);
    };

    // Entry state: Sᵀ[j][c] = S[c][j]. The fp16 copy (operand of the first
    // chunk's products) is the state itself; TMEM holds it multiplied by the
    // first chunk's decay Γ, ready for the first update Sᵀ ← Sᵀ Γ + Uᵀ K_end.
    wait(&full[0], 0);
    {
      const float* gC = reinterpret_cast<const float*>(smem + S_STAGE0 + SL_GC);
      const float* S0 = S_in ? S_in + (size_t)bh * D * D : nullptr;
      for (int cb = hw * 64; cb < hw * 64 + 64; cb += 16) {
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
    publish(b_slo);
    if (tid == 0) mbar_arrive(b_shi);

    // fp16 copy of 32 key columns [k0, k0 + 32) of Sᵀ for the next chunk's
    // products, and Sᵀ ← Sᵀ Γ_next in TMEM.
    auto copy_state = [&](int k0, const float* gN) {
      float v[32];
      tmem_ld16(t_lane + ST_S + k0, v);
      tmem_ld16(t_lane + ST_S + k0 + 16, v + 16);
      tmem_wait_ld();
#pragma unroll
      for (int cb = 0; cb < 32; cb += 8) st16(smem, S_ST + sw_off(row, k0 + cb, BS_ROW128), pack8_f16(v + cb));
#pragma unroll
      for (int u = 0; u < 32; ++u) v[u] *= gN[k0 + u];
      tmem_st16(t_lane + ST_S + k0, v);
      tmem_st16(t_lane + ST_S + k0 + 16, v + 16);
      tmem_wait_st();
    };

    for (int c = 0; c < n_seg; ++c) {
      const int s = c & 1;
      const uint32_t ph = (uint32_t)(c & 1);
      const uint8_t* stg = smem + (s ? S_STAGE1 : S_STAGE0);
      const uint8_t* nstg = smem + (s ? S_STAGE0 : S_STAGE1);
      // Uᵀ = U_wᵀ − (Y S)ᵀ
      wait(&full[s], (uint32_t)((c >> 1) & 1));
      wait(b_ys, ph);
      {
        const int c0 = hw * 32;
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
      publish(b_u);
      // the state for the next chunk, one key half at a time (barriers are
      // reached by every epilogue thread whatever its own waits returned)
      const bool more = c + 1 < n_seg;
      if (more) wait(&full[s ^ 1], (uint32_t)(((c + 1) >> 1) & 1));
      const float* gN = reinterpret_cast<const float*>(nstg + SL_GC);
      wait(b_sa, ph);
      if (more) {
        copy_state(hw * 32, gN);
        publish(b_slo);
      }
      wait(b_sb, ph);
      if (more) {
        copy_state(64 + hw * 32, gN);
        publish(b_shi);
      }
      // stop together: every thread's flag update precedes the first barrier,
      // one thread samples the flag, all read the sample after the second
      if (!ok) atomicOr(sflag, 1);
      epi_sync();
      if (tid == 0) *estop = *vflag;
      epi_sync();
      if (*estop) {
        ok = false;
        break;
      }
    }
    // S_T (the loop ran to its end on every thread or stopped on every thread)
    const bool done = *estop == 0;
    if (S_out && done && ok) {
      float* ST = S_out + (size_t)bh * D * D;
      for (int cb = hw * 64; cb < hw * 64 + 64; cb += 16) {
        float v[16];
        tmem_ld16(t_lane + ST_S + cb, v);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) ST[(size_t)(cb + u) * D + row] = v[u];
      }
    }
    if (!ok) atomicOr(sflag, 1);
  } else {
    // ------------------------------------------------------------ output warps
    // Oᵀ (TMEM buffer of chunk c) → staging tile [rows][128] of TOut →
    // contiguous 16-byte stores to o, O_ROWS tokens at a time; the buffer is
    // released as soon as it has been read.
    const int lq = warp & 3;
    const uint32_t t_lane = tmem + ((uint32_t)(lq * 32) << 16);
    const int row = lq * 32 + lane;
    const int otid = tid - 256;
    bool ok = true;
    TOut* so = reinterpret_cast<TOut*>(smem + S_OS);
    constexpr int O_ROWS = 16384 / (D * (int)sizeof(TOut));   // 64 (bf16) or 32 (fp32)
    constexpr int VEC = 16 / (int)sizeof(TOut);               // elements per 16 bytes
    for (int c = 0; c < n_seg; ++c) {
      const int s = c & 1;
      const int t0 = (c_begin + c) * C;
      const int Lc = min(C, a.T - t0);
      if (ok && !mbar_wait_or_stop(&b_ob[s], (uint32_t)((c >> 1) & 1), vflag)) {
        ok = false;
        atomicOr(sflag, 1);
      }
      fence_after_sync();
      float v[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld16(t_lane + ST_O + 64u * (uint32_t)s + 16 * q, v + 16 * q);
      tmem_wait_ld();
      fence_before_sync();
#pragma unroll
      for (int r0 = 0; r0 < C; r0 += O_ROWS) {
#pragma unroll
        for (int u = 0; u < O_ROWS; ++u) so[u * D + row] = from_f32<TOut>(a.scale * v[r0 + u]);
        out_sync();
        if (r0 == 0 && otid == 0) mbar_arrive(&b_of[s]);
        const int nvec = O_ROWS * D / VEC;
        for (int e = otid; e < nvec; e += NO) {
          const int rr = e / (D / VEC), cc = (e % (D / VEC)) * VEC;
          const int i = r0 + rr;
          if (i < Lc)
            *reinterpret_cast<uint4*>(og + (((size_t)bi * a.T + t0 + i) * a.Hv + h) * D + cc) =
                *reinterpret_cast<const uint4*>(so + rr * D + cc);
        }
        out_sync();
      }
      // stop together (as the chain warps do)
      if (!ok) atomicOr(sflag, 1);
      out_sync();
      if (otid == 0) *ostop = *vflag;
      out_sync();
      if (*ostop) break;
    }
  }
  fence_before_sync();
  __syncthreads();
  if (tid == 0 && *sflag) atomicOr(static_cast<int*>(a.workspace), 1);
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
  // all of the unified L1/shared storage as shared memory, so that two prep CTAs fit an SM
  if ((e = cudaFuncSetAttribute(chunk_prep_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
    return e;
  auto scan = o_bf16 ? chunk_scan_kernel<__nv_bfloat16> : chunk_scan_kernel<float>;
  if ((e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize, S_SMEM)) != cudaSuccess) return e;

  int dev = 0, sms = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  // Persistent prep: two CTAs per SM. Two fit by shared memory (2 × 113 KB),
  // registers (2 × 256 × 128) and tensor memory (2 × 256 of 512 columns); the
  // occupancy calculator reports one for any kernel that allocates tensor
  // memory, so the count is set here. CTAs beyond those resident would only
  // start later (items are independent).
  const int prep_ctas = sms * 2;
  const float* s_in = a.S0;
  for (int c0 = 0; c0 < nchunks; c0 += seg) {
    const int n = std::min(seg, nchunks - c0);
    const bool last = c0 + n >= nchunks;
    float* s_out = last ? a.ST : carry;
    chunk_prep_kernel<<<std::min(BH * n, prep_ctas), NP, P_SMEM, s>>>(a, c0, n);
    scan<<<BH, NS, S_SMEM, s>>>(a, c0, n, s_in, s_out);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    s_in = carry;
  }
  return cudaSuccess;
}

}  // namespace gdn2
