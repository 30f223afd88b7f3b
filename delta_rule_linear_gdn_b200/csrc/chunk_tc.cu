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
// Everything is computed transposed so that the MMA's M dimension is always
// 128 (d_v or d_k or a stacked pair of 64-token operands):
//     (Y S)ᵀ = Sᵀ Yᵀ,  Oᵀ = Sᵀ Q̄ᵀ + Uᵀ Aqkᵀ,  Sᵀ ← Sᵀ Γ + Uᵀ K_end,
//     Yᵀ = Ēᵀ Aᵀ,  U_wᵀ = Zᵀ Aᵀ,  [T; Aqk] = [Ē'; Q̄'] K̃'ᵀ.
// Sᵀ lives in TMEM in fp32 for the whole sequence; an fp16 copy in shared
// memory feeds the next chunk's MMAs.
//
// Decay factors of the Gram matrices. Π_{j<s≤i} α is split into two factors
// about a reference token so that one factor multiplies row i and the other
// row j (and each GEMM stays a GEMM):
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
// Aqk, Y, U and the copy of S) is bounded in magnitude and is stored as fp16
// (11-bit significand), which is eight times finer than bf16 at the same
// tensor-core rate; this is what keeps the chunked result within 2e-2 of the
// float64 token loop. The Gram factors contain reciprocals of decay products
// and use fp16 only when the chunk's largest factor is below 2^14, bf16
// (fp32 range) otherwise. The fp16 operands require |S| and |v| below 6e4.

#include "common.cuh"
#include "tc_prims.cuh"

namespace gdn2 {
namespace {

using namespace tc;

constexpr int D = 128;            // d_k = d_v
constexpr int C = 64;             // chunk
constexpr int NT = 256;           // threads (8 warps)

// Shared-memory map (bytes). Region G holds the Gram operands and is reused
// after the Gram MMAs for the solve, the inverse and the scan's U and Y tiles.
constexpr int OFF_GB = 0;                      // [Ē_bnd ; Q̄_bnd] 128 × 128 (rows 32..63, 96..127 used)
constexpr int OFF_GM = OFF_GB + 128 * D * 2;   // [Ē_mid ; Q̄_mid] 128 × 128
constexpr int OFF_KM = OFF_GM + 128 * D * 2;   // K̃_mid 64 × 128
constexpr int OFF_KB = OFF_KM + C * D * 2;     // K̃_bnd 32 × 128
constexpr int G_END = OFF_KB + 32 * D * 2;     // 90112
// reuse of region G after the Gram MMAs
constexpr int OFF_AINV = 0;                    // A = (I+T)⁻¹ fp16 64 × 64
constexpr int OFF_AQK = OFF_AINV + C * C * 2;  // Aqk fp16 64 × 64
constexpr int TP = C + 1;                      // padded fp32 row stride
constexpr int OFF_T = OFF_AQK + C * C * 2;     // T fp32 [64][65]
constexpr int OFF_INV = OFF_T + C * TP * 4;    // inverse fp32 [64][65]
constexpr int OFF_TMP = OFF_INV + C * TP * 4;  // temp fp32 [64][65]
constexpr int OFF_YT = OFF_T;                  // Yᵀ fp16 128 × 64 (after the inverse is packed)
constexpr int OFF_UT = OFF_YT + D * C * 2;     // Uᵀ fp16 128 × 64
static_assert(OFF_TMP + C * TP * 4 <= G_END, "region G overflow");
static_assert(OFF_UT + D * C * 2 <= G_END, "region G overflow");
// persistent tiles
constexpr int OFF_EB = G_END;                  // Ē   [64 tok][128 key]
constexpr int OFF_Z = OFF_EB + C * D * 2;      // Z   [64 tok][128 dv]
constexpr int OFF_QB = OFF_Z + C * D * 2;      // Q̄   [64 tok][128 key]
constexpr int OFF_KE = OFF_QB + C * D * 2;     // K_end [64 tok][128 key]
constexpr int OFF_ST = OFF_KE + C * D * 2;     // Sᵀ fp16 [128 dv][128 key]
constexpr int OFF_GC = OFF_ST + D * D * 2;     // γ_C fp32 [128]
constexpr int OFF_BAR = OFF_GC + D * 4;        // mbarrier
constexpr int OFF_TMEMP = OFF_BAR + 16;        // TMEM base address
constexpr int OFF_FLAG = OFF_TMEMP + 16;       // error flag
constexpr int OFF_RED = OFF_FLAG + 16;         // per-warp reduction slots [8]
constexpr int SMEM_BYTES = OFF_RED + 32;

// TMEM columns (fp32, 128 lanes).
constexpr uint32_t TM_S = 0;        // Sᵀ [dv lanes][128 key]
constexpr uint32_t TM_GM = 128;     // Gram mid [128][64]
constexpr uint32_t TM_GB = 192;     // Gram bnd [128][32]
constexpr uint32_t TM_YT = 224;     // Yᵀ [key lanes][64 tok]
constexpr uint32_t TM_UW = 288;     // U_wᵀ [dv][64]
constexpr uint32_t TM_YS = 352;     // (Y S)ᵀ [dv][64]
constexpr uint32_t TM_O = 416;      // Oᵀ [dv][64]
constexpr uint32_t TM_COLS = 512;

__device__ __forceinline__ void st16(uint8_t* base, uint32_t off, uint4 v) {
  *reinterpret_cast<uint4*>(base + off) = v;
}

__device__ __forceinline__ void load8_f32(const float* p, float* x) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* p, float* x) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// Wait for the tensor core to finish the MMAs committed to `bar`; all threads
// take part. On a timeout the CTA's error flag is raised (uniformly read after
// the barrier that follows).
__device__ __forceinline__ void wait_mma(uint64_t* bar, uint32_t& phase, int* sflag) {
  if (!mbar_wait(bar, phase)) atomicOr(sflag, 1);
  phase ^= 1u;
  fence_after_sync();
}

template <typename TOut>
__global__ void __launch_bounds__(NT, 1) chunk_tc_kernel(ChunkArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + OFF_TMEMP);
  int* sflag = reinterpret_cast<int*>(smem + OFF_FLAG);
  float* sgC = reinterpret_cast<float*>(smem + OFF_GC);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int h = bh % a.Hv, bi = bh / a.Hv;
  const int hq = h / (a.Hv / a.Hqk);
  const int mode = a.gate_mode;
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);
  TOut* og = static_cast<TOut*>(a.o);

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    *sflag = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, TM_COLS);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_ptr;
  uint32_t phase = 0;

  // TMEM lane quarter of this warp and the row this thread owns there.
  const int lq = warp & 3;
  const uint32_t t_lane = tmem + ((uint32_t)(lq * 32) << 16);
  const int row = lq * 32 + lane;          // dv index (or key / token-row index)
  const bool lo = warp < 4;                // warps 0-3: first column half; 4-7: second

  // ---------------------------------------------------------------- entry state
  {
    // Thread (row = dv j) owns Sᵀ[j][*] = S[*][j]; each warp pair splits the 128 key columns.
    const int c0 = lo ? 0 : 64;
    const float* S0 = a.S0 ? a.S0 + (size_t)bh * D * D : nullptr;
    for (int cb = c0; cb < c0 + 64; cb += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = S0 ? __ldg(S0 + (size_t)(cb + u) * D + row) : 0.f;
      tmem_st16(t_lane + TM_S + cb, v);
      st16(smem + OFF_ST, tile_off(row, cb, D), pack8_f16(v));
      st16(smem + OFF_ST, tile_off(row, cb + 8, D), pack8_f16(v + 8));
    }
    tmem_wait_st();
  }

  const int nchunks = (a.T + C - 1) / C;
  // Element mapping of the load/elementwise passes: lane r = token within a
  // 16-token quarter, 8 channels per thread.
  const int r16 = lane & 15;
  const int cg = 2 * warp + (lane >> 4);
  const int ch0 = cg * 8;

  for (int ck = 0; ck < nchunks; ++ck) {
    const int t0 = ck * C;
    const int Lc = min(C, a.T - t0);

    // ------------------------------------------------ pass 1: α quarter products
    float fw[4][8], bw[4][8], Pq[4][8];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int i = 16 * m + r16;
      const int t = t0 + i;
      float al[8];
      if (i < Lc) {
        const size_t gt = ((size_t)bi * a.T + t) * a.Hv + h;
        if (mode == GDN2_GATES_GDN) {
          const float s = __ldg(a.alpha + gt);
#pragma unroll
          for (int c = 0; c < 8; ++c) al[c] = s;
        } else {
          load8_f32(a.alpha + gt * D + ch0, al);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) al[c] = 1.f;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float x = al[c];   // forward inclusive product within the quarter
#pragma unroll
        for (int dd = 1; dd < 16; dd <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, dd, 16);
          if (r16 >= dd) x *= y;
        }
        fw[m][c] = x;
        Pq[m][c] = __shfl_sync(0xffffffffu, x, 15, 16);
        float z = al[c];   // backward inclusive product within the quarter
#pragma unroll
        for (int dd = 1; dd < 16; dd <<= 1) {
          const float y = __shfl_down_sync(0xffffffffu, z, dd, 16);
          if (r16 + dd < 16) z *= y;
        }
        const float zn = __shfl_down_sync(0xffffffffu, z, 1, 16);
        bw[m][c] = (r16 == 15) ? 1.f : zn;   // exclusive: Π_{s>i} within the quarter
      }
    }
    if (r16 == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c) sgC[ch0 + c] = Pq[0][c] * Pq[1][c] * Pq[2][c] * Pq[3][c];
    }
    // Smallest decay product whose reciprocal enters a Gram factor: fp16 Gram
    // operands when every factor stays below 2^14.
    bool gram_bf16;
    {
      float mn = 1.f;
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int c = 0; c < 8; ++c) mn = fminf(mn, (m & 1) ? fw[m][c] : bw[m][c]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      float* sred = reinterpret_cast<float*>(smem + OFF_RED);
      if (lane == 0) sred[warp] = mn;
      __syncthreads();
      float mall = sred[0];
#pragma unroll
      for (int w_ = 1; w_ < 8; ++w_) mall = fminf(mall, sred[w_]);
      gram_bf16 = !(mall > 6.103515625e-05f);   // 2^-14
    }

    // ------------------------------------------------ pass 2: operand tiles
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int i = 16 * m + r16;
      const int t = t0 + i;
      float kx[8], qx[8], ex[8], zx[8];
      if (i < Lc) {
        const size_t tq = ((size_t)bi * a.T + t) * a.Hqk + hq;
        const size_t gt = ((size_t)bi * a.T + t) * a.Hv + h;
        load8_bf16(kg + tq * D + ch0, kx);
        load8_bf16(qg + tq * D + ch0, qx);
        float bx[8], wx[8], vx[8];
        load8_bf16(vg + gt * D + ch0, vx);
        if (mode == GDN2_GATES_FULL) {
          load8_f32(a.b + gt * D + ch0, bx);
          load8_f32(a.w + gt * D + ch0, wx);
        } else {
          const float beta = __ldg(a.b + gt);
#pragma unroll
          for (int c = 0; c < 8; ++c) { bx[c] = beta; wx[c] = beta; }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          ex[c] = bx[c] * kx[c];
          zx[c] = wx[c] * vx[c];
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) { kx[c] = 0.f; qx[c] = 0.f; ex[c] = 0.f; zx[c] = 0.f; }
      }
      float o_eb[8], o_qb[8], o_ke[8], o_em[8], o_qm[8], o_km[8], o_x1[8], o_x2[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float pre = 1.f, suf = 1.f;
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
          if (mm < m) pre *= Pq[mm][c];
          if (mm > m) suf *= Pq[mm][c];
        }
        const float g = pre * fw[m][c];          // γ_i
        const float bk = bw[m][c] * suf;          // Π_{i<s≤63} α
        o_eb[c] = ex[c] * g;
        o_qb[c] = qx[c] * g;
        o_ke[c] = kx[c] * bk;
        // reference at the quarter boundary inside the half
        float fe, fk;
        if ((m & 1) == 0) {
          fe = __fdividef(1.f, bw[m][c]);
          fk = bw[m][c];
        } else {
          fe = fw[m][c];
          fk = __fdividef(1.f, fw[m][c]);
        }
        o_em[c] = ex[c] * fe;
        o_qm[c] = qx[c] * fe;
        o_km[c] = kx[c] * fk;
        // reference at the half boundary (token 31 | 32)
        if (m >= 2) {
          const float fq = (m == 3 ? Pq[2][c] : 1.f) * fw[m][c];
          o_x1[c] = ex[c] * fq;   // Ē_bnd
          o_x2[c] = qx[c] * fq;   // Q̄_bnd
        } else {
          const float fb = bw[m][c] * (m == 0 ? Pq[1][c] : 1.f);
          o_x1[c] = kx[c] * fb;   // K̃_bnd
          o_x2[c] = 0.f;
        }
      }
      st16(smem + OFF_EB, tile_off(i, ch0, D), pack8_f16(o_eb));
      st16(smem + OFF_QB, tile_off(i, ch0, D), pack8_f16(o_qb));
      st16(smem + OFF_KE, tile_off(i, ch0, D), pack8_f16(o_ke));
      st16(smem + OFF_Z, tile_off(i, ch0, D), pack8_f16(zx));
      st16(smem + OFF_GM, tile_off(i, ch0, D), pack8(o_em, gram_bf16));
      st16(smem + OFF_GM, tile_off(64 + i, ch0, D), pack8(o_qm, gram_bf16));
      st16(smem + OFF_KM, tile_off(i, ch0, D), pack8(o_km, gram_bf16));
      if (m >= 2) {
        st16(smem + OFF_GB, tile_off(i, ch0, D), pack8(o_x1, gram_bf16));
        st16(smem + OFF_GB, tile_off(64 + i, ch0, D), pack8(o_x2, gram_bf16));
      } else {
        st16(smem + OFF_KB, tile_off(i, ch0, D), pack8(o_x1, gram_bf16));
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // ------------------------------------------------ Gram MMAs
    if (tid == 0) {
      const uint32_t gm = smem_u32(smem + OFF_GM), km = smem_u32(smem + OFF_KM);
      const uint32_t gb = smem_u32(smem + OFF_GB), kb = smem_u32(smem + OFF_KB);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        mma16(tmem + TM_GM, desc_kmajor(gm + ks * 256, D), desc_kmajor(km + ks * 256, D),
              idesc_16(128, 64, false, false, gram_bf16), ks > 0);
        mma16(tmem + TM_GB, desc_kmajor(gb + ks * 256, D), desc_kmajor(kb + ks * 256, D),
              idesc_16(128, 32, false, false, gram_bf16), ks > 0);
      }
      mma_commit(bar);
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);

    // ------------------------------------------------ T and Aqk from TMEM
    float* sT = reinterpret_cast<float*>(smem + OFF_T);
    if (warp < 4) {
      // lanes 0..63: T rows; lanes 64..127: Aqk rows
      const bool is_t = row < 64;
      const int i = row & 63;
      float dm[64], db[32];
#pragma unroll
      for (int cb = 0; cb < 64; cb += 16) tmem_ld16(t_lane + TM_GM + cb, dm + cb);
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) tmem_ld16(t_lane + TM_GB + cb, db + cb);
      tmem_wait_ld();
      float val[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const bool keep = is_t ? (j < i) : (j <= i);
        const bool same = (j >> 5) == (i >> 5);
        float x = same ? dm[j] : (j < 32 ? db[j & 31] : 0.f);
        val[j] = keep ? x : 0.f;
      }
      if (is_t) {
#pragma unroll
        for (int j = 0; j < 64; ++j) sT[i * TP + j] = val[j];
      } else {
#pragma unroll
        for (int j = 0; j < 64; j += 8) st16(smem + OFF_AQK, tile_off(i, j, C), pack8_f16(val + j));
      }
    }
    __syncthreads();

    // ------------------------------------------------ A = (I + T)⁻¹, blocked
    float* sI = reinterpret_cast<float*>(smem + OFF_INV);
    float* sX = reinterpret_cast<float*>(smem + OFF_TMP);
    // zero the strict upper triangle region we never write otherwise
    for (int idx = tid; idx < C * C; idx += NT) {
      const int i = idx >> 6, j = idx & 63;
      if (j > i) sI[i * TP + j] = 0.f;
    }
    // level 0: 16 × 16 diagonal blocks by forward substitution, one column per thread
    if (tid < 64) {
      const int blk = tid >> 4, j = tid & 15, base = blk * 16;
      float x[16];
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        float acc = (ii == j) ? 1.f : 0.f;
        if (ii > j) {
#pragma unroll
          for (int l = 0; l < 16; ++l)
            if (l >= j && l < ii) acc -= sT[(base + ii) * TP + base + l] * x[l];
        }
        x[ii] = (ii >= j) ? acc : 0.f;
      }
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) sI[(base + ii) * TP + base + j] = x[ii];
    }
    __syncthreads();
    // level 1: off-diagonal 16 × 16 block of each 32-half: X = −I22 T21 I11
    {
      // tmp = T21 · I11 for both halves: 2 × 256 outputs
      for (int o = tid; o < 512; o += NT) {
        const int hf = o >> 8, ii = (o >> 4) & 15, jj = o & 15;
        const int r0 = hf * 32 + 16, c0 = hf * 32;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc += sT[(r0 + ii) * TP + c0 + l] * sI[(c0 + l) * TP + c0 + jj];
        sX[(r0 + ii) * TP + c0 + jj] = acc;
      }
      __syncthreads();
      for (int o = tid; o < 512; o += NT) {
        const int hf = o >> 8, ii = (o >> 4) & 15, jj = o & 15;
        const int r0 = hf * 32 + 16, c0 = hf * 32;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc += sI[(r0 + ii) * TP + r0 + l] * sX[(r0 + l) * TP + c0 + jj];
        sI[(r0 + ii) * TP + c0 + jj] = -acc;
      }
      __syncthreads();
    }
    // level 2: lower-left 32 × 32 block: X = −I_QQ T_QP I_PP
    {
      for (int o = tid; o < 1024; o += NT) {
        const int ii = o >> 5, jj = o & 31;
        float acc = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) acc += sT[(32 + ii) * TP + l] * sI[l * TP + jj];
        sX[(32 + ii) * TP + jj] = acc;
      }
      __syncthreads();
      for (int o = tid; o < 1024; o += NT) {
        const int ii = o >> 5, jj = o & 31;
        float acc = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) acc += sI[(32 + ii) * TP + 32 + l] * sX[(32 + l) * TP + jj];
        sI[(32 + ii) * TP + jj] = -acc;
      }
      __syncthreads();
    }
    // pack A (fp16, [i][j], 64 columns)
    for (int o = tid; o < C * 8; o += NT) {
      const int i = o >> 3, j0 = (o & 7) * 8;
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = sI[i * TP + j0 + u];
      st16(smem + OFF_AINV, tile_off(i, j0, C), pack8_f16(x));
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // ------------------------------------------------ Yᵀ = Ēᵀ Aᵀ, U_wᵀ = Zᵀ Aᵀ
    if (tid == 0) {
      const uint32_t eb = smem_u32(smem + OFF_EB), z = smem_u32(smem + OFF_Z);
      const uint32_t ai = smem_u32(smem + OFF_AINV);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks) {
        const uint64_t bdesc = desc_kmajor(ai + ks * 256, C);
        mma16(tmem + TM_YT, desc_mnmajor(eb + ks * 2 * (D / 8) * 128, D), bdesc,
                 idesc_f16(128, 64, true, false), ks > 0);
        mma16(tmem + TM_UW, desc_mnmajor(z + ks * 2 * (D / 8) * 128, D), bdesc,
                 idesc_f16(128, 64, true, false), ks > 0);
      }
      mma_commit(bar);
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);

    // Yᵀ (TMEM, key lanes) → fp16 tile [key][tok] (an MN-major B operand)
    {
      const int c0 = lo ? 0 : 32;
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) {
        float v[16];
        tmem_ld16(t_lane + TM_YT + c0 + cb, v);
        tmem_wait_ld();
        st16(smem + OFF_YT, tile_off(row, c0 + cb, C), pack8_f16(v));
        st16(smem + OFF_YT, tile_off(row, c0 + cb + 8, C), pack8_f16(v + 8));
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // ------------------------------------------------ (Y S)ᵀ = Sᵀ Yᵀ, Oᵀ = Sᵀ Q̄ᵀ
    if (tid == 0) {
      const uint32_t st = smem_u32(smem + OFF_ST), yt = smem_u32(smem + OFF_YT);
      const uint32_t qb = smem_u32(smem + OFF_QB);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t adesc = desc_kmajor(st + ks * 256, D);
        mma16(tmem + TM_YS, adesc, desc_mnmajor(yt + ks * 2 * (C / 8) * 128, C),
                 idesc_f16(128, 64, false, true), ks > 0);
        mma16(tmem + TM_O, adesc, desc_kmajor(qb + ks * 256, D), idesc_f16(128, 64, false, false), ks > 0);
      }
      mma_commit(bar);
    }
    // meanwhile: Sᵀ ← Sᵀ Γ in TMEM (column c scaled by γ_C[c]); the running MMAs
    // read only the fp16 copy.
    {
      const int c0 = lo ? 0 : 64;
      for (int cb = c0; cb < c0 + 64; cb += 16) {
        float v[16];
        tmem_ld16(t_lane + TM_S + cb, v);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] *= sgC[cb + u];
        tmem_st16(t_lane + TM_S + cb, v);
      }
      tmem_wait_st();
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);

    // Uᵀ = U_wᵀ − (Y S)ᵀ → fp16 tile [dv][tok] (K-major A operand)
    {
      const int c0 = lo ? 0 : 32;
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) {
        float uw[16], ys[16];
        tmem_ld16(t_lane + TM_UW + c0 + cb, uw);
        tmem_ld16(t_lane + TM_YS + c0 + cb, ys);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) uw[u] -= ys[u];
        st16(smem + OFF_UT, tile_off(row, c0 + cb, C), pack8_f16(uw));
        st16(smem + OFF_UT, tile_off(row, c0 + cb + 8, C), pack8_f16(uw + 8));
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // ------------------------------------------------ Sᵀ += Uᵀ K_end, Oᵀ += Uᵀ Aqkᵀ
    if (tid == 0) {
      const uint32_t ut = smem_u32(smem + OFF_UT), ke = smem_u32(smem + OFF_KE);
      const uint32_t aq = smem_u32(smem + OFF_AQK);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks) {
        const uint64_t adesc = desc_kmajor(ut + ks * 256, C);
        mma16(tmem + TM_S, adesc, desc_mnmajor(ke + ks * 2 * (D / 8) * 128, D),
                 idesc_f16(128, 128, false, true), 1);
        mma16(tmem + TM_O, adesc, desc_kmajor(aq + ks * 256, C), idesc_f16(128, 64, false, false), 1);
      }
      mma_commit(bar);
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);

    // outputs: thread (dv j) writes o[t0 + i][h][j]
    {
      const int c0 = lo ? 0 : 32;
      TOut* orow = og + (((size_t)bi * a.T + t0) * a.Hv + h) * D + row;
      const size_t tstride = (size_t)a.Hv * D;
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) {
        float v[16];
        tmem_ld16(t_lane + TM_O + c0 + cb, v);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int i = c0 + cb + u;
          if (i < Lc) orow[(size_t)i * tstride] = from_f32<TOut>(a.scale * v[u]);
        }
      }
    }
    // next chunk's fp16 Sᵀ operand
    {
      const int c0 = lo ? 0 : 64;
      for (int cb = c0; cb < c0 + 64; cb += 16) {
        float v[16];
        tmem_ld16(t_lane + TM_S + cb, v);
        tmem_wait_ld();
        st16(smem + OFF_ST, tile_off(row, cb, D), pack8_f16(v));
        st16(smem + OFF_ST, tile_off(row, cb + 8, D), pack8_f16(v + 8));
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (*sflag) break;
  }

  // ---------------------------------------------------------------- final state
  if (a.ST && !*sflag) {
    const int c0 = lo ? 0 : 64;
    float* ST = a.ST + (size_t)bh * D * D;
    for (int cb = c0; cb < c0 + 64; cb += 16) {
      float v[16];
      tmem_ld16(t_lane + TM_S + cb, v);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 16; ++u) ST[(size_t)(cb + u) * D + row] = v[u];
    }
  }
  if (*sflag && tid == 0 && a.workspace) atomicOr(static_cast<int*>(a.workspace), 1);
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs& a, int qkv_bf16) {
  return qkv_bf16 && a.dk == D && a.dv == D && a.chunk == C && a.conv_w == nullptr && !a.l2norm;
}

size_t chunk_tc_workspace(const ChunkArgs&) { return 256; }

cudaError_t launch_chunk_tc(const ChunkArgs& a, int o_bf16, cudaStream_t s) {
  const int grid = a.B * a.Hv;
  cudaError_t e = cudaMemsetAsync(a.workspace, 0, sizeof(int), s);
  if (e != cudaSuccess || grid == 0) return e;
  if (o_bf16) {
    auto k = chunk_tc_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    k<<<grid, NT, SMEM_BYTES, s>>>(a);
  } else {
    auto k = chunk_tc_kernel<float>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    k<<<grid, NT, SMEM_BYTES, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace gdn2
