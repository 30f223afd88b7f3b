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
//   * prep: persistent CTAs over the (chunk, sequence, value head) items,
//     all independent. Per item it builds T and Aqk (tensor cores), inverts
//     I + T (fp32 blocks, then a tensor-core merge), forms Yᵀ and U_wᵀ
//     (tensor cores) and writes the chunk's scan operands — −Yᵀ, −Q̄ᵀ, U_wᵀ,
//     K_end, −Aqk as fp16 tiles already in the MMA shared-memory layout, and
//     γ_C — to one 73 KB workspace slot, every tile by a bulk copy.
//   * scan: one CTA per (sequence, value head) walks the chunks in order. It
//     streams the slots into shared memory with bulk copies (double-buffered,
//     chunk c+1 in flight while c computes) and holds the state transposed,
//     Sᵀ in tensor memory with one value column per lane, so that the state
//     and U are A operands read from tensor memory and the slot's tiles are B
//     operands read from shared memory as the prep wrote them:
//         Dᵀ = Sᵀ (−Zᵀ), Zᵀ = [Yᵀ | Q̄ᵀ]  (columns 0..63: −(Y S)ᵀ; 64..127: −(Q̄ S)ᵀ)
//         Uᵀ = U_wᵀ + Dᵀ[:, 0..63],   Sᵀ ← Sᵀ Γ + Uᵀ K_end,
//         Dᵀ[:, 64..127] += Uᵀ (−Aqkᵀ)  (= −Oᵀ / scale).
// Forms selected by the call's parameters: the depthwise causal conv and the
// L2 norm of q, k fused into the prep's load (with the conv's history from
// the caller before a sequence's first token), gates as bf16 logits (σ
// applied where they are read), α and b owned by the QK heads, and sequences
// of different lengths packed along T (items and scan CTAs find their
// sequence's chunks and tokens in offset tables passed with the launch). The
// prep has one compiled copy per combination, so that no form pays for
// another's addressing.
// All MMA operand tiles use the 128-byte-swizzled layout (see tc_prims.cuh),
// so that a warp writing or reading whole rows is free of bank conflicts.
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

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
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
constexpr int SL_YT = 0;              // −Yᵀ  fp16 [128 key][64 tok]  ┐ −Zᵀ = [−Yᵀ | −Q̄ᵀ]: the two
constexpr int SL_QT = 16384;          // −Q̄ᵀ  fp16 [128 key][64 tok]  ┘ 64-column blocks, BS 16384
constexpr int SL_UW = 32768;          // U_wᵀ fp16 [128 dv][64 tok]
constexpr int SL_KE = 49152;          // K_end fp16 [64 tok][128 key] BS 8192
constexpr int SL_AQ = 65536;          // −Aqk fp16 [64 i][64 j]
constexpr int SL_GC = 73728;          // γ_C  fp32 [128]
constexpr int SL_WM = 74240;          // max |U_w| over the chunk (fp32; 16 bytes)
constexpr int SLOT_USED = 74256;      // bytes copied per chunk
constexpr int SL_FLAG = SLOT_USED;    // int: 1 = the slot is written by the exact kernel (not copied)
constexpr int SLOT = 74752;           // slot stride (1 KB multiple)
static_assert(SL_QT == SL_YT + 16384 && SL_UW == SL_QT + 16384 && SL_KE == SL_UW + 16384 &&
                  SL_AQ == SL_KE + 16384 && SL_GC == SL_AQ + 8192 && SL_WM == SL_GC + 512 &&
                  SLOT_USED == SL_WM + 16,
              "slot layout: the head-shared tiles around the per-head U_w, then the per-head max");
// Least α product over an aligned 16-token quarter (per channel) that the
// prep's reciprocal factorisation takes; items below it run exactly.
constexpr float kStrongDecay = 5.421010862427522e-20f;   // 2^-64
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
// After the Gram MMAs, [24K, 63K) holds the fp32 arrays of the inverse,
// [0, 8K) the fp16 A = (I+T)⁻¹ (64 × 64), and [64K, 80K) Q̄ᵀ and [96K, 112K)
// K_end wait there for their bulk stores. Two CTAs of this layout fit one SM.
constexpr int P_GB = 0;
constexpr int P_KB = 0;
constexpr int P_PQ = 8192;            // quarter products [4][128] fp32
constexpr int P_RED = P_PQ + 4 * D * 4;
constexpr int P_SUMS = P_RED + 32;    // fused load: per-half sums of squares of k, q [2][64 tok][2] fp32
static_assert(P_SUMS + 2 * C * 2 * 4 <= 12288, "quarter products and sums must stay in the unused Gram rows");
constexpr int P_BETA = P_RED + 128;   // scalar β of the next item (TMA box: 64 tokens × 16 bytes of heads);
                                      // not with the fused load, whose sums use these bytes
static_assert(P_BETA % 128 == 0 && P_BETA + C * 16 <= 12288, "β box in the unused Gram rows");
constexpr int P_GM = 32768;
constexpr int P_KM = 65536;
constexpr int P_EB = 81920;
constexpr int P_Z = 98304;
constexpr int P_END = 114688;
constexpr int P_AINV = 0;
constexpr int P_KES = P_Z;            // K_end staged for its bulk store (Z is written after the store has read it)
constexpr int P_QTS = P_KM;           // Q̄ᵀ staged for its bulk store (after the Gram products have read K̃_mid)
constexpr int P_ALPHA = P_EB;         // α of the next item (fp32 [64 tok][128 ch], 32 KB), loaded by TMA once
                                      // the Y/U_w products have read Ē and Z; read by pass 1
static_assert(P_ALPHA + C * D * 4 == P_END, "α tile over the Ē and Z tiles");
constexpr int P_YS = P_GM;            // Yᵀ then U_wᵀ (16 KB each), staged for the bulk stores
constexpr int P_AQS = 16384;          // −Aqk (8 KB) staged for its bulk store: in Gb's block 1,
                                      // read only as don't-care rows by the level-2 products
// level-2 inverse tiles (fp16, 128-byte rows), in the Gram operand space
constexpr int P_L2I = 0;              // A11, MN-major B  (32 rows)
constexpr int P_L2P = 4096;           // P = T21 A11, MN-major B (32 rows)
constexpr int P_L2T = 8192;           // T21, K-major A (first 32 of 128 rows)
constexpr int P_L2J = 12288;          // A22, K-major A (first 32 of 128 rows)
static_assert(P_AQS >= P_L2J + 4096 && P_AQS + 8192 <= 32768, "staging of -Aqk clear of the level-2 tiles");
constexpr int TS = 68;                // fp32 row stride of T and its inverse
constexpr int P_T = 24576;            // T   [64][68] (after the Gram products; clear of −Aqk's staging)
constexpr int P_I = P_T + C * TS * 4; // inv [64][68]
constexpr int P_X = P_I + C * TS * 4; // tmp [32][36]
static_assert(P_T >= P_AQS + 8192 && P_X + 32 * 36 * 4 <= P_QTS, "prep smem overlap");
constexpr int P_BAR = P_END;
constexpr int P_TMEMP = P_BAR + 16;
constexpr int P_FLAG = P_TMEMP + 16;
constexpr int P_SMEM = P_FLAG + 16;
// prep TMEM columns
constexpr uint32_t PT_GM = 0, PT_GB = 64, PT_YT = 128, PT_UW = 192, PT_COLS = 256;
constexpr uint32_t PT_L2P = 0, PT_L2A = 64;   // level-2 inverse accumulators (after the Gram read-out)

__device__ __forceinline__ void st16(uint8_t* base, uint32_t off, uint4 v) {
  *reinterpret_cast<uint4*>(base + off) = v;
}
__device__ __forceinline__ void st8(uint8_t* base, uint32_t off, uint2 v) {
  *reinterpret_cast<uint2*>(base + off) = v;
}

// (element 0 in the low half; no address of the argument is taken, so that
// the packed words stay in registers whatever the inlining order)
__device__ __forceinline__ void unpack4_f16(uint2 u, float* x) {
  x[0] = __half2float(__ushort_as_half((unsigned short)(u.x & 0xffffu)));
  x[1] = __half2float(__ushort_as_half((unsigned short)(u.x >> 16)));
  x[2] = __half2float(__ushort_as_half((unsigned short)(u.y & 0xffffu)));
  x[3] = __half2float(__ushort_as_half((unsigned short)(u.y >> 16)));
}
// bf16 is the upper half of an fp32: widening is a shift.
__device__ __forceinline__ void unpack4_bf16(uint2 u, float* x) {
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xffff0000u);
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
  const uint16_t *k, *q, *v;      // bf16
};

// Gate of one token for 4 channels, or the token's scalar gate broadcast: the
// fp32 values, or σ of the bf16 logits (LG).
// σ(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh approximation: one
// special-function operation where the exponential and the reciprocal take
// two. For the erase and write strengths b, w only, which enter fp16 operand
// tiles whose rounding is of the same order as this form's error; the decay
// α, whose products compound over a chunk, keeps the exponential form.
__device__ __forceinline__ float sigmoid_tanh_f32(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

template <bool LG, bool FAST = false>
__device__ __forceinline__ float4 gate4(const float* g, size_t gt, int c0, bool per_channel) {
  if (!LG) {
    if (per_channel) return __ldg(reinterpret_cast<const float4*>(g + gt * D + c0));
    const float s = __ldg(g + gt);
    return make_float4(s, s, s, s);
  }
  const uint16_t* h = reinterpret_cast<const uint16_t*>(g);
  if (per_channel) {
    float x[4];
    unpack4_bf16(__ldg(reinterpret_cast<const uint2*>(h + gt * D + c0)), x);
    if (FAST)
      return make_float4(sigmoid_tanh_f32(x[0]), sigmoid_tanh_f32(x[1]), sigmoid_tanh_f32(x[2]), sigmoid_tanh_f32(x[3]));
    return make_float4(sigmoid_f32(x[0]), sigmoid_f32(x[1]), sigmoid_f32(x[2]), sigmoid_f32(x[3]));
  }
  const float s = sigmoid_f32(__uint_as_float((uint32_t)__ldg(h + gt) << 16));
  return make_float4(s, s, s, s);
}

// Where the slots of a launch live: chunk c_begin + j of sequence-head bh is
// slot bh · stride + off + j of the workspace (stride: slots per
// sequence-head in the workspace; off: the launch's first chunk there).
// Packed sequences of different lengths: the nc chunks of sequence n, value
// head h are slots cu_chk[n] · H_v + h · nc + j.
struct SlotMap {
  int stride, off;
};
__device__ __forceinline__ size_t slot_index(SlotMap m, int bh, int j) {
  return (size_t)bh * m.stride + m.off + j;
}

// A work item: chunk cl of sequence bi (bh = bi · H_v + h), tokens t0 .. t0 +
// Lc − 1 of the q, k, v buffers (bi is 0 for packed sequences, whose t0 is
// already in the packed stream), and its slot. With groups of G value heads
// per item (the heads reading one QK head, when α and b belong to it), h is
// the group's first head and the group's slots are slot + g · hstride.
struct Item {
  int bh, cl, h, bi, hq, t0, Lc;
  size_t slot, hstride;
};
template <bool VL, bool GROUPS = false>
__device__ __forceinline__ Item decode_item(const ChunkArgs& a, int c_begin, int item, SlotMap sm) {
  Item it;
  // GROUPS: one item per group of G = H_v / H_qk value heads (ng per sequence)
  const int G = GROUPS ? a.Hv / a.Hqk : 1;
  const int ng = GROUPS ? a.Hqk : a.Hv;
  if (VL) {
    // item = global chunk · ng + head group; the sequence is the last n with
    // cu_chk[n] ≤ the chunk (empty sequences own no chunk and are passed over)
    it.h = GROUPS ? (item % ng) * G : item % a.Hv;
    const int g = item / ng;
    int lo = 0, hi = a.nseq;            // cu_chk[lo] ≤ g < cu_chk[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.cu_chk[mid] <= g) lo = mid; else hi = mid;
    }
    const int nc = a.cu_chk[lo + 1] - a.cu_chk[lo];
    it.bi = 0;
    it.bh = lo * a.Hv + it.h;
    it.cl = g - a.cu_chk[lo];
    it.hq = it.h / (a.Hv / a.Hqk);
    it.t0 = a.cu_tok[lo] + it.cl * C;
    it.Lc = min(C, a.cu_tok[lo + 1] - it.t0);
    it.slot = (size_t)a.cu_chk[lo] * a.Hv + (size_t)it.h * nc + it.cl;
    it.hstride = (size_t)nc;
  } else if (GROUPS) {
    const int r = item % (a.B * ng);  // QK head fastest
    it.cl = item / (a.B * ng);
    it.bi = r / ng;
    it.h = (r % ng) * G;
    it.bh = it.bi * a.Hv + it.h;
    it.hq = it.h / (a.Hv / a.Hqk);
    it.t0 = (c_begin + it.cl) * C;
    it.Lc = min(C, a.T - it.t0);
    it.slot = slot_index(sm, it.bh, it.cl);
    it.hstride = (size_t)sm.stride;
  } else {
    it.bh = item % (a.B * a.Hv);      // value head fastest: heads sharing q, k run together
    it.cl = item / (a.B * a.Hv);
    it.h = it.bh % a.Hv;
    it.bi = it.bh / a.Hv;
    it.hq = it.h / (a.Hv / a.Hqk);
    it.t0 = (c_begin + it.cl) * C;
    it.Lc = min(C, a.T - it.t0);
    it.slot = slot_index(sm, it.bh, it.cl);
    it.hstride = (size_t)sm.stride;
  }
  return it;
}

// Items are taken in order (chunk-major, value head fastest): by a fixed stride
// of the grid, or, with `counter`, one at a time from that device counter
// (zero before the launch), so that CTAs which start late take fewer.
// CV: the depthwise causal conv and/or the L2 norm of q, k are fused into the
// load (see the fused-load steps below); LG: the gates are bf16 logits; QKG:
// alpha and b belong to the QK heads; VL: sequences of different lengths
// packed along T (one compiled copy each, so that no form pays for the
// others' addressing at the register limit).
// Gates that come by TMA, one item ahead (bits of `tgates`): the per-channel α tile;
// a box of scalar α (Gated DeltaNet layout); a box of scalar β (tied layouts,
// b = w = β). Each box holds the item's 64 tokens × 16 bytes of heads.
// The boxes exist in a compiled copy of their own (BOX), so that the
// per-channel copies carry none of their code.
constexpr int TG_ATILE = 1, TG_ABOX = 2, TG_BBOX = 4;
template <bool CV, bool LG, bool QKG, bool VL, bool BOX>
__global__ void __launch_bounds__(NP, 2) chunk_prep_kernel(ChunkArgs a, int c_begin, int n_seg, SlotMap sm,
                                                           int* counter, const __grid_constant__ CUtensorMap amap,
                                                           const __grid_constant__ CUtensorMap bmap, int tgates) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + P_BAR);
  uint64_t* bar_a = bar + 1;            // the α tile has landed
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + P_TMEMP);
  int* sflag = reinterpret_cast<int*>(smem + P_FLAG);
  float* sPq = reinterpret_cast<float*>(smem + P_PQ);
  float* sred = reinterpret_cast<float*>(smem + P_RED);
  float* sT = reinterpret_cast<float*>(smem + P_T);
  float* sI = reinterpret_cast<float*>(smem + P_I);
  float* sX = reinterpret_cast<float*>(smem + P_X);

  int* s_item = sflag + 1;               // the next item, when taken from the counter
  uint32_t* s_wmax = reinterpret_cast<uint32_t*>(sflag + 2);   // max |U_w| of the item (float bits)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // QKG: one item per (chunk, sequence, QK head), for its G value heads
  const int G = QKG ? a.Hv / a.Hqk : 1;
  const int n_items = (VL ? a.cu_chk[a.nseq] * a.Hv : a.B * a.Hv * n_seg) / G;
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_a, 1);
    fence_mbar_init();
    *sflag = 0;
    *s_item = counter ? atomicAdd(counter, 1) : 0;
    *s_wmax = 0;
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
  const PrepSrc src{a.alpha, a.b, full ? a.w : a.b, static_cast<const uint16_t*>(a.k),
                    static_cast<const uint16_t*>(a.q), static_cast<const uint16_t*>(a.v)};

  // Input schedule of an item: α of the thread's 8 tokens and the key side
  // (b, k, q) of tokens 0..3 first; the key side of token u + 4 as soon as
  // token u is packed (its registers are free); w and v after pass 2, their
  // latency covered by the Gram products. (Requesting the next item's inputs
  // earlier than this needs registers the 2-CTA/SM budget does not have.)
  float f[8][4];                   // α, then its forward products within the quarter
  float4 bq[4];
  uint2 kk[4], qq[4];
  // rows of alpha, b (per value head, or shared per QK head) and of w
  auto gate_row = [&](const Item& it, int u) -> size_t {
    const size_t r = (size_t)it.bi * a.T + it.t0 + i0 + u;
    return QKG ? r * a.Hqk + it.hq : r * a.Hv + it.h;
  };
  auto w_row = [&](const Item& it, int hv, int u) -> size_t {   // w of value head hv
    return full ? ((size_t)it.bi * a.T + it.t0 + i0 + u) * a.Hv + hv : gate_row(it, u);
  };
  auto qkv_tok = [&](const Item& it, int u) -> size_t {
    return (size_t)it.bi * a.T + it.t0 + i0 + u;
  };
  constexpr int GE = LG ? 8 : 4;       // gate values per 16 bytes
  // a scalar gate of token row u of the item from a box (σ of a logit)
  auto box_gate = [&](const Item& it, int off, int u) -> float {
    const int col = (QKG ? it.hq : it.h) % GE;
    if (LG) return sigmoid_f32(__uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(smem + off + u * 16 + col * 2) << 16));
    return *reinterpret_cast<const float*>(smem + off + u * 16 + col * 4);
  };
  auto load_key1 = [&](const Item& it, int u, int s) {
    const bool ok = it.Lc == C || i0 + u < it.Lc;
    const size_t tq = qkv_tok(it, u) * a.Hqk + it.hq;
    if (BOX && (tgates & TG_BBOX)) {
      const float bt = ok ? box_gate(it, P_BETA, i0 + u) : 0.f;
      bq[s] = make_float4(bt, bt, bt, bt);
    } else {
      bq[s] = ok ? gate4<LG, true>(src.b, gate_row(it, u), c0, full) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if constexpr (!CV) {   // (CV: k and q come from pass 0)
      kk[s] = ok ? __ldg(reinterpret_cast<const uint2*>(src.k + tq * D + c0)) : make_uint2(0, 0);
      qq[s] = ok ? __ldg(reinterpret_cast<const uint2*>(src.q + tq * D + c0)) : make_uint2(0, 0);
    }
  };
  // The per-channel α tile of an item comes by one TMA copy (rows of the
  // tensor map [B·T][H_g][128]), requested by thread 0 one item ahead; so do
  // the boxes of scalar gates (rows of [B·T][H_g], the 16-byte column block
  // that holds the item's head).
  auto fetch_alpha = [&](int item_) {
    const Item nx = decode_item<VL, QKG>(a, c_begin, item_, sm);
    const int hg = QKG ? nx.hq : nx.h;
    const int row = nx.bi * a.T + nx.t0;
    mbar_arrive_expect_tx(bar_a, ((tgates & TG_ATILE) ? C * D * (LG ? 2 : 4) : 0) + ((BOX && (tgates & TG_ABOX)) ? C * 16 : 0) +
                                     ((BOX && (tgates & TG_BBOX)) ? C * 16 : 0));
    if (tgates & TG_ATILE) tma_load_3d(smem + P_ALPHA, &amap, 0, hg, row, bar_a);
    if constexpr (BOX) {
      if (tgates & TG_ABOX) tma_load_2d(smem + P_ALPHA, &amap, hg / GE * GE, row, bar_a);
      if (tgates & TG_BBOX) tma_load_2d(smem + P_BETA, &bmap, hg / GE * GE, row, bar_a);
    }
  };
  uint32_t phase_a = 0;
  auto load_alpha_key0 = [&](int item_) {
    const Item it = decode_item<VL, QKG>(a, c_begin, item_, sm);
    if (BOX && (tgates & TG_BBOX)) {
      wait_mma(bar_a, phase_a, sflag);   // (β of the key side is in the box)
#pragma unroll
      for (int u = 0; u < 4; ++u) load_key1(it, u, u);
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) load_key1(it, u, u);
      if (tgates) wait_mma(bar_a, phase_a, sflag);
    }
    if (BOX && (tgates & TG_ABOX)) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool ok = it.Lc == C || i0 + u < it.Lc;    // rows past the sequence's end: α = 1
        const float al = ok ? box_gate(it, P_ALPHA, i0 + u) : 1.f;
        f[u][0] = al; f[u][1] = al; f[u][2] = al; f[u][3] = al;
      }
    } else if (tgates & TG_ATILE) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool ok = it.Lc == C || i0 + u < it.Lc;    // rows past the sequence's end: α = 1
        float4 al = make_float4(1.f, 1.f, 1.f, 1.f);
        if (ok && LG) {
          float x[4];
          unpack4_bf16(*reinterpret_cast<const uint2*>(smem + P_ALPHA + (i0 + u) * (D * 2) + c0 * 2), x);
          al = make_float4(sigmoid_f32(x[0]), sigmoid_f32(x[1]), sigmoid_f32(x[2]), sigmoid_f32(x[3]));
        } else if (ok) {
          al = *reinterpret_cast<const float4*>(smem + P_ALPHA + (i0 + u) * (D * 4) + c0 * 4);
        }
        f[u][0] = al.x; f[u][1] = al.y; f[u][2] = al.z; f[u][3] = al.w;
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool ok = it.Lc == C || i0 + u < it.Lc;
        const float4 al = ok ? gate4<LG>(src.alpha, gate_row(it, u), c0, alpha_pc) : make_float4(1.f, 1.f, 1.f, 1.f);
        f[u][0] = al.x; f[u][1] = al.y; f[u][2] = al.z; f[u][3] = al.w;
      }
    }
  };

  // ---- fused load (CV). Raw bf16 rows of 4 channels: token t0 + r of the
  // item's row of tokens, the sequence's conv history for tokens before its
  // first one (zeros without a history), zeros past its end.
  const uint16_t* hist = static_cast<const uint16_t*>(a.conv_in);
  const size_t hrow = (size_t)(2 * a.Hqk + a.Hv) * D;
  auto raw4 = [&](const uint16_t* base, int H, int hh, int choff, const Item& it, int r) -> uint2 {
    const int t = it.t0 + r;
    const int sq = VL ? it.bh / a.Hv : it.bi;   // the sequence (its history row)
    const int seq0 = VL ? a.cu_tok[sq] : 0;     // and its first token in the row of tokens
    if (t >= seq0) {
      if (r >= it.Lc) return make_uint2(0, 0);
      return __ldg(reinterpret_cast<const uint2*>(base + (((size_t)it.bi * a.T + t) * H + hh) * D + c0));
    }
    if (hist == nullptr) return make_uint2(0, 0);
    return __ldg(reinterpret_cast<const uint2*>(hist + ((size_t)sq * 3 + 3 + (t - seq0)) * hrow + choff + c0));
  };
  // Channel c of y_t = Σ_j W[c][j] · x_{t−3+j}: x holds the raw rows of
  // tokens t−3 .. t (in x[u] .. x[u + 3]), W the taps of the 4 channels.
  auto conv4 = [](const uint2* x, int u, const float4* W, float* y) {
    float x0[4], x1[4], x2[4], x3[4];
    unpack4_bf16(x[u], x0);
    unpack4_bf16(x[u + 1], x1);
    unpack4_bf16(x[u + 2], x2);
    unpack4_bf16(x[u + 3], x3);
    y[0] = W[0].x * x0[0] + W[0].y * x1[0] + W[0].z * x2[0] + W[0].w * x3[0];
    y[1] = W[1].x * x0[1] + W[1].y * x1[1] + W[1].z * x2[1] + W[1].w * x3[1];
    y[2] = W[2].x * x0[2] + W[2].y * x1[2] + W[2].z * x2[2] + W[2].w * x3[2];
    y[3] = W[3].x * x0[3] + W[3].y * x1[3] + W[3].z * x2[3] + W[3].w * x3[3];
  };
  float* ssum = reinterpret_cast<float*>(smem + P_SUMS);   // [k, q][64 tokens][channel half]
  // Pass 0 (CV): k and q of the thread's 8 tokens and 4 channels, convolved,
  // stored un-normalised as fp16 in exactly the bytes of the Gm tile (Ē and Q̄
  // halves) that this thread overwrites in pass 2 after reading them back; the
  // token's sum of squares over the warp's 64 channels to shared memory (the
  // two channel halves are added, and the norm applied, in pass 2, after the
  // barrier that follows pass 1).
  // (the raw rows of both k and q are requested before the wait for the
  // previous item's stores, so that their latency overlaps it)
  auto fused_qk = [&](const Item& it) {
    const bool conv = a.conv_w != nullptr;
    uint2 xs[2][11];
#pragma unroll
    for (int arr = 0; arr < 2; ++arr) {
#pragma unroll
      for (int j = 0; j < 11; ++j)
        xs[arr][j] = (conv || j >= 3) ? raw4(arr == 0 ? src.k : src.q, a.Hqk, it.hq,
                                             (arr == 0 ? a.Hqk * D : 0) + it.hq * D, it, i0 - 3 + j)
                                      : make_uint2(0, 0);
    }
    // the previous item's stores still read the Gram space: wait, then fill it
    if (tid == 0) bulk_wait_read_all();
    __syncthreads();
#pragma unroll
    for (int arr = 0; arr < 2; ++arr) {
      const int choff = (arr == 0 ? a.Hqk * D : 0) + it.hq * D;
      const uint2* x = xs[arr];
      float4 W[4];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        W[c] = conv ? __ldg(reinterpret_cast<const float4*>(a.conv_w + (size_t)(choff + c0 + c) * 4))
                    : make_float4(0.f, 0.f, 0.f, 1.f);
      float ss[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float y[4];
        conv4(x, u, W, y);
        ss[u] = y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3];
        st8(smem, P_GM + (arr ? 64 * 128 : 0) + (uint32_t)(i0 + u) * 128 + piece(u, BS_ROW128),
            pack4_f16(y[0], y[1], y[2], y[3]));
      }
      if (a.l2norm) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
#pragma unroll
          for (int off = 1; off < 16; off <<= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
        }
        if (cg == 0) {
#pragma unroll
          for (int u = 0; u < 8; ++u) ssum[(arr * C + i0 + u) * 2 + (warp & 1)] = ss[u];
        }
      }
    }
  };

  uint32_t phase = 0;
  if (tgates && tid == 0 && (counter ? *s_item : (int)blockIdx.x) < n_items)
    fetch_alpha(counter ? *s_item : (int)blockIdx.x);
  for (int item = counter ? *s_item : (int)blockIdx.x; item < n_items;) {
    const Item it = decode_item<VL, QKG>(a, c_begin, item, sm);
    uint8_t* slot = static_cast<uint8_t*>(a.workspace) + WS_HEAD + it.slot * SLOT;
    if constexpr (CV) fused_qk(it);
    load_alpha_key0(item);

    // -------- pass 1: α's forward products within the quarter
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
    if (tid == 0) bulk_wait_read_all();   // the previous item's Yᵀ, U_wᵀ staging is read
    __syncthreads();
    // every thread has read s_item for this item (at the end of the previous one)
    if (counter && tid == 0) *s_item = atomicAdd(counter, 1);

    bool gram_bf16, exact;
    {
      float mall = sred[0];
#pragma unroll
      for (int w_ = 1; w_ < NP / 32; ++w_) mall = fminf(mall, sred[w_]);
      // every in-quarter forward/backward product is ≥ the quarter product
      gram_bf16 = !(mall > 6.103515625e-05f);   // 2^-14
      // Below 2^-64 the reciprocal factors of the Gram operands leave the
      // fp32 range (and an α product that underflows makes them inf): the
      // item goes to the exact kernel (chunk_fix_kernel), which writes its
      // slot before the scan reads it. The comparison is false for NaN too.
      exact = !(mall >= kStrongDecay);
    }
    if (exact) {
      if (tid == 0)
        for (int g = 0; g < G; ++g) *reinterpret_cast<int*>(slot + (size_t)g * it.hstride * SLOT + SL_FLAG) = 1;
      // every thread has read the quarter minima and α (pass 1); thread 0's
      // s_item is visible after this barrier
      __syncthreads();
      const int nx = counter ? *s_item : item + (int)gridDim.x;
      if (tgates && tid == 0 && nx < n_items) fetch_alpha(nx);
      item = nx;
      continue;
    }
    if (tid < D) {
      const float g = sPq[tid] * sPq[D + tid] * sPq[2 * D + tid] * sPq[3 * D + tid];
      reinterpret_cast<float*>(slot + SL_GC)[tid] = g;
    }
    // Per-channel factors of quarter qt from the quarter products P_m:
    //   γ_i = pre · f_i,                      pre = Π_{m<qt} P_m  (held negated: see below)
    //   Π_{i<s≤63} α = (P_qt · suf) / f_i,      suf = Π_{m>qt} P_m
    //   mid-reference factors: f_i / P_qt and P_qt / f_i (first quarter of a
    //   half), f_i and 1 / f_i (second quarter);
    //   half-boundary factors: P_2 f_i (quarter 3), f_i (quarter 2) for rows
    //   of the second half; P_qt P_1 / f_i (quarter 0), P_qt / f_i (quarter 1)
    //   for keys of the first half. In every quarter these are the
    //   mid-reference factor times one constant: P_2 for rows (quarters 2,
    //   3), P_1 for keys (quarters 0, 1); likewise the K_end factor is the
    //   key's mid-reference factor times suf (even quarter) or P_qt · suf (odd).
    float pre[4], se[4], sk[4], ke[4], xb[4];
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
        pre[c] = -pr;                            // Ē and Q̄ leave with the sign the scan wants
        const bool even = (qt & 1) == 0;
        se[c] = even ? rcp_approx(own) : 1.f;
        sk[c] = even ? own : 1.f;
        ke[c] = even ? su : own * su;            // K_end row = K̃_mid row · ke
        xb[c] = qt >= 2 ? P[2][c] : P[1][c];     // boundary row = mid row · xb
      }
    }

    // -------- pass 2: key-side operand tiles, tile by tile per token; one
    // copy of the loop per Gram operand type, so each packs only its own
    uint32_t qpk[4][4];
    float qlo[4];
#define GDN2_TILE(dst, off, expr)                                             \
  {                                                                           \
    _Pragma("unroll") for (int c = 0; c < 4; ++c) o[c] = (expr);              \
    st8(dst, off, pack4_f16(o[0], o[1], o[2], o[3]));                         \
  }
#define GDN2_GRAM_TILE(dst, off, expr, BF)                                    \
  {                                                                           \
    _Pragma("unroll") for (int c = 0; c < 4; ++c) o[c] = (expr);              \
    st8(dst, off, (BF) ? pack4_bf16(o[0], o[1], o[2], o[3]) : pack4_f16(o[0], o[1], o[2], o[3])); \
  }
#define GDN2_PASS2(BF)                                                                          \
  _Pragma("unroll") for (int u = 0; u < 8; ++u) {                                               \
    const int uk = u & 3;                                                                       \
    const uint32_t i128 = (uint32_t)(i0 + u) * 128;                                             \
    const uint32_t p64 = i128 + piece(u, BS_ROW64), p128 = i128 + piece(u, BS_ROW128);          \
    float kx[4], qx[4], e[4], rf[4], g[4], fe[4], o[4];                                         \
    if constexpr (CV) {                                                                         \
      unpack4_f16(*reinterpret_cast<const uint2*>(smem + P_GM + p128), kx);                     \
      unpack4_f16(*reinterpret_cast<const uint2*>(smem + P_GM + 64 * 128 + p128), qx);          \
      if (a.l2norm) {                                                                           \
        const int ti = i0 + u;                                                                  \
        const float nk = rsqrtf(ssum[ti * 2] + ssum[ti * 2 + 1] + kL2Eps);                      \
        const float nq = rsqrtf(ssum[(C + ti) * 2] + ssum[(C + ti) * 2 + 1] + kL2Eps);          \
        _Pragma("unroll") for (int c = 0; c < 4; ++c) { kx[c] *= nk; qx[c] *= nq; }             \
      }                                                                                         \
    } else {                                                                                    \
      unpack4_bf16(kk[uk], kx);                                                                 \
      unpack4_bf16(qq[uk], qx);                                                                 \
    }                                                                                           \
    e[0] = bq[uk].x * kx[0]; e[1] = bq[uk].y * kx[1]; e[2] = bq[uk].z * kx[2]; e[3] = bq[uk].w * kx[3]; \
    _Pragma("unroll") for (int c = 0; c < 4; ++c) {                                             \
      rf[c] = rcp_approx(f[u][c]);                                                              \
      g[c] = pre[c] * f[u][c];                                                                  \
      fe[c] = se[c] * f[u][c];                                                                  \
    }                                                                                           \
    /* Q̄ᵀ: each key's token pairs packed as they are produced */                              \
    if ((u & 1) == 0) {                                                                         \
      _Pragma("unroll") for (int c = 0; c < 4; ++c) qlo[c] = qx[c] * g[c];                     \
    } else {                                                                                    \
      _Pragma("unroll") for (int c = 0; c < 4; ++c) qpk[c][u >> 1] = pack2_f16(qlo[c], qx[c] * g[c]); \
    }                                                                                           \
    float km[4], gme[4], gmq[4];                                                                \
    _Pragma("unroll") for (int c = 0; c < 4; ++c) {                                             \
      km[c] = kx[c] * (sk[c] * rf[c]);                                                          \
      gme[c] = e[c] * fe[c];                                                                    \
      gmq[c] = qx[c] * fe[c];                                                                   \
    }                                                                                           \
    GDN2_TILE(smem, P_KES + p64, km[c] * ke[c])                                                 \
    GDN2_TILE(smem, P_EB + p64, e[c] * g[c])                                                    \
    GDN2_GRAM_TILE(smem, P_GM + p128, gme[c], BF)                                               \
    GDN2_GRAM_TILE(smem, P_GM + 64 * 128 + p128, gmq[c], BF)                                    \
    GDN2_GRAM_TILE(smem, P_KM + p64, km[c], BF)                                                 \
    if (qt >= 2) {                                                                              \
      GDN2_GRAM_TILE(smem, P_GB + p128, gme[c] * xb[c], BF)                                     \
      GDN2_GRAM_TILE(smem, P_GB + 64 * 128 + p128, gmq[c] * xb[c], BF)                          \
    } else {                                                                                    \
      GDN2_GRAM_TILE(smem, P_KB + p128, km[c] * xb[c], BF)                                      \
    }                                                                                           \
    if (u < 4) load_key1(it, u + 4, u);                                                         \
  }
    if (gram_bf16) {
      GDN2_PASS2(true)
    } else {
      GDN2_PASS2(false)
    }
#undef GDN2_PASS2
#undef GDN2_GRAM_TILE
#undef GDN2_TILE
    // the write side of value head hv, consumed after the Gram products
    float4 wv[8];
    constexpr int NV = CV ? 11 : 8;   // CV: raw v of the 8 tokens and the 3 before them (conv at the Z step)
    uint2 vv[NV];
    auto load_write = [&](int hv) {
      const int choff_v = 2 * a.Hqk * D + hv * D;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool ok = it.Lc == C || i0 + u < it.Lc;
        if (BOX && (tgates & TG_BBOX)) {
          // tied: w = β, the same for every head of the group (QKG); from the
          // box for the first head, kept for the others (whose turn comes after
          // the inverse has reused the box's bytes)
          if (hv == it.h) {
            const float bt = ok ? box_gate(it, P_BETA, i0 + u) : 0.f;
            wv[u] = make_float4(bt, bt, bt, bt);
          }
        } else {
          wv[u] = ok ? gate4<LG, true>(src.w, w_row(it, hv, u), c0, full) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if constexpr (!CV)
          vv[u] = ok ? __ldg(reinterpret_cast<const uint2*>(src.v + (qkv_tok(it, u) * a.Hv + hv) * D + c0))
                     : make_uint2(0, 0);
      }
      if constexpr (CV) {
#pragma unroll
        for (int j = 0; j < NV; ++j)
          vv[j] = (a.conv_w != nullptr || j >= 3) ? raw4(src.v, a.Hv, hv, choff_v, it, i0 - 3 + j) : make_uint2(0, 0);
      }
    };
    // Z = w ⊙ v of value head hv (no decay) to its tile, read by the U_w
    // product (CV: v convolved here, from its raw rows)
    auto write_z = [&](int hv) {
      const int choff_v = 2 * a.Hqk * D + hv * D;
      float4 Wv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        Wv[c] = CV && a.conv_w ? __ldg(reinterpret_cast<const float4*>(a.conv_w + (size_t)(choff_v + c0 + c) * 4))
                               : make_float4(0.f, 0.f, 0.f, 1.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float vx[4];
        if constexpr (CV)
          conv4(vv, u, Wv, vx);
        else
          unpack4_bf16(vv[u], vx);
        st8(smem, P_Z + (uint32_t)(i0 + u) * 128 + piece(u, BS_ROW64),
            pack4_f16(wv[u].x * vx[0], wv[u].y * vx[1], wv[u].z * vx[2], wv[u].w * vx[3]));
      }
    };
    if constexpr (QKG) {
      load_write(it.h);
    } else {
      const int choff_v = 2 * a.Hqk * D + it.h * D;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool ok = it.Lc == C || i0 + u < it.Lc;
        if (BOX && (tgates & TG_BBOX)) {              // tied: w = β, from the box
          const float bt = ok ? box_gate(it, P_BETA, i0 + u) : 0.f;
          wv[u] = make_float4(bt, bt, bt, bt);
        } else {
          wv[u] = ok ? gate4<LG, true>(src.w, w_row(it, it.h, u), c0, full) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if constexpr (!CV)
          vv[u] = ok ? __ldg(reinterpret_cast<const uint2*>(src.v + (qkv_tok(it, u) * a.Hv + it.h) * D + c0))
                     : make_uint2(0, 0);
      }
      if constexpr (CV) {
#pragma unroll
        for (int j = 0; j < NV; ++j)
          vv[j] = (a.conv_w != nullptr || j >= 3) ? raw4(src.v, a.Hv, it.h, choff_v, it, i0 - 3 + j) : make_uint2(0, 0);
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
      bulk_s2g(slot + SL_KE, smem + P_KES, 16384);   // K_end, byte for byte the slot's layout
      bulk_commit();
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);
    // Q̄ᵀ [key][tok], staged: the thread's 8 tokens of each of its keys form one 16-byte chunk
#pragma unroll
    for (int c = 0; c < 4; ++c)
      st16(smem, P_QTS + sw_off(c0 + c, i0, BS_ROW128), make_uint4(qpk[c][0], qpk[c][1], qpk[c][2], qpk[c][3]));

    // -------- T (fp32, shared) and −Aqk (fp16, staged) from TMEM. Lanes
    // 0..63 hold rows of T, lanes 64..127 rows of Aqk; the two warps of a lane
    // quarter take 32 columns each. Every case is warp-uniform: a row i ≥ 32
    // against keys j < 32 takes the half-boundary product, the other pairs
    // the mid-reference product. The inverse reads only the strictly lower
    // part of T, so T is stored unmasked; Aqk is masked to j ≤ i.
    {
      const int i = row & 63;
      const int j0 = 32 * hc;
      const bool bnd = hc == 0 && i >= 32;
      const uint32_t col = bnd ? PT_GB : PT_GM + j0;
      float d[32];
      tmem_ld16(t_lane + col, d);
      tmem_ld16(t_lane + col + 16, d + 16);
      tmem_wait_ld();
      if (row < 64) {
#pragma unroll
        for (int u = 0; u < 32; u += 4)
          *reinterpret_cast<float4*>(sT + i * TS + j0 + u) = make_float4(d[u], d[u + 1], d[u + 2], d[u + 3]);
      } else {
        const int li = bnd ? 31 : (hc == 1 && i < 32 ? -1 : (i & 31));   // keep column u ≤ li
#pragma unroll
        for (int u = 0; u < 32; ++u) d[u] = u <= li ? -d[u] : 0.f;
#pragma unroll
        for (int cb = 0; cb < 32; cb += 8) st16(smem, P_AQS + sw_off(i, j0 + cb, BS_ROW64), pack8_f16(d + cb));
      }
    }
    fence_async_smem();
    if (tid == 0) bulk_wait_read_all();   // K_end's staging is read: the Z tile may be written
    __syncthreads();
    if (tid == 0) {
      bulk_s2g(slot + SL_AQ, smem + P_AQS, 8192);   // −Aqk and −Q̄ᵀ, byte for byte the slot's layout
      bulk_s2g(slot + SL_QT, smem + P_QTS, 16384);
      bulk_commit();
    }


    if constexpr (QKG) {
      write_z(it.h);
    } else {
      const int choff_v = 2 * a.Hqk * D + it.h * D;
      float4 Wv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        Wv[c] = CV && a.conv_w ? __ldg(reinterpret_cast<const float4*>(a.conv_w + (size_t)(choff_v + c0 + c) * 4))
                               : make_float4(0.f, 0.f, 0.f, 1.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float vx[4];
        if constexpr (CV)
          conv4(vv, u, Wv, vx);
        else
          unpack4_bf16(vv[u], vx);
        st8(smem, P_Z + (uint32_t)(i0 + u) * 128 + piece(u, BS_ROW64),
            pack4_f16(wv[u].x * vx[0], wv[u].y * vx[1], wv[u].z * vx[2], wv[u].w * vx[3]));
      }
    }

    // Gates as logits: the next item's rows of k, q, v (and of the bf16
    // logits of b and w when they are per channel) toward L2 while this
    // item's inverse and products run, so that its own loads of them, early in
    // its operand passes, wait on L2 rather than on DRAM. Every such row is
    // 256 bytes, two lines: thread t with t % 4 < 2 covers line t % 4 of
    // token row t / 4 (only rows the item reads). (With fp32 gates, QK-owned
    // gates or the conv in the load the same hint made the prep slower.)
    if constexpr (LG && !QKG && !CV) {
      const int nx = counter ? *s_item : item + (int)gridDim.x;
      const int tok = tid >> 2, sub = tid & 3;
      if (nx < n_items && sub < 2) {
        const Item nt = decode_item<VL, QKG>(a, c_begin, nx, sm);
        if (nt.Lc == C || tok < nt.Lc) {
          const size_t r = (size_t)nt.bi * a.T + nt.t0 + tok;
          const size_t qk_off = (r * a.Hqk + nt.hq) * D + sub * 64, v_off = (r * a.Hv + nt.h) * D + sub * 64;
          prefetch_l2(src.k + qk_off);
          prefetch_l2(src.q + qk_off);
          prefetch_l2(src.v + v_off);
          if (full) {
            prefetch_l2(reinterpret_cast<const uint16_t*>(src.b) + v_off);
            prefetch_l2(reinterpret_cast<const uint16_t*>(src.w) + v_off);
          }
        }
      }
    }

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
    // level 2 on the tensor cores: P = T21 A11, then A21 = −A22 P (32 × 32
    // blocks, fp16 operands, fp32 accumulation). The tiles live in the Gram
    // operand space, free since the Gram products: T21 and A22 are the first
    // 32 rows of two K-major 128-row A operands (the rows after them only
    // produce accumulator rows ≥ 32, which are not read), A11 and P are
    // 32-row MN-major B operands (their columns ≥ 32 only produce accumulator
    // columns ≥ 32).
    for (int q = tid; q < 384; q += NP) {
      const int t = q >> 7, r = (q >> 2) & 31, cb = (q & 3) * 8;
      const float* src = t == 0 ? sT + (32 + r) * TS + cb : (t == 1 ? sI + r * TS + cb : sI + (32 + r) * TS + 32 + cb);
      const float4 p0 = *reinterpret_cast<const float4*>(src);
      const float4 p1 = *reinterpret_cast<const float4*>(src + 4);
      const float x[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
      st16(smem, (t == 0 ? P_L2T : (t == 1 ? P_L2I : P_L2J)) + sw_off(r, cb, BS_ROW64), pack8_f16(x));
    }
    sync_for_mma();
    if (tid == 0) {
      const uint64_t a1 = desc_k_sw(smem_u32(smem + P_L2T), 0, BS_ROW64);
      const uint64_t b1 = desc_mn_sw(smem_u32(smem + P_L2I), 0, BS_ROW64);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        mma16(tmem + PT_L2P, a1 + k_step_sw(ks, BS_ROW64), b1 + mn_step_sw(ks), idesc_f16(128, 64, false, true), ks > 0);
      mma_commit(bar);
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);
    if (lq == 0) {   // P rows 0..31: TMEM lanes 0..31 (warps 0 and 4, 16 columns each)
      float v[16];
      tmem_ld16(t_lane + PT_L2P + 16 * hc, v);
      tmem_wait_ld();
      st16(smem, P_L2P + sw_off(lane, 16 * hc, BS_ROW64), pack8_f16(v));
      st16(smem, P_L2P + sw_off(lane, 16 * hc + 8, BS_ROW64), pack8_f16(v + 8));
    }
    sync_for_mma();
    if (tid == 0) {
      const uint64_t a2 = desc_k_sw(smem_u32(smem + P_L2J), 0, BS_ROW64);
      const uint64_t b2 = desc_mn_sw(smem_u32(smem + P_L2P), 0, BS_ROW64);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        mma16(tmem + PT_L2A, a2 + k_step_sw(ks, BS_ROW64), b2 + mn_step_sw(ks), idesc_f16(128, 64, false, true), ks > 0);
      mma_commit(bar);
    }
    __syncwarp();
    wait_mma(bar, phase, sflag);
    if (lq == 0) {   // A21 = −(A22 P): rows 32..63 of A, columns 0..31
      float v[16];
      tmem_ld16(t_lane + PT_L2A + 16 * hc, v);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 16; u += 4)
        *reinterpret_cast<float4*>(sI + (32 + lane) * TS + 16 * hc + u) = make_float4(-v[u], -v[u + 1], -v[u + 2], -v[u + 3]);
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

    // -------- −Yᵀ = −Ēᵀ Aᵀ, U_wᵀ = Zᵀ Aᵀ (Ē carries the sign, Z here is the write side w ⊙ v)
    if constexpr (!QKG) {
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
      // the products have read Ē and Z: their space takes the next item's α
      if (tgates && tid == 0) {
        const int nx = counter ? *s_item : item + (int)gridDim.x;
        if (nx < n_items) fetch_alpha(nx);
      }

      {
        // warps 0..3: Yᵀ rows (key lanes); warps 4..7: U_wᵀ rows (dv lanes),
        // staged in the (now free) Gram operand space and stored by two bulk
        // copies, byte for byte the slot's layout
        const uint32_t col = hc == 0 ? PT_YT : PT_UW;
        const int stg = P_YS + hc * 16384;
        uint32_t wm = 0;                 // max |U_w| (the scan scales its state by it)
#pragma unroll
        for (int cb0 = 0; cb0 < 64; cb0 += 32) {
          float v[32];
          tmem_ld16(t_lane + col + cb0, v);
          tmem_ld16(t_lane + col + cb0 + 16, v + 16);
          tmem_wait_ld();
#pragma unroll
          for (int cb = 0; cb < 32; cb += 8) st16(smem, stg + sw_off(row, cb0 + cb, BS_ROW128), pack8_f16(v + cb));
          if (hc == 1) {
#pragma unroll
            for (int u = 0; u < 32; ++u) wm = max(wm, __float_as_uint(v[u]) & 0x7fffffffu);
          }
        }
        if (hc == 1) {
          wm = __reduce_max_sync(0xffffffffu, wm);
          if (lane == 0) atomicMax(s_wmax, wm);
        }
      }
      fence_async_smem();
      fence_before_sync();
      __syncthreads();
      fence_after_sync();
      if (tid == 0) {
        bulk_s2g(slot + SL_YT, smem + P_YS, 16384);
        bulk_s2g(slot + SL_UW, smem + P_YS + 16384, 16384);
        bulk_commit();
        *reinterpret_cast<int*>(slot + SL_FLAG) = 0;   // written here, not by the exact kernel
        *reinterpret_cast<uint32_t*>(slot + SL_WM) = *s_wmax;
        *s_wmax = 0;                     // (the next item's maxima come after two barriers)
      }
    } else {
      // With α and b owned by the QK head (QKG) everything so far is shared by its
      // G value heads: the item makes U_w for each in turn (the next head's w, v
      // requested while the current product runs) and writes the shared tiles
      // once, to the slot of the group's first head, where every head's scan
      // reads them.
      for (int g = 0; g < G; ++g) {
        uint8_t* slot_g = slot + (size_t)g * it.hstride * SLOT;
        if (g > 0) {
          write_z(it.h + g);
          sync_for_mma();
        }
        if (tid == 0) {
          const uint64_t eb = desc_mn_sw(smem_u32(smem + P_EB), 0, BS_ROW64);
          const uint64_t z = desc_mn_sw(smem_u32(smem + P_Z), 0, BS_ROW64);
          const uint64_t ai = desc_k_sw(smem_u32(smem + P_AINV), 0, BS_ROW64);
          if (g == 0) {
  #pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
              mma16(tmem + PT_YT, eb + mn_step_sw(ks), ai + k_step_sw(ks, BS_ROW64), idesc_f16(128, 64, true, false),
                    ks > 0);
          }
  #pragma unroll
          for (int ks = 0; ks < C / 16; ++ks)
            mma16(tmem + PT_UW, z + mn_step_sw(ks), ai + k_step_sw(ks, BS_ROW64), idesc_f16(128, 64, true, false),
                  ks > 0);
          mma_commit(bar);
        }
        if (QKG && g + 1 < G) load_write(it.h + g + 1);   // (this thread's Z of head g is written)
        __syncwarp();
        wait_mma(bar, phase, sflag);
        // the products have read Ē and Z: their space takes the next item's α
        if (g == G - 1 && tgates && tid == 0) {
          const int nx = counter ? *s_item : item + (int)gridDim.x;
          if (nx < n_items) fetch_alpha(nx);
        }
        if (g > 0) {                       // the previous head's U_wᵀ staging has been read
          if (tid == 0) bulk_wait_read_all();
          __syncthreads();
        }
        if (g == 0 || hc == 1) {
          // warps 0..3: Yᵀ rows (key lanes; first head only); warps 4..7: U_wᵀ
          // rows (dv lanes), staged in the (now free) Gram operand space and
          // stored by bulk copies, byte for byte the slot's layout
          const uint32_t col = hc == 0 ? PT_YT : PT_UW;
          const int stg = P_YS + hc * 16384;
          uint32_t wm = 0;                 // max |U_w| (the scan scales its state by it)
  #pragma unroll
          for (int cb0 = 0; cb0 < 64; cb0 += 32) {
            float v[32];
            tmem_ld16(t_lane + col + cb0, v);
            tmem_ld16(t_lane + col + cb0 + 16, v + 16);
            tmem_wait_ld();
  #pragma unroll
            for (int cb = 0; cb < 32; cb += 8) st16(smem, stg + sw_off(row, cb0 + cb, BS_ROW128), pack8_f16(v + cb));
            if (hc == 1) {
  #pragma unroll
              for (int u = 0; u < 32; ++u) wm = max(wm, __float_as_uint(v[u]) & 0x7fffffffu);
            }
          }
          if (hc == 1) {
            wm = __reduce_max_sync(0xffffffffu, wm);
            if (lane == 0) atomicMax(s_wmax, wm);
          }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
          if (g == 0) bulk_s2g(slot + SL_YT, smem + P_YS, 16384);
          bulk_s2g(slot_g + SL_UW, smem + P_YS + 16384, 16384);
          bulk_commit();
          *reinterpret_cast<int*>(slot_g + SL_FLAG) = 0;   // written here, not by the exact kernel
          *reinterpret_cast<uint32_t*>(slot_g + SL_WM) = *s_wmax;
          *s_wmax = 0;                     // (the next maxima come after two barriers)
        }
      }
    }
    item = counter ? *s_item : item + (int)gridDim.x;   // written before the barriers above
  }
  if (tid == 0) bulk_wait_all();      // the last item's copies
  if (*sflag && tid == 0) atomicOr(static_cast<int*>(a.workspace), 1);
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, PT_COLS);
  // Launched beside the previous segment's scan, this grid completes only
  // after it: the next scan, ordered after this grid, then also follows that
  // scan (whose final state it reads).
  griddep_wait();
}

// =============================================================================
// Exact prep of the items the prep kernel flagged (decay too strong for its
// reciprocal factors). Same algebra and same slot contents, in fp32 with the
// decay of every pair formed as the running product Π_{j<s≤i} α_s — no
// reciprocal and no logarithm — so it holds for every α ∈ [0, 1]:
//     T_ij  = Σ_c e_ic k_jc Π_{j<s≤i} α_sc (j < i),  Aqk_ij likewise with q (j ≤ i)
//     A = (I + T)⁻¹ (forward substitution), Y = A (γ ⊙ e), U_w = A (w ⊙ v),
//     Q̄ = γ ⊙ q, K_end,j = k_j ⊙ Π_{j<s≤C} α_s, γ_C.
// One CTA reads the flags of FX_ITEMS consecutive items and does the flagged
// ones in turn; with nothing flagged it only reads the flags.
// =============================================================================
constexpr int FX_THREADS = 256;
constexpr int FX_ITEMS = 32;
constexpr int FX_LD = D + 4;          // fp32 row stride of the [64][128] arrays
constexpr int FX_TS = C + 1;          // fp32 row stride of the [64][64] arrays
constexpr size_t FX_SMEM = (size_t)(4 * C * FX_LD + 3 * C * FX_TS) * sizeof(float) + 16;   // + mask, max

template <bool VL>
__global__ void __launch_bounds__(FX_THREADS, 1) chunk_fix_kernel(ChunkArgs a, int c_begin, int n_seg, SlotMap sm) {
  extern __shared__ __align__(16) float fsm[];
  float* sAl = fsm;                     // α, later Z = w ⊙ v      [64][FX_LD]
  float* sE = sAl + C * FX_LD;          // e = b ⊙ k, later Ē = γ ⊙ e
  float* sK = sE + C * FX_LD;           // k, later K_end
  float* sQ = sK + C * FX_LD;           // q, later Q̄ = γ ⊙ q
  float* sT = sQ + C * FX_LD;           // T (strict lower)        [64][FX_TS]
  float* sAq = sT + C * FX_TS;          // Aqk (lower incl.)
  float* sI = sAq + C * FX_TS;          // (I + T)⁻¹
  uint32_t* smask = reinterpret_cast<uint32_t*>(sI + C * FX_TS);
  uint32_t* swm = smask + 1;            // max |U_w| of the item (float bits)

  const int tid = threadIdx.x;
  const int n_items = VL ? a.cu_chk[a.nseq] * a.Hv : a.B * a.Hv * n_seg;
  const int first = (int)blockIdx.x * FX_ITEMS;
  if (tid < 32) {
    const int item = first + tid;
    bool flagged = false;
    if (item < n_items) {
      const Item it = decode_item<VL>(a, c_begin, item, sm);
      const uint8_t* slot = static_cast<const uint8_t*>(a.workspace) + WS_HEAD + it.slot * SLOT;
      flagged = *reinterpret_cast<const volatile int*>(slot + SL_FLAG) != 0;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, flagged);
    if (tid == 0) *smask = m;
  }
  __syncthreads();
  uint32_t mask = *smask;
  if (mask == 0) return;

  const bool full = a.gate_mode == GDN2_GATES_FULL;
  const bool alpha_pc = a.gate_mode != GDN2_GATES_GDN;
  const bool lg = a.gate_logits != 0, qkg = a.Hg != a.Hv;
  const bool conv = a.conv_w != nullptr;
  const __nv_bfloat16* hist = static_cast<const __nv_bfloat16*>(a.conv_in);
  const size_t hrow = (size_t)(2 * a.Hqk + a.Hv) * D;
  // channel c of tensor x (H heads, head hh, conv channels from choff) at
  // token i of the item, after the conv when there is one: y_t = Σ_j W[c][j]
  // x_{t−3+j}, with the sequence's history rows before its first token
  auto in_val = [&](const void* x, int H, int hh, int choff, const Item& it, int i, int c) -> float {
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    const int sq = VL ? it.bh / a.Hv : it.bi;   // the sequence (its history row)
    const int seq0 = VL ? a.cu_tok[sq] : 0;     // and its first token in the row of tokens
    auto raw = [&](int r) -> float {
      const int t = it.t0 + r;
      if (t >= seq0) return __bfloat162float(xb[(((size_t)it.bi * a.T + t) * H + hh) * D + c]);
      return hist ? __bfloat162float(hist[((size_t)sq * 3 + 3 + (t - seq0)) * hrow + choff + c]) : 0.f;
    };
    if (!conv) return raw(i);
    const float4 W = __ldg(reinterpret_cast<const float4*>(a.conv_w + (size_t)(choff + c) * 4));
    return W.x * raw(i - 3) + W.y * raw(i - 2) + W.z * raw(i - 1) + W.w * raw(i);
  };

  while (mask) {
    const int bit = __ffs(mask) - 1;
    mask &= mask - 1;
    const Item it = decode_item<VL>(a, c_begin, first + bit, sm);
    uint8_t* slot = static_cast<uint8_t*>(a.workspace) + WS_HEAD + it.slot * SLOT;
    __syncthreads();   // the previous item's arrays (and its max) are read
    if (tid == 0) *swm = 0;

    // ---- inputs (tokens past the sequence's end: α = 1, everything else 0);
    // q, k after the conv, then L2-normalised by rows; then e = b ⊙ k
    for (int idx = tid; idx < C * D; idx += FX_THREADS) {
      const int i = idx / D, c = idx % D;
      float al = 1.f, bb = 0.f, kx = 0.f, qx = 0.f;
      if (i < it.Lc) {
        const size_t r = (size_t)it.bi * a.T + it.t0 + i;
        const size_t gr = qkg ? r * a.Hqk + it.hq : r * a.Hv + it.h;
        al = gate_at(a.alpha, alpha_pc ? gr * D + c : gr, lg);
        kx = in_val(a.k, a.Hqk, it.hq, a.Hqk * D + it.hq * D, it, i, c);
        qx = in_val(a.q, a.Hqk, it.hq, it.hq * D, it, i, c);
        bb = gate_at(a.b, full ? gr * D + c : gr, lg);
      }
      sAl[i * FX_LD + c] = al;
      sE[i * FX_LD + c] = bb;
      sK[i * FX_LD + c] = kx;
      sQ[i * FX_LD + c] = qx;
    }
    __syncthreads();
    if (a.l2norm) {
      const int lane = tid & 31;
      for (int row = tid >> 5; row < 2 * C; row += FX_THREADS / 32) {
        float* x = (row < C ? sK : sQ) + (row % C) * FX_LD;
        float ss = 0.f;
        for (int c = lane; c < D; c += 32) ss += x[c] * x[c];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = rsqrtf(ss + kL2Eps);
        for (int c = lane; c < D; c += 32) x[c] *= inv;
      }
      __syncthreads();
    }
    for (int idx = tid; idx < C * D; idx += FX_THREADS) {
      const int i = idx / D, c = idx % D;
      sE[i * FX_LD + c] *= sK[i * FX_LD + c];
    }
    __syncthreads();

    // ---- T and Aqk. Thread (j, part) runs down column j over its 32
    // channels c = 16m + 4·part + r, carrying Π_{j<s≤i} α_s per channel;
    // the four parts of a column are adjacent lanes and add by shuffles.
    {
      const int j = tid >> 2, part = tid & 3;
      float kj[32], dd[32];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float4 k4 = *reinterpret_cast<const float4*>(sK + j * FX_LD + 16 * m + 4 * part);
        kj[4 * m] = k4.x; kj[4 * m + 1] = k4.y; kj[4 * m + 2] = k4.z; kj[4 * m + 3] = k4.w;
      }
#pragma unroll
      for (int u = 0; u < 32; ++u) dd[u] = 1.f;
      for (int i = (tid >> 5) * 8; i < C; ++i) {      // from the warp's first column
        float at = 0.f, aa = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int off = i * FX_LD + 16 * m + 4 * part;
          const float4 al = *reinterpret_cast<const float4*>(sAl + off);
          const float4 e4 = *reinterpret_cast<const float4*>(sE + off);
          const float4 q4 = *reinterpret_cast<const float4*>(sQ + off);
          const float alv[4] = {al.x, al.y, al.z, al.w}, ev[4] = {e4.x, e4.y, e4.z, e4.w},
                      qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int u = 4 * m + r;
            dd[u] *= i > j ? alv[r] : 1.f;
            const float kd = kj[u] * dd[u];
            at = fmaf(ev[r], kd, at);
            aa = fmaf(qv[r], kd, aa);
          }
        }
        at += __shfl_xor_sync(0xffffffffu, at, 1);
        aa += __shfl_xor_sync(0xffffffffu, aa, 1);
        at += __shfl_xor_sync(0xffffffffu, at, 2);
        aa += __shfl_xor_sync(0xffffffffu, aa, 2);
        if (part == 0 && i >= j) {
          sT[i * FX_TS + j] = i > j ? at : 0.f;
          sAq[i * FX_TS + j] = aa;
        }
      }
    }
    __syncthreads();

    // ---- threads 0..127, channel c: γ_i (forward product), Ē, Q̄ in place;
    // K_end (backward product) and γ_C. Threads 128..191: column j of
    // (I + T)⁻¹ by forward substitution.
    if (tid < D) {
      const int c = tid;
      float g = 1.f;
      for (int i = 0; i < C; ++i) {
        g *= sAl[i * FX_LD + c];
        sE[i * FX_LD + c] *= g;
        sQ[i * FX_LD + c] *= g;
      }
      reinterpret_cast<float*>(slot + SL_GC)[c] = g;
      float p = 1.f;
      for (int j = C - 1; j >= 0; --j) {
        sK[j * FX_LD + c] *= p;
        p *= sAl[j * FX_LD + c];
      }
    } else if (tid < D + C) {
      const int j = tid - D;
      for (int i = 0; i < C; ++i) {
        float x = (i == j) ? 1.f : 0.f;
        if (i > j) {
          float acc = 0.f;
          for (int l = j; l < i; ++l) acc = fmaf(sT[i * FX_TS + l], sI[l * FX_TS + j], acc);
          x = -acc;
        }
        sI[i * FX_TS + j] = x;
      }
    }
    __syncthreads();
    // Z = w ⊙ v over the α array
    for (int idx = tid; idx < C * D; idx += FX_THREADS) {
      const int i = idx / D, c = idx % D;
      float z = 0.f;
      if (i < it.Lc) {
        const size_t r = (size_t)it.bi * a.T + it.t0 + i;
        const size_t wr = full ? (r * a.Hv + it.h) * D + c : (qkg ? r * a.Hqk + it.hq : r * a.Hv + it.h);
        z = gate_at(full ? a.w : a.b, wr, lg) * in_val(a.v, a.Hv, it.h, 2 * a.Hqk * D + it.h * D, it, i, c);
      }
      sAl[i * FX_LD + c] = z;
    }
    __syncthreads();

    // ---- −Yᵀ (threads 0..127) and U_wᵀ (128..255): row c of the [128][64]
    // fp16 tile, one thread each, from column c of Ē or Z.
    {
      const int c = tid & (D - 1);
      const bool yside = tid < D;
      const float* src = yside ? sE : sAl;
      float acc[C];
#pragma unroll
      for (int i = 0; i < C; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < C; ++j) {
        const float x = src[j * FX_LD + c];
#pragma unroll
        for (int i = j; i < C; ++i) acc[i] = fmaf(sI[i * FX_TS + j], x, acc[i]);
      }
      const float sg = yside ? -1.f : 1.f;
      uint8_t* dst = slot + (yside ? SL_YT : SL_UW);
      if (!yside) {
        uint32_t wm = 0;
#pragma unroll
        for (int i = 0; i < C; ++i) wm = max(wm, __float_as_uint(acc[i]) & 0x7fffffffu);
        wm = __reduce_max_sync(0xffffffffu, wm);
        if ((tid & 31) == 0) atomicMax(swm, wm);
      }
#pragma unroll
      for (int i0 = 0; i0 < C; i0 += 8) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = sg * acc[i0 + u];
        *reinterpret_cast<uint4*>(dst + sw_off(c, i0, BS_ROW128)) = pack8_f16(x);
      }
    }
    // −Q̄ᵀ: row c (key) of a [128][64] tile, threads 0..127
    if (tid < D) {
      const int c = tid;
#pragma unroll
      for (int i0 = 0; i0 < C; i0 += 8) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = -sQ[(i0 + u) * FX_LD + c];
        *reinterpret_cast<uint4*>(slot + SL_QT + sw_off(c, i0, BS_ROW128)) = pack8_f16(x);
      }
    }
    // K_end [64 tok][128 key]: 1024 pieces of 8 keys; −Aqk [64][64] masked j ≤ i: 512 pieces
    for (int pc = tid; pc < C * D / 8; pc += FX_THREADS) {
      const int j = pc >> 4, c0 = (pc & 15) * 8;
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = sK[j * FX_LD + c0 + u];
      *reinterpret_cast<uint4*>(slot + SL_KE + sw_off(j, c0, BS_ROW64)) = pack8_f16(x);
    }
    for (int pc = tid; pc < C * C / 8; pc += FX_THREADS) {
      const int i = pc >> 3, j0 = (pc & 7) * 8;
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = (j0 + u <= i) ? -sAq[i * FX_TS + j0 + u] : 0.f;
      *reinterpret_cast<uint4*>(slot + SL_AQ + sw_off(i, j0, BS_ROW64)) = pack8_f16(x);
    }
    __syncthreads();
    if (tid == 0) *reinterpret_cast<uint32_t*>(slot + SL_WM) = *swm;
  }
}

// =============================================================================
// scan kernel: one CTA per (sequence, value head), walking the chunks of the
// segment in order with the state held transposed: Sᵀ (d_v × d_k, fp32) lives
// in tensor memory with one value column of S per TMEM lane, so that both
// operands that change along the sweep (the state and U) are A operands read
// from tensor memory, and every chunk operand from the slot is a B operand
// read from shared memory as the slot holds it. Per chunk c, with
// Zᵀ = [Yᵀ | Q̄ᵀ] along the columns:
//   Dᵀ = Sᵀ (−Zᵀ)                  columns 0..63: −(Y S)ᵀ, 64..127: −(Q̄ S)ᵀ
//   Uᵀ = U_wᵀ + Dᵀ[:, 0..63]        (per lane, in the epilogue)
//   Sᵀ ← Sᵀ Γ + Uᵀ K_end            (TMEM holds Sᵀ Γ already)
//   Dᵀ[:, 64..127] += Uᵀ (−Aqkᵀ)    (= −Oᵀ / scale)
// The recurrence never mixes d_v columns, so each lane's row of Sᵀ carries its
// own block floating point scale. Four state warps (TMEM lane quarters;
// thread r = value column r) turn Dᵀ's U part into the 16-bit A operand Uᵀ
// and the new state into the 16-bit A operand Sᵀ (and back into TMEM times
// the next chunk's Γ); four output warps (the same lanes) read the finished
// chunks' outputs out of the other D buffer and store them; the last warp
// issues the products and the slot copies (one thread). No operand is
// written to shared memory during the sweep.
// =============================================================================
struct ScanLayout {
  static constexpr int STAGE = (SLOT_USED + 1023) / 1024 * 1024;   // one chunk's slot, byte for byte
  static constexpr int BAR = 2 * STAGE;          // 16 mbarriers
  static constexpr int KSC = BAR + 128;          // output scale per value column, chunks c mod 4: [4][128] fp32
  static constexpr int OST = KSC + 4 * 128 * 4;  // outputs of chunks c mod 2, staged [64 tok][128] (fp32 or bf16)
  static constexpr int FLAG = OST + 2 * C * D * 4;
  static constexpr int TMEMP = FLAG + 16;
  static constexpr int SMEM = TMEMP + 16;
  static constexpr int NE = 128;                 // state threads (one per value column)
  static constexpr int NO = 128;                 // output threads (one per value column)
  static constexpr int NS = NE + NO + 32;        // + the MMA warp
  // TMEM columns
  static constexpr uint32_t T_S = 0;             // Sᵀ fp32 [128 d_v lanes][128 keys]
  static constexpr uint32_t T_D = 128;           // Dᵀ fp32 [128][128 tokens], two buffers
  static constexpr uint32_t T_SH = 384;          // Sᵀ fp16, key pairs [128][64]
  static constexpr uint32_t T_UH = 448;          // Uᵀ fp16, token pairs [128][32]
  static constexpr uint32_t T_COLS = 512;
};
static_assert(ScanLayout::T_UH + 32 <= ScanLayout::T_COLS, "scan tensor memory");
static_assert(ScanLayout::SMEM <= 232448, "scan shared memory");

// pairs of fp32 values as fp16 pairs, 16 columns of a TMEM A operand
__device__ __forceinline__ void tmem_st16_f16(uint32_t taddr, const float* x) {
  float p[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) p[j] = __uint_as_float(pack2_f16(x[2 * j], x[2 * j + 1]));
  tmem_st16(taddr, p);
}

template <typename TOut> __device__ __forceinline__ void store_out(TOut* dst, float x);
template <> __device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* dst, float x) {
  *dst = __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ void store_out<float>(float* dst, float x) { *dst = x; }

// SHARED: α and b belong to the QK heads, and the tiles a QK head's value heads
// share sit in the slots of each group's first head (see the prep).
template <typename TOut, bool SHARED>
__global__ void __launch_bounds__(ScanLayout::NS, 1) chunk_scan_kernel(ChunkArgs a, int c_begin, int n_seg_arg,
                                                                      SlotMap sm, const float* S_in, float* S_out) {
  using L = ScanLayout;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR);
  uint64_t* full = bars;                // [2] stage s loaded
  uint64_t* b_d = bars + 2;             // Sᵀ(−Zᵀ) done
  uint64_t* b_u = bars + 3;             // fp16 Uᵀ written (one arrival per epilogue warp)
  uint64_t* b_s = bars + 4;             // state update done
  uint64_t* b_sh = bars + 5;            // fp16 Sᵀ written (one arrival per epilogue warp)
  uint64_t* b_o = bars + 6;             // [2] every product of the chunk in D buffer s done
  uint64_t* b_fin = bars + 8;           // the products issued before a give-up have completed
  uint64_t* b_never = bars + 9;         // nothing arrives on it (the failure-path test hook waits here)
  uint64_t* b_k = bars + 10;            // [4] output scales of chunk c (c mod 4) written (one arrival per state warp)
  uint64_t* b_of = bars + 14;           // [2] D buffer s read out (one arrival per output warp)
  float* ksc = reinterpret_cast<float*>(smem + L::KSC);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + L::TMEMP);
  int* sflag = reinterpret_cast<int*>(smem + L::FLAG);
  const volatile int* vflag = sflag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = (int)blockIdx.x;
  // resident: the next segment's prep, launched as a programmatic dependent,
  // may take the SMs this grid leaves free
  griddep_launch_dependents();
  const int h = bh % a.Hv, bi = bh / a.Hv;
  // This CTA's chunks, their slots, and its tokens in the o buffer: the
  // launch's segment of sequence bi, or all chunks of packed sequence bi.
  const int n_seg = a.nseq ? a.cu_chk[bi + 1] - a.cu_chk[bi] : n_seg_arg;
  const size_t slot0 = a.nseq ? (size_t)a.cu_chk[bi] * a.Hv + (size_t)h * n_seg : slot_index(sm, bh, 0);
  const size_t tok0 = a.nseq ? (size_t)a.cu_tok[bi] : (size_t)bi * a.T + (size_t)c_begin * C;
  const int trem = a.nseq ? a.cu_tok[bi + 1] - a.cu_tok[bi] : a.T - c_begin * C;
  const uint8_t* slots = static_cast<const uint8_t*>(a.workspace) + WS_HEAD + slot0 * SLOT;
  // SHARED: the tiles the value heads of a QK head share come from the slots
  // of the group's first head (U_w and max |U_w| are every head's own)
  const int hg = SHARED ? h % (a.Hv / a.Hqk) : 0;
  const uint8_t* slots_sh = slots - (size_t)hg * (a.nseq ? (size_t)n_seg : (size_t)sm.stride) * SLOT;
  TOut* og = static_cast<TOut*>(a.o);
  if (n_seg == 0) {
    // an empty packed sequence: its final state is its initial one
    if (S_out) {
      for (int idx = tid; idx < D * D; idx += L::NS) {
        const size_t e = (size_t)bh * D * D + idx;
        S_out[e] = S_in ? S_in[e] : 0.f;
      }
    }
    return;
  }

  if (tid == 0) {
    for (int i = 0; i < 16; ++i) mbar_init(&bars[i], i < 10 ? ((&bars[i] == b_sh || &bars[i] == b_u) ? L::NE / 32 : 1) : 4);
    fence_mbar_init();
    sflag[0] = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, L::T_COLS);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_ptr;

  if (warp == (L::NE + L::NO) / 32) {
    // ------------------------------------------------------------ MMA thread
    if (lane == 0) {
      auto load = [&](int c) {
        uint8_t* stg = smem + (c & 1) * L::STAGE;
        const uint8_t* own = slots + (size_t)c * SLOT;
        mbar_arrive_expect_tx(&full[c & 1], SLOT_USED);
        if (!SHARED || hg == 0) {
          bulk_g2s(stg, own, SLOT_USED, &full[c & 1]);
        } else {
          const uint8_t* sh = slots_sh + (size_t)c * SLOT;
          bulk_g2s(stg + SL_YT, sh + SL_YT, SL_UW - SL_YT, &full[c & 1]);
          bulk_g2s(stg + SL_UW, own + SL_UW, SL_KE - SL_UW, &full[c & 1]);
          bulk_g2s(stg + SL_KE, sh + SL_KE, SL_WM - SL_KE, &full[c & 1]);
          bulk_g2s(stg + SL_WM, own + SL_WM, SLOT_USED - SL_WM, &full[c & 1]);
        }
      };
      int issued = 0, landed = 0;       // chunks whose copies were issued / seen complete
      bool any_mma = false;
      for (int c = 0; c < n_seg && c < 2; ++c) {
        load(c);
        ++issued;
      }
      const uint32_t id_zs = idesc_f16(128, 64, false, true);    // Sᵀ (TMEM) × −Yᵀ or −Q̄ᵀ (MN)
      const uint32_t id_uk = idesc_f16(128, 128, false, true);   // Uᵀ (TMEM) × K_end (MN)
      const uint32_t id_ua = idesc_f16(128, 64, false, false);   // Uᵀ (TMEM) × −Aqkᵀ (K)
      // Failure-path test hook: a bounded wait that cannot complete, taken
      // before any product is issued, so the give-up path below has only
      // the two slot copies to drain.
      bool ok = a.stall_polls == 0 || mbar_wait_or_stop(b_never, 0, vflag, a.stall_polls);
      for (int c = 0; c < n_seg && ok; ++c) {
        const int s = c & 1;
        const uint32_t ph = (uint32_t)(c & 1);
        uint8_t* stg = smem + s * L::STAGE;
        const uint32_t db = tmem + L::T_D + 128u * (uint32_t)s;
        ok = mbar_wait_or_stop(&full[s], (uint32_t)((c >> 1) & 1), vflag) &&
             (c < 2 || mbar_wait_or_stop(&b_of[s], (uint32_t)(((c - 2) >> 1) & 1), vflag));
        if (!ok) break;
        ++landed;
        ok = mbar_wait_or_stop(b_sh, ph, vflag);
        if (!ok) break;
        fence_after_sync();
        // Dᵀ = Sᵀ (−Zᵀ), K = the 128 keys: the U part (−Yᵀ) first, which
        // the epilogue waits for, then the output part (−Q̄ᵀ), which runs
        // while the epilogue works
        const uint64_t y0 = desc_mn_sw(smem_u32(stg + SL_YT), 0, BS_ROW128);
        const uint64_t q0 = desc_mn_sw(smem_u32(stg + SL_QT), 0, BS_ROW128);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma16_ts(db, tmem + L::T_SH + 8 * ks, y0 + mn_step_sw(ks), id_zs, ks > 0);
        mma_commit(b_d);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma16_ts(db + 64, tmem + L::T_SH + 8 * ks, q0 + mn_step_sw(ks), id_zs, ks > 0);
        any_mma = true;
        ok = mbar_wait_or_stop(b_u, ph, vflag);
        if (!ok) break;
        fence_after_sync();
        // Sᵀ += Uᵀ K_end, then Dᵀ[:, 64..127] += Uᵀ (−Aqkᵀ): K = the 64 tokens
        const uint64_t ke0 = desc_mn_sw(smem_u32(stg + SL_KE), 0, BS_ROW64);
        const uint64_t aq0 = desc_k_sw(smem_u32(stg + SL_AQ), 0, BS_ROW64);
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          mma16_ts(tmem + L::T_S, tmem + L::T_UH + 8 * ks, ke0 + mn_step_sw(ks), id_uk, 1);
        mma_commit(b_s);
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          mma16_ts(db + 64, tmem + L::T_UH + 8 * ks, aq0 + k_step_sw(ks, BS_ROW64), id_ua, 1);
        mma_commit(&b_o[s]);
        // stage s is free once this chunk's products are done: chunk c + 2
        if (c + 2 < n_seg) {
          ok = mbar_wait_or_stop(&b_o[s], (uint32_t)((c >> 1) & 1), vflag);
          if (!ok) break;
          load(c + 2);
          ++issued;
        }
      }
      if (!ok) {
        atomicOr(sflag, 1);
        // products and copies still in flight complete (bounded) before
        // tensor and shared memory are released
        if (any_mma) {
          mma_commit(b_fin);
          mbar_wait(b_fin, 0, 1u << 16);
        }
        for (int k = landed; k < issued; ++k) mbar_wait(&full[k & 1], (uint32_t)((k >> 1) & 1), 1u << 16);
      }
    }
    __syncwarp();
  } else if (warp >= L::NE / 32) {
    // ------------------------------------------------------------ output warps
    // Chunk c's outputs: Dᵀ columns 64..127 of buffer c mod 2 hold −2^k Oᵀ / s
    // (k: the column's scale in that chunk); row 64 + i is token i, and this
    // thread writes its value column of it.
    const int q = warp - L::NE / 32;
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    const int r = q * 32 + lane;
    const size_t tstride = (size_t)a.Hv * D;
    for (int c = 0; c < n_seg; ++c) {
      const int s = c & 1;
      // (the four output warps take the same way: each warp agrees on its
      // waits, and the barrier below ORs the warps' failures)
      bool okw = mbar_wait_or_stop(&b_o[s], (uint32_t)((c >> 1) & 1), vflag) &&
                 mbar_wait_or_stop(&b_k[c & 3], (uint32_t)((c >> 2) & 1), vflag);
      okw = __all_sync(0xffffffffu, okw);
      TOut* st = reinterpret_cast<TOut*>(smem + L::OST + s * (C * D * 4));
      if (okw) {
        fence_after_sync();
        const float sc = ksc[(c & 3) * 128 + r];
        float v[C];
#pragma unroll
        for (int cb = 0; cb < C; cb += 16) tmem_ld16(t_lane + L::T_D + 128u * (uint32_t)s + 64 + cb, v + cb);
        tmem_wait_ld();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b_of[s]);
        // through shared memory (this thread's column of the [token][d_v]
        // tile), then whole rows in 16-byte pieces
#pragma unroll
        for (int i = 0; i < C; ++i) store_out<TOut>(st + i * D + r, sc * v[i]);
      }
      uint32_t failed;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.eq.u32 p, %1, 0;\n\t"
          "barrier.cta.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
          : "=r"(failed)
          : "r"((uint32_t)okw), "n"(L::NO)
          : "memory");
      if (failed) {
        atomicOr(sflag, 1);
        break;
      }
      const int t0o = c * C;
      const int Lco = min(C, trem - t0o);
      constexpr int PIECES = D * (int)sizeof(TOut) / 16;   // 16-byte pieces per row
      TOut* dst = og + ((tok0 + t0o) * a.Hv + h) * D;
      for (int idx = tid - L::NE; idx < C * PIECES; idx += L::NO) {
        const int i = idx / PIECES, pc = idx % PIECES;
        if (i < Lco)
          *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(dst + (size_t)i * tstride) + pc * 16) =
              *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(st + i * D) + pc * 16);
      }
    }
  } else {
    // ------------------------------------------------------------ state warps
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    const int r = warp * 32 + lane;     // the value column this thread carries (TMEM lane)
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {   // (the warp agrees on the outcome)
      bool got = ok && mbar_wait_or_stop(bar, parity, vflag);
      got = __all_sync(0xffffffffu, got);
      if (ok && !got) {
        ok = false;
        atomicOr(sflag, 1);
      }
      fence_after_sync();
      return ok;
    };
    auto publish = [&](uint64_t* bar) {   // this warp's TMEM stores are complete: one arrival
      tmem_wait_st();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };

    // Block floating point, per value column. Column r of chunk c runs with a
    // power-of-two scale 2^k on its state in TMEM, its fp16 copy, its row of
    // Dᵀ and of Uᵀ, so that the 16-bit operands stay in fp16's range however
    // small or large the state becomes: k is chosen, from max |S| over the
    // column at the chunk's entry and max |U_w| of the chunk (stored by the
    // prep), to put the larger of the two in [2^8, 2^9), leaving 2^7 of
    // headroom below fp16's largest value for U = U_w − Y S. The outputs
    // and S_T of the column are divided by 2^k.
    auto exp2i = [](int k) -> float { return __uint_as_float((uint32_t)(127 + k) << 23); };   // |k| ≤ 126
    // k that brings `ref` (> 0) to [2^8, 2^9); a zero (or NaN) reference keeps k
    auto pick_k = [](float ref, int k) -> int {
      if (!(ref > 0.f)) return k;
      const int e = (int)((__float_as_uint(ref) >> 23) & 0xffu) - 127;   // ⌊log2 ref⌋ (subnormal: −127)
      return max(-60, min(60, 8 - e));
    };
    auto absmax = [](const float* x) -> float {   // max |x| over half a row (8 independent chains)
      float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int u = 0; u < D / 2; ++u) m[u & 7] = fmaxf(m[u & 7], fabsf(x[u]));
#pragma unroll
      for (int j = 4; j > 0; j >>= 1)
#pragma unroll
        for (int i = 0; i < j; ++i) m[i] = fmaxf(m[i], m[i + j]);
      return m[0];
    };
    // the output scale of chunk c (−s / 2^k) for the output warps
    auto post_scale = [&](int c, int kk) {
      ksc[(c & 3) * 128 + r] = -a.scale * exp2i(-kk);
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_k[c & 3]);
    };
    auto times_gamma = [](float* x, const uint8_t* gsrc) {   // half a row times its 64 entries of γ_C
      const float4* g4 = reinterpret_cast<const float4*>(gsrc);
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        const float4 g = g4[j];
        x[4 * j] *= g.x; x[4 * j + 1] *= g.y; x[4 * j + 2] *= g.z; x[4 * j + 3] *= g.w;
      }
    };
    int k = 0;
    constexpr int HK = D / 2;           // a row of Sᵀ is handled in two halves of 64 keys
    float x[HK];

    // The entry state: fp16 2^k Sᵀ for the first chunk's products, TMEM ←
    // 2^k Sᵀ Γ of the first chunk.
    wait(&full[0], 0);
    {
      const float* S0 = S_in ? S_in + (size_t)bh * D * D + r : nullptr;
      auto load_half = [&](int hf) {
#pragma unroll
        for (int j = 0; j < HK; ++j) x[j] = S0 ? __ldg(S0 + (size_t)(hf * HK + j) * D) : 0.f;
      };
      float M = 0.f;
      for (int hf = 0; hf < 2; ++hf) {
        load_half(hf);
        M = fmaxf(M, absmax(x));
      }
      k = pick_k(fmaxf(M, *reinterpret_cast<const float*>(smem + SL_WM)), 0);
      post_scale(0, k);
      const float sg = exp2i(k);
      for (int hf = 0; hf < 2; ++hf) {
        load_half(hf);
#pragma unroll
        for (int j = 0; j < HK; ++j) x[j] *= sg;
#pragma unroll
        for (int cb = 0; cb < HK; cb += 32) tmem_st16_f16(t_lane + L::T_SH + (hf * HK + cb) / 2, x + cb);
        times_gamma(x, smem + SL_GC + hf * HK * 4);
#pragma unroll
        for (int cb = 0; cb < HK; cb += 16) tmem_st16(t_lane + L::T_S + hf * HK + cb, x + cb);
      }
      publish(b_sh);
    }

    for (int c = 0; c < n_seg && ok; ++c) {
      const int s = c & 1;
      const uint32_t ph = (uint32_t)(c & 1);
      const uint32_t db = L::T_D + 128u * (uint32_t)s;
      const uint8_t* stg = smem + s * L::STAGE;
      const int k_c = k;                  // this chunk's scale
      // ---- Uᵀ = 2^k (U_wᵀ − (Y S)ᵀ): 2^k U_w of the stage's U_wᵀ row r
      // (tokens, 16-byte pieces swizzled), taken while the product runs,
      // plus Dᵀ columns 0..63 → fp16 A operand
      if (!wait(&full[s], (uint32_t)((c >> 1) & 1))) break;
      {
        float v[C], w[C];
        const float sg = exp2i(k_c);
        const uint8_t* uw = stg + SL_UW + r * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 p = *reinterpret_cast<const uint4*>(uw + ((j ^ (r & 7)) << 4));
          const uint32_t w4[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int q2 = 0; q2 < 4; ++q2) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[q2]));
            w[8 * j + 2 * q2] = sg * f.x;
            w[8 * j + 2 * q2 + 1] = sg * f.y;
          }
        }
        if (!wait(b_d, ph)) break;
#pragma unroll
        for (int cb = 0; cb < C; cb += 16) tmem_ld16(t_lane + db + cb, v + cb);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < C; ++j) v[j] += w[j];
#pragma unroll
        for (int cb = 0; cb < C; cb += 32) tmem_st16_f16(t_lane + L::T_UH + cb / 2, v + cb);
        publish(b_u);
      }
      // ---- the state: fp16 Sᵀ for the next chunk and TMEM ← Sᵀ Γ_next; S_T after the last
      const bool more = c + 1 < n_seg;
      if (more && !wait(&full[s ^ 1], (uint32_t)(((c + 1) >> 1) & 1))) break;
      if (!wait(b_s, ph)) break;
      auto ld_half = [&](int hf) {       // 2^k_c Sᵀ_{c+1}, keys hf·64 ..
#pragma unroll
        for (int cb = 0; cb < HK; cb += 16) tmem_ld16(t_lane + L::T_S + hf * HK + cb, x + cb);
        tmem_wait_ld();
      };
      if (more) {
        const uint8_t* nx = smem + (s ^ 1) * L::STAGE;
        ld_half(0);
        float M = absmax(x);
        ld_half(1);
        M = fmaxf(M, absmax(x)) * exp2i(-k_c);
        k = pick_k(fmaxf(M, *reinterpret_cast<const float*>(nx + SL_WM)), k_c);
        const float rs = exp2i(k - k_c);
        // fp16 copy: the half in registers, then the other one
#pragma unroll
        for (int j = 0; j < HK; ++j) x[j] *= rs;
#pragma unroll
        for (int cb = 0; cb < HK; cb += 32) tmem_st16_f16(t_lane + L::T_SH + (HK + cb) / 2, x + cb);
        ld_half(0);
#pragma unroll
        for (int j = 0; j < HK; ++j) x[j] *= rs;
#pragma unroll
        for (int cb = 0; cb < HK; cb += 32) tmem_st16_f16(t_lane + L::T_SH + cb / 2, x + cb);
        publish(b_sh);
        post_scale(c + 1, k);
        // the TMEM state times Γ_next, while the next products run (complete
        // before this warp's next arrival on b_u, which orders it before the
        // next state update)
        times_gamma(x, nx + SL_GC);
#pragma unroll
        for (int cb = 0; cb < HK; cb += 16) tmem_st16(t_lane + L::T_S + cb, x + cb);
        ld_half(1);
#pragma unroll
        for (int j = 0; j < HK; ++j) x[j] *= rs;
        times_gamma(x, nx + SL_GC + HK * 4);
#pragma unroll
        for (int cb = 0; cb < HK; cb += 16) tmem_st16(t_lane + L::T_S + HK + cb, x + cb);
      } else if (S_out) {
        const float rs = exp2i(-k_c);
        float* ST = S_out + (size_t)bh * D * D + r;
        for (int hf = 0; hf < 2; ++hf) {
          ld_half(hf);
#pragma unroll
          for (int j = 0; j < HK; ++j) ST[(size_t)(hf * HK + j) * D] = rs * x[j];
        }
      }
    }
    if (!ok) atomicOr(sflag, 1);
  }
  fence_before_sync();
  __syncthreads();
  if (tid == 0 && *sflag) atomicOr(static_cast<int*>(a.workspace), 1);
  if (warp == 0) tmem_dealloc(tmem, L::T_COLS);
}

size_t state_bytes(const ChunkArgs& a) { return (size_t)a.B * a.Hv * D * D * sizeof(float); }

}  // namespace

bool chunk_tc_supported(const ChunkArgs& a, int qkv_bf16) {
  return qkv_bf16 && a.dk == D && a.dv == D && a.chunk == C;
}

namespace {
// the conv and/or the L2 norm run in the prep's load
bool fused_load(const ChunkArgs& a) { return a.conv_w != nullptr || a.l2norm; }
// Workspace per chunk of a segment: the slots of every sequence-head.
size_t bytes_per_chunk(const ChunkArgs& a) { return (size_t)a.B * a.Hv * SLOT; }
}  // namespace

// Workspace for the whole sequence in one segment (packed sequences: the
// slots of all their chunks).
size_t chunk_tc_workspace(const ChunkArgs& a) {
  if (a.nseq) return WS_HEAD + (size_t)a.cu_chk[a.nseq] * a.Hv * SLOT;
  const size_t nchunks = (a.T + C - 1) / C;
  return WS_HEAD + nchunks * bytes_per_chunk(a);
}

size_t chunk_tc_min_workspace(const ChunkArgs& a, bool carry_state) {
  if (a.nseq) return chunk_tc_workspace(a);   // packed sequences run in one pass
  return WS_HEAD + bytes_per_chunk(a) + (carry_state ? state_bytes(a) : 0);
}

namespace {
// The scan of segment k and the prep of segment k + 1 overlap when the scan
// leaves SMs idle (fewer scan CTAs than SMs) and the
// workspace holds every chunk's slot: the prep is launched as a programmatic
// dependent of the scan, so it starts once the scan's CTAs are resident and
// takes the SMs they leave free (items from a counter, so that CTAs which start
// only when the scan ends take fewer); it does not complete before the scan.
constexpr int OVERLAP_SEGMENTS = 4;     // segments of an overlapped call
constexpr int OVERLAP_MIN_CHUNKS = 32;  // per segment
constexpr int OVERLAP_LAST_MIN = 16;    // chunks of the last segment, at least
constexpr int MAX_COUNTERS = (int)(WS_HEAD / sizeof(int)) - 1;   // item counters after the status word

template <typename... Args>
cudaError_t launch_dependent(void (*kernel)(Args...), int grid, int block, size_t smem, cudaStream_t s,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}
}  // namespace

namespace {
// Tensor map of the per-channel α gates [B·T][H_g][128] (fp32, or bf16 logits; H_g heads own
// them: H_v, or H_qk when shared) for the prep's tile loads (box: 64 tokens × 1 head × 128
// channels). false if the driver entry point is unavailable (the prep then reads α with
// plain loads).
PFN_cuTensorMapEncodeTiled tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled encode = [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      fn = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled>(fn);
  }();
  return encode;
}

// Tensor map of a scalar gate [B·T][H_g] (fp32, or bf16 logits) for boxes of
// 64 tokens × 16 bytes of heads. false where a row of heads is not a multiple
// of 16 bytes (the map's stride rule; the prep then reads the gate with
// plain loads) or the driver entry point is unavailable.
bool encode_scalar_gate_map(const ChunkArgs& a, const float* g, CUtensorMap* m) {
  const cuuint64_t esz = a.gate_logits ? 2 : 4;
  PFN_cuTensorMapEncodeTiled encode = tensor_map_encoder();
  if (encode == nullptr || ((cuuint64_t)a.Hg * esz) % 16 != 0) return false;
  const cuuint64_t rows = a.nseq ? (cuuint64_t)a.T : (cuuint64_t)a.B * (cuuint64_t)a.T;
  const cuuint64_t dims[2] = {(cuuint64_t)a.Hg, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)a.Hg * esz};
  const cuuint32_t box[2] = {(cuuint32_t)(16 / esz), (cuuint32_t)C};
  const cuuint32_t estr[2] = {1, 1};
  return encode(m, a.gate_logits ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                const_cast<float*>(g), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_alpha_map(const ChunkArgs& a, CUtensorMap* m) {
  const cuuint64_t esz = a.gate_logits ? 2 : 4;
  PFN_cuTensorMapEncodeTiled encode = tensor_map_encoder();
  if (encode == nullptr) return false;
  const cuuint64_t rows = a.nseq ? (cuuint64_t)a.T : (cuuint64_t)a.B * (cuuint64_t)a.T;   // token rows
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.Hg, rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * esz, (cuuint64_t)a.Hg * D * esz};   // bytes, dims 1 and 2
  const cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)C};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode(m, a.gate_logits ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                const_cast<float*>(a.alpha), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

// Runs the chunks in segments when the workspace holds fewer chunks than the
// sequence has; the state is carried between segments through S_T (or, when
// S_T is NULL, through the end of the workspace). Workspace: status word and
// item counters (256 bytes), slots [B·H_v][seg], carried state (only when
// needed). With the whole
// sequence in the workspace and SMs left idle by the scan, the segments are
// pipelined (see the note on overlapped segments above).
using PrepFn = void (*)(ChunkArgs, int, int, SlotMap, int*, const CUtensorMap, const CUtensorMap, int);
template <bool VL>
PrepFn prep_variant(bool cv, bool lg, bool qkg) {
  if (cv)
    return lg ? (qkg ? chunk_prep_kernel<true, true, true, VL, false> : chunk_prep_kernel<true, true, false, VL, false>)
              : (qkg ? chunk_prep_kernel<true, false, true, VL, false> : chunk_prep_kernel<true, false, false, VL, false>);
  return lg ? (qkg ? chunk_prep_kernel<false, true, true, VL, false> : chunk_prep_kernel<false, true, false, VL, false>)
            : (qkg ? chunk_prep_kernel<false, false, true, VL, false> : chunk_prep_kernel<false, false, false, VL, false>);
}
// the copies with the scalar-gate boxes (tied gate layouts; fixed-length sequences, no fused load)
PrepFn prep_box_variant(bool lg, bool qkg) {
  return lg ? (qkg ? chunk_prep_kernel<false, true, true, false, true> : chunk_prep_kernel<false, true, false, false, true>)
            : (qkg ? chunk_prep_kernel<false, false, true, false, true> : chunk_prep_kernel<false, false, false, false, true>);
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, int o_bf16, cudaStream_t s) {
  const bool vl = a.nseq > 0;
  const int BH = a.B * a.Hv;
  // chunks per sequence; for packed sequences all chunks of all of them
  const int nchunks = vl ? a.cu_chk[a.nseq] : (a.T + C - 1) / C;
  if (a.ws_bytes < WS_HEAD) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(a.workspace, 0, WS_HEAD, s);   // status word and counters
  if (e != cudaSuccess || BH == 0) return e;
  if (nchunks == 0 && !vl) return e;
  const bool cv = fused_load(a);
  float* carry = a.ST;
  uint8_t* const ws = static_cast<uint8_t*>(a.workspace);
  int seg = nchunks;
  if (vl) {
    // packed sequences run in one pass with every chunk's slot in the workspace
    if (a.ws_bytes < chunk_tc_workspace(a)) return cudaErrorInvalidValue;
  } else {
    const size_t per_chunk = bytes_per_chunk(a);
    size_t avail = a.ws_bytes - WS_HEAD;
    seg = (int)std::min<size_t>(nchunks, avail / per_chunk);
    if (seg < nchunks && carry == nullptr) {
      const size_t sb = state_bytes(a);
      avail = avail > sb ? avail - sb : 0;
      seg = (int)std::min<size_t>(nchunks, avail / per_chunk);
      carry = reinterpret_cast<float*>(ws + WS_HEAD + (size_t)seg * per_chunk);
    }
    if (seg < 1) return cudaErrorInvalidValue;
  }

  for (int f16 : {0, 1, 2})   // (the fused-load copy, the plain one, the one with the gate boxes)
    for (bool lg : {false, true})
      for (bool qg : {false, true}) {
        const PrepFn prep = f16 == 2 ? prep_box_variant(lg, qg)
                          : vl       ? prep_variant<true>(f16 == 1, lg, qg)
                                     : prep_variant<false>(f16 == 1, lg, qg);
        if ((e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM)) != cudaSuccess)
          return e;
        // all of the unified L1/shared storage as shared memory, so that two prep CTAs fit an SM
        if ((e = cudaFuncSetAttribute(prep, cudaFuncAttributePreferredSharedMemoryCarveout,
                                      cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
          return e;
      }
  int dev = 0, sms = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  // Scan: one CTA per (sequence, value head).
  const int scan_ctas = BH;
  const bool qkg = a.Hg != a.Hv;
  auto scan = o_bf16 ? (qkg ? chunk_scan_kernel<__nv_bfloat16, true> : chunk_scan_kernel<__nv_bfloat16, false>)
                     : (qkg ? chunk_scan_kernel<float, true> : chunk_scan_kernel<float, false>);
  const int scan_threads = ScanLayout::NS;
  const int scan_smem = ScanLayout::SMEM;
  if ((e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize, scan_smem)) != cudaSuccess)
    return e;
  auto fix = vl ? chunk_fix_kernel<true> : chunk_fix_kernel<false>;
  if ((e = cudaFuncSetAttribute(fix, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FX_SMEM)) != cudaSuccess)
    return e;
  // Persistent prep: two CTAs per SM. Two fit by shared memory (2 × 113 KB),
  // registers (2 × 256 × 128) and tensor memory (2 × 256 of 512 columns); the
  // occupancy calculator reports one for any kernel that allocates tensor
  // memory, so the count is set here.
  const int prep_ctas = sms * 2;
  CUtensorMap amap{}, bmap{};
  int tgates = 0;   // gates by TMA
  if (a.gate_mode != GDN2_GATES_GDN) {
    if (a.alpha != nullptr && encode_alpha_map(a, &amap)) tgates |= TG_ATILE;
  } else if (a.alpha != nullptr && encode_scalar_gate_map(a, a.alpha, &amap)) {
    tgates |= TG_ABOX;
  }
  // (the fused load keeps its sums where the β box would go)
  if (a.gate_mode != GDN2_GATES_FULL && !cv && a.b != nullptr && encode_scalar_gate_map(a, a.b, &bmap)) tgates |= TG_BBOX;
  // the boxes of scalar gates: in their own copy of the prep, for fixed-length sequences without the fused load
  const bool box = !vl && !cv && (tgates & (TG_ABOX | TG_BBOX)) != 0;
  if (!box) tgates &= TG_ATILE;
  const PrepFn prep = box ? prep_box_variant(a.gate_logits != 0, qkg)
                    : vl  ? prep_variant<true>(cv, a.gate_logits != 0, qkg)
                          : prep_variant<false>(cv, a.gate_logits != 0, qkg);

  // overlapped segments: whole sequence in the workspace, idle SMs beside the
  // scan, S_T given (the state passes from segment to segment through it)
  int nseg_ov = 0;
  if (!vl && seg == nchunks && a.ST != nullptr && scan_ctas < sms && nchunks >= 2 * OVERLAP_MIN_CHUNKS)
    nseg_ov = std::min(std::min(OVERLAP_SEGMENTS, nchunks / OVERLAP_MIN_CHUNKS), MAX_COUNTERS);

  // Segment lengths. Overlapped: the last scan has no prep beside it, so the
  // last segment is short (1/8 of the chunks, at least OVERLAP_LAST_MIN; 1/4,
  // 1/6, 1/10, 1/16 and 1/32 measured slower at T=32768) and the others share
  // the rest equally.
  const int n_last = nseg_ov > 0 ? std::max(OVERLAP_LAST_MIN, nchunks / 8) : 0;
  const int step = nseg_ov > 0 ? (nchunks - n_last + nseg_ov - 2) / (nseg_ov - 1) : seg;
  const float* s_in = a.S0;
  int k = 0;
  // (packed sequences: one pass, also when every sequence is empty, so that
  // the scan copies their states)
  for (int c0 = 0; c0 < nchunks || (vl && k == 0); ++k) {
    const int n = nseg_ov > 0 && k == nseg_ov - 1 ? nchunks - c0 : std::min(step, nchunks - c0);
    const bool last = c0 + n >= nchunks;
    float* s_out = last ? a.ST : carry;
    // overlapped: every chunk has its own slot; otherwise the segment's slots start at 0
    const SlotMap sm = nseg_ov > 0 ? SlotMap{nchunks, c0} : SlotMap{seg, 0};
    int* counter = nseg_ov > 0 ? reinterpret_cast<int*>(ws) + 1 + k : nullptr;
    const int items = vl ? nchunks * a.Hv : BH * n;           // (chunk, sequence, value head)
    const int prep_items = qkg ? items / (a.Hv / a.Hqk) : items;   // QK-owned gates: one per head group
    const int grid = std::min(prep_items, prep_ctas);
    if (items == 0) {
      // nothing to prepare (packed sequences, all empty)
    } else if (nseg_ov > 0 && k > 0) {
      if ((e = launch_dependent(prep, grid, NP, P_SMEM, s, a, c0, n, sm, counter, amap, bmap, tgates)) != cudaSuccess)
        return e;
    } else {
      prep<<<grid, NP, P_SMEM, s>>>(a, c0, n, sm, counter, amap, bmap, tgates);
    }
    // the items whose decay the prep's factors cannot take, exactly
    if (items > 0) fix<<<(items + FX_ITEMS - 1) / FX_ITEMS, FX_THREADS, FX_SMEM, s>>>(a, c0, n, sm);
    scan<<<scan_ctas, scan_threads, scan_smem, s>>>(a, c0, n, sm, s_in, s_out);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    s_in = carry;
    c0 += n;
  }
  return cudaSuccess;
}

}  // namespace gdn2
