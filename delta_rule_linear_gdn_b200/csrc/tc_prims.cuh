// sm_100a primitives: tcgen05 tensor-core MMA with TMEM accumulators, TMEM
// loads/stores, shared-memory matrix descriptors and mbarriers (inline PTX).
//
// Operand tiles in shared memory use the non-swizzled ("interleaved")
// canonical layout: the matrix is cut into core matrices of 8 rows × 16 bytes
// (8 × 8 bf16), each stored as 128 contiguous bytes (row r of the core at byte
// 16·r). A tile X[R][C] (logical row-major, bf16) is stored core-row-major:
// core (rb, cb) at byte (rb·C/8 + cb)·128. The same storage serves as
//   * a K-major operand (rows = M or N, columns = K):
//       leading byte offset (LBO, between K core matrices)   = 128
//       stride byte offset  (SBO, between 8-row groups)      = C/8 · 128
//   * an MN-major operand (rows = K, columns = M or N):
//       LBO (between K groups of 8 rows)                     = C/8 · 128
//       SBO (between MN groups of 8 columns)                 = 128
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gdn2 {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of element (r, c) of a tiled bf16 matrix with C columns.
__host__ __device__ __forceinline__ uint32_t tile_off(int r, int c, int C) {
  return (uint32_t)(((r >> 3) * (C >> 3) + (c >> 3)) * 128 + (r & 7) * 16 + (c & 7) * 2);
}

// 128-byte-swizzled tiles. A tile X[R][C] (16-bit, C a multiple of 64) is
// stored as 64-column blocks, block b at byte b·BS (BS ≥ R·128, 1024-aligned);
// row r of a block occupies bytes [r·128, r·128 + 128) and its 16-byte chunk j
// sits at chunk position j XOR (r mod 8). A warp writing or reading whole rows
// touches every bank once, and the tensor core reads the tile with
//   K-major  (rows = M/N, columns = K): SBO = 1024 (8-row groups); a K=16 step
//            moves the start by 32 bytes inside a block and by BS across blocks;
//   MN-major (rows = K, columns = M/N): SBO = 1024 (8 K-rows), LBO = BS (next
//            64 columns of M/N); a K=16 step moves the start by 2048 bytes.
__host__ __device__ __forceinline__ uint32_t sw_off(int r, int c, int BS) {
  return (uint32_t)((c >> 6) * BS + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

// Shared-memory matrix descriptor, no swizzle, Blackwell version field = 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // version
  // base offset 0, LBO mode 0, layout type 0 (no swizzle)
  return d;
}

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return sdesc(saddr, lbo, sbo) | ((uint64_t)2 << 61);   // layout type 2: 128-byte swizzle
}
// Descriptor of K step `ks` (16 elements) of a swizzled tile.
__device__ __forceinline__ uint64_t desc_k_sw(uint32_t base, int ks, int BS) {
  return sdesc_sw128(base + (uint32_t)((ks >> 2) * BS + (ks & 3) * 32), 16, 1024);
}
__device__ __forceinline__ uint64_t desc_mn_sw(uint32_t base, int ks, int BS) {
  return sdesc_sw128(base + (uint32_t)(ks * 2048), (uint32_t)BS, 1024);
}

// Increments to add to the descriptor of K step 0 to reach K step `ks` (the
// start-address field counts 16-byte units; shared addresses stay < 256 KB,
// so the addition never carries out of the field).
__host__ __device__ constexpr uint64_t k_step_sw(int ks, int BS) {
  return (uint64_t)(((ks >> 2) * BS + (ks & 3) * 32) >> 4);
}
__host__ __device__ constexpr uint64_t mn_step_sw(int ks) { return (uint64_t)((ks * 2048) >> 4); }

// Descriptors for a tiled X[R][C] used as a K-major or MN-major operand.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr, int C) { return sdesc(saddr, 128, (C / 8) * 128); }
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr, int C) { return sdesc(saddr, (C / 8) * 128, 128); }

// Instruction descriptor of kind::f16 with an fp32 accumulator. A and B
// share one 16-bit type: `bf16` selects bf16, otherwise fp16.
__host__ __device__ constexpr uint32_t idesc_16(int M, int N, bool a_mn, bool b_mn, bool bf16) {
  return (1u << 4)                          // D format f32
         | ((bf16 ? 1u : 0u) << 7)          // A format (0 = f16, 1 = bf16)
         | ((bf16 ? 1u : 0u) << 10)         // B format
         | ((a_mn ? 1u : 0u) << 15)         // A major (0 = K)
         | ((b_mn ? 1u : 0u) << 16)         // B major
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return idesc_16(M, N, a_mn, b_mn, true);
}
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn, bool b_mn) {
  return idesc_16(M, N, a_mn, b_mn, false);
}

// D[tmem] (+)= A · B for one K=16 step. Issued by a single thread.
__device__ __forceinline__ void mma16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
      :
      : "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation issued so far by this
// thread has completed.
// The same product with the A operand in tensor memory (M lanes, K 16-bit
// elements packed two per 32-bit column, the lower half first): a_tmem is the
// TMEM address of K step 0's columns, step ks at a_tmem + 8·ks.
__device__ __forceinline__ void mma16_ts(uint32_t tmem_d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
      :
      : "r"(tmem_d), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_u32(mbar))
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// Make generic-proxy shared-memory writes visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// TMEM allocation (one full warp executes these).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes
// 32·(w%4) .. +31; taddr carries that lane base in bits 31:16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// mbarriers.
__device__ __forceinline__ void mbar_init(uint64_t* mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(mbar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* mbar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(mbar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false if the phase did not complete within the limit
// (each try_wait itself suspends for a hardware-defined interval).
__device__ __forceinline__ bool mbar_wait(uint64_t* mbar, uint32_t parity, uint32_t limit = (1u << 24)) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(mbar, parity)) return true;
  return false;
}

// Bounded wait that also gives up as soon as *stop becomes nonzero (another
// thread of the CTA met an error); returns true only if the phase completed.
__device__ __forceinline__ bool mbar_wait_or_stop(uint64_t* mbar, uint32_t parity, const volatile int* stop,
                                                  uint32_t limit = (1u << 22)) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(mbar, parity)) return true;
    if ((i & 15u) == 15u && *stop) return false;
  }
  return false;
}

// Plain arrive (count 1) on an mbarrier.
__device__ __forceinline__ void mbar_arrive(uint64_t* mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(mbar)) : "memory");
}

// Arrive on an mbarrier and add `bytes` to the transaction count it waits for.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(mbar)), "r"(bytes)
               : "memory");
}

// Bulk (non-tensor) asynchronous copy global → shared of `bytes` (multiple of
// 16, both addresses 16-byte aligned), completing on `mbar` as transactions;
// the destination is this CTA's own shared memory only.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(mbar))
      : "memory");
}

// Tiled tensor copy global → shared of one box of a 3-D tensor map into this
// CTA's own shared memory, completing on `mbar` as transactions. The innermost coordinate
// x times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_3d(void* dst_smem, const void* tmap, int x, int y, int z, uint64_t* mbar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n"
      ::"r"(smem_u32(dst_smem)), "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(mbar))
      : "memory");
}

// The same for one box of a 2-D tensor map.
__device__ __forceinline__ void tma_load_2d(void* dst_smem, const void* tmap, int x, int y, uint64_t* mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
      ::"r"(smem_u32(dst_smem)), "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(mbar))
      : "memory");
}

// Hint that the 128-byte line holding `p` (a valid global address) be brought
// into L2; no register receives data and nothing waits for it.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
}

// Bulk (non-tensor) asynchronous copy shared → global of `bytes` (multiple of
// 16, both addresses 16-byte aligned), tracked by the issuing thread's bulk
// groups: commit, then wait until the source may be overwritten (.read) or
// until the writes are done.
__device__ __forceinline__ void bulk_s2g(void* dst_gmem, const void* src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n" ::"l"(dst_gmem),
               "r"(smem_u32(src_smem)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }

// Programmatic dependent launch: a kernel launched after this one with
// programmatic stream serialization may start once every CTA of this one has
// executed launch_dependents (or exited); griddep_wait blocks until the grids
// this one depends on have completed and their writes are visible (it returns
// at once for a kernel launched without that attribute).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// Approximate reciprocal (the PTX rcp.approx.ftz.f32 instruction: at most
// one ulp of error, subnormal inputs and results flushed to zero).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Pairs of floats to 16-bit pairs (the first value in the low half), round to
// nearest even, one cvt each; no address is taken, so that the packed words
// stay in registers whatever the inlining order.
__device__ __forceinline__ uint32_t pack2_f16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}
__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

// Pack 8 floats to 8 bf16 / fp16 (16 bytes).
__device__ __forceinline__ uint4 pack8_bf16(const float* x) {
  return make_uint4(pack2_bf16(x[0], x[1]), pack2_bf16(x[2], x[3]), pack2_bf16(x[4], x[5]), pack2_bf16(x[6], x[7]));
}
__device__ __forceinline__ uint4 pack8_f16(const float* x) {
  return make_uint4(pack2_f16(x[0], x[1]), pack2_f16(x[2], x[3]), pack2_f16(x[4], x[5]), pack2_f16(x[6], x[7]));
}
__device__ __forceinline__ uint4 pack8(const float* x, bool bf16) { return bf16 ? pack8_bf16(x) : pack8_f16(x); }

// Pack 4 floats to 4 16-bit values (8 bytes).
__device__ __forceinline__ uint2 pack4_f16(float a, float b, float c, float d) {
  return make_uint2(pack2_f16(a, b), pack2_f16(c, d));
}
__device__ __forceinline__ uint2 pack4_bf16(float a, float b, float c, float d) {
  return make_uint2(pack2_bf16(a, b), pack2_bf16(c, d));
}
__device__ __forceinline__ uint2 pack4(const float* x, bool bf16) {
  return bf16 ? pack4_bf16(x[0], x[1], x[2], x[3]) : pack4_f16(x[0], x[1], x[2], x[3]);
}

}  // namespace tc
}  // namespace gdn2
