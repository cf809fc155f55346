// Thin inline-PTX wrappers for the sm_100a features the attention kernel
// uses: mbarriers, TMA (cp.async.bulk.tensor), and the 5th-generation tensor
// core (tcgen05: TMEM allocation, MMA, commit, TMEM loads and stores).
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace svg {

// Host: TMA map of a [BH][N][d] bf16 tensor viewed as (d, N, BH), box
// 64 x 128 x 1 with 128-byte swizzle; rows past N are zero-filled on load.
bool make_tma_map_3d(CUtensorMap* m, const void* base, int BH, int N, int d);

namespace sm100 {

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// The mbarrier receives an arrive once every cp.async issued so far by this
// thread has completed (the pending count is raised now and dropped then, so
// the phase also needs its regular arrivals).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];\n" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(z), "r"(smem_u32(src))
      : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// Arrives on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                      uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                      uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The K-steps of one tile in a single asm block, so the issuing thread
// spends about two instructions per MMA (a 32-bit add on the descriptor's
// start-address field and the MMA itself).  Start addresses are in 16-byte
// units inside the low word; every buffer lies below 256 KB, so the field
// never carries into the high word.
//
// S (+)= A B^T, K = 64 (four K-steps of 32 bytes inside one 128-byte
// swizzle atom); A and B from shared memory, K-major.
__device__ __forceinline__ void mma_ss_k64(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc) {
  asm volatile(
      "{\n .reg .pred p0, p1;\n .reg .b32 al, ah, bl, bh, x, y;\n .reg .b64 da, db;\n"
      " setp.ne.b32 p0, %4, %4;\n setp.eq.b32 p1, %4, %4;\n"
      " mov.b64 {al, ah}, %1;\n mov.b64 {bl, bh}, %2;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p0;\n"
      " add.u32 x, al, 2;\n add.u32 y, bl, 2;\n mov.b64 da, {x, ah};\n mov.b64 db, {y, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p1;\n"
      " add.u32 x, al, 4;\n add.u32 y, bl, 4;\n mov.b64 da, {x, ah};\n mov.b64 db, {y, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p1;\n"
      " add.u32 x, al, 6;\n add.u32 y, bl, 6;\n mov.b64 da, {x, ah};\n mov.b64 db, {y, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p1;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(0u)
      : "memory");
}
// K = 128 as two 64-column atoms `atom_units` (16-byte units) apart.
__device__ __forceinline__ void mma_ss_k128(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t atom_units) {
  mma_ss_k64(d_tmem, adesc, bdesc, idesc);
  asm volatile(
      "{\n .reg .pred p1;\n .reg .b32 al, ah, bl, bh, x, y;\n .reg .b64 da, db;\n"
      " setp.eq.b32 p1, %4, %4;\n"
      " mov.b64 {al, ah}, %1;\n mov.b64 {bl, bh}, %2;\n"
      " add.u32 al, al, %4;\n add.u32 bl, bl, %4;\n"
      " mov.b64 da, {al, ah};\n mov.b64 db, {bl, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p1;\n"
      " add.u32 x, al, 2;\n add.u32 y, bl, 2;\n mov.b64 da, {x, ah};\n mov.b64 db, {y, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p1;\n"
      " add.u32 x, al, 4;\n add.u32 y, bl, 4;\n mov.b64 da, {x, ah};\n mov.b64 db, {y, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p1;\n"
      " add.u32 x, al, 6;\n add.u32 y, bl, 6;\n mov.b64 da, {x, ah};\n mov.b64 db, {y, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p1;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(atom_units)
      : "memory");
}
// O (+)= P V over 128 keys: eight K-steps of 16 keys, P from TMEM (8
// columns per step), V from shared memory (16 rows of 128 bytes per step,
// MN-major).  accumulate == 0 overwrites O in the first step.
__device__ __forceinline__ void mma_ts_k128(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p0, p1;\n .reg .b32 bl, bh, x, ta;\n .reg .b64 db;\n"
      " setp.ne.b32 p0, %4, 0;\n setp.eq.b32 p1, %4, %4;\n"
      " mov.b64 {bl, bh}, %2;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n"
      " add.u32 ta, %1, 8;\n add.u32 x, bl, 128;\n mov.b64 db, {x, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, p1;\n"
      " add.u32 ta, %1, 16;\n add.u32 x, bl, 256;\n mov.b64 db, {x, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, p1;\n"
      " add.u32 ta, %1, 24;\n add.u32 x, bl, 384;\n mov.b64 db, {x, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, p1;\n"
      " add.u32 ta, %1, 32;\n add.u32 x, bl, 512;\n mov.b64 db, {x, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, p1;\n"
      " add.u32 ta, %1, 40;\n add.u32 x, bl, 640;\n mov.b64 db, {x, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, p1;\n"
      " add.u32 ta, %1, 48;\n add.u32 x, bl, 768;\n mov.b64 db, {x, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, p1;\n"
      " add.u32 ta, %1, 56;\n add.u32 x, bl, 896;\n mov.b64 db, {x, bh};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, p1;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, K-major A,
// B K-major (QK^T) or MN-major (PV), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4)                          // D format: f32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16)   // B major
         | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor, kind::f16: fp16 A and B, fp32 D, K-major A,
// B K-major or MN-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool b_mn_major) {
  return (1u << 4)                          // D format: f32
         | ((b_mn_major ? 1u : 0u) << 16)   // B major (A and B format 0: f16)
         | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
// One 32-bit TMEM column of this thread's lane.
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n" : "=r"(r) : "r"(taddr));
  return r;
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}
__device__ __forceinline__ void reg_fence1(uint32_t& r) { asm volatile("" : "+r"(r)); }

// ------------------------------------------------------------------ packed fp32

// (d0, d1) = (a0 * b0 + c0, a1 * b1 + c1) in one f32x2 instruction.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                     float c0, float c1) {
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
// (d0, d1) = (a0 + b0, a1 + b1) in one f32x2 instruction.
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// (acc0, acc1) += (lo, hi) of an fp16 pair, each converted exactly to fp32
// inside the add (mixed-precision add, sm_100).
__device__ __forceinline__ void add_f16x2_to_f32(float& acc0, float& acc1, uint32_t h2) {
  asm("{\n .reg .f16 lo, hi;\n mov.b32 {lo, hi}, %2;\n add.rn.f32.f16 %0, lo, %0;\n"
      " add.rn.f32.f16 %1, hi, %1;\n}\n"
      : "+f"(acc0), "+f"(acc1)
      : "r"(h2));
}
// max of three floats in one instruction.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
// Ties the 32 registers of a tcgen05.ld to this point in program order, so
// that no use of them is scheduled before the preceding tcgen05.wait::ld.
__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31]));
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// Warpgroup-wide register budget changes (all warps of a warpgroup execute
// them).  The budgets of all warpgroups must add up to at most the registers
// the block was launched with.
template <int N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(N));
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace sm100
}  // namespace svg
