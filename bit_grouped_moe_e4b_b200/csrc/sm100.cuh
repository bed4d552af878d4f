// Thin wrappers over the sm_100a PTX used by the tcgen05 grouped GEMM:
// mbarriers (with bounded waits), TMA tile and row-gather loads, cp.async,
// proxy fences and the tcgen05 family (TMEM allocation, MMA, commit, loads).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "common.cuh"

namespace e4b {
namespace sm100 {

E4B_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------- mbarrier
E4B_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

E4B_DEV void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

E4B_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

E4B_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Raises the transaction count the current phase waits for, without arriving.
E4B_DEV void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

E4B_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity.
E4B_DEV bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Barrier `id` over the first `nthreads` threads that also returns, to every
// one of them, the OR of their `v`.
E4B_DEV bool named_bar_or(int id, int nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %3, 0;\n\t"
      "bar.red.or.pred p, %1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(nthreads), "r"(uint32_t(v))
      : "memory");
  return r != 0;
}

// Barrier `id` (1..15) over the first `nthreads` threads of the CTA.
E4B_DEV void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Waits until the phase with the given parity completes, polling at most
// `limit` times (with a short sleep between polls after the first 64).
// Returns false if it gave up or if *abort became nonzero while waiting.
E4B_DEV bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t limit,
                               const volatile int* abort) {
  uint32_t polls = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (polls >= limit) return false;
    if (abort && *abort) return false;
    ++polls;
    if (polls > 64) __nanosleep(64);
  }
}

// Non-tensor bulk copy of `bytes` contiguous bytes, global -> this CTA's shared
// memory, completing on `bar` (both addresses 16-byte aligned, bytes % 16 == 0).
E4B_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

E4B_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// ------------------------------------------------------------------ TMA
E4B_DEV void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

E4B_DEV void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Four rows of a 2-D tensor (rows r0..r3, columns [x, x + box width)) into
// four consecutive rows of the destination tile. The tensor map's box must be
// one row high.
E4B_DEV void tma_gather4_2d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t r0,
                            int32_t r1, int32_t r2, int32_t r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------- cp.async
// 16-byte copy; src_bytes = 0 fills the destination with zeros.
E4B_DEV void cp_async_16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
E4B_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
E4B_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
E4B_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy reads (the tensor cores read operands through the async proxy).
E4B_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
E4B_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
E4B_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
E4B_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
E4B_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
E4B_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate).
E4B_DEV void mma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on the mbarrier when all tcgen05 ops issued so far by this
// thread have completed.
E4B_DEV void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp gets lane
// (base lane + i), columns [col, col + 16).
E4B_DEV void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
E4B_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major bf16 tile stored as 128-byte
// rows with the 128B swizzle (8-row atoms of 1024 bytes, atoms contiguous).
// The tile must start on a 1024-byte boundary; moving along K by 16 elements
// inside the atom adds 32 bytes to the start address.
E4B_DEV uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);  // start address
  d |= uint64_t(1) << 16;                  // leading byte offset (unused for this layout)
  d |= uint64_t(1024 >> 4) << 32;          // stride byte offset: 8-row atoms are 1024 B apart
  d |= uint64_t(1) << 46;                  // descriptor version for sm_100
  d |= uint64_t(2) << 61;                  // layout: 128B swizzle
  return d;
}

// Shared-memory matrix descriptor for an MN-major bf16 tile with the 128B
// swizzle: atoms of 8 K-rows x 128 bytes (64 consecutive M or N elements per
// row, 1024 bytes per atom); lbo = bytes between atoms along M/N, sbo = bytes
// between atoms along K. Each atom starts on a 1024-byte boundary.
E4B_DEV uint64_t sw128_mnmajor_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);  // start address
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;                  // descriptor version for sm_100
  d |= uint64_t(2) << 61;                  // layout: 128B swizzle
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 D, both
// operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | (uint32_t(N >> 3) << 17)     // N / 8
         | (uint32_t(M >> 4) << 24);    // M / 16
}

// ------------------------------------------------ block-scaled MMA (MX)
// D[tmem] (+)= (A * 2^sfa) * (B * 2^sfb)^T, kind::mxf8f6f4 with one e8m0 scale
// per 32 elements of K for every row of A and B (scale_vec 1X, K = 32 per
// instruction). The scales are read from TMEM at sfa_tmem / sfb_tmem; which
// byte of their 32-bit words is in the instruction descriptor.
E4B_DEV void mma_mxf8f6f4_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor for kind::mxf8f6f4 with e8m0 scales, both operands
// K-major, shape M x N; a_fmt / b_fmt: 0 = E4M3, 5 = E2M1. sf_ids: the byte of
// the scale words (k-block of 32 within a 128-wide K chunk) for A and B.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N, uint32_t a_fmt, uint32_t b_fmt) {
  return (a_fmt << 7) | (b_fmt << 10) | (uint32_t(N >> 3) << 17) | (1u << 23)  // scale type e8m0
         | (uint32_t(M >> 4) << 24);
}
E4B_DEV uint32_t idesc_mx_ids(uint32_t idesc, uint32_t sfa_id, uint32_t sfb_id) {
  return idesc | (sfa_id << 29) | (sfb_id << 4);
}

// Copies 32 rows x 16 bytes of shared memory (rows 16 bytes apart, one
// 512-byte chunk) into TMEM columns [taddr, taddr + 4) of lanes 0-31, and the
// same data into each of the other three lane quarters.
E4B_DEV void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a 512-byte chunk of 32 rows x 16 bytes without
// swizzle (core matrices of 8 rows x 16 bytes, 128 bytes apart).
E4B_DEV uint64_t chunk512_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(128 >> 4) << 32;  // stride byte offset between 8-row core matrices
  d |= uint64_t(1) << 46;         // descriptor version for sm_100
  return d;                       // layout type 0: no swizzle
}

// ------------------------------------------------- CTA pairs (cta_group::2)
// A cluster of two CTAs on two SMs issues one MMA of M = 256: each CTA holds
// 128 rows of A and half of B's N rows in its own shared memory (same
// offsets), and each CTA's TMEM receives its 128 rows of D over all N.
// Every tcgen05 instruction of a kernel that uses pairs names cta_group::2.
E4B_DEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of both CTAs; orders the shared-memory writes before it
// (barrier initialisation included) with the reads after it, cluster-wide.
E4B_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared::cluster address of the same shared-memory offset in CTA `rank`.
E4B_DEV uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// Arrive on an mbarrier given by its cluster address (possibly the other
// CTA's). Default semantics (release at CTA scope): a release at cluster scope
// costs a fence of ~1000 clocks per arrival, and what the arrival publishes
// here is shared memory the pair MMA reads through the async proxy, which the
// writer has already made visible with fence.proxy.async.
E4B_DEV void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// try_wait with acquire at cluster scope: for barriers completed by the other
// CTA of the pair (remote arrivals, or the pair MMA's commits).
E4B_DEV bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of a phase, acquire at cluster scope.
E4B_DEV bool mbar_test_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

E4B_DEV bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity, uint32_t limit,
                                       const volatile int* abort) {
  uint32_t polls = 0;
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (polls >= limit) return false;
    if (abort && *abort) return false;
    ++polls;
    if (polls > 64) __nanosleep(64);
  }
}

E4B_DEV void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
E4B_DEV void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
E4B_DEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A * B^T over the pair, kind::f16: issued by the even CTA only.
E4B_DEV void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One arrival on the mbarrier at this offset in both CTAs of the pair once
// the pair MMAs issued so far by this thread have completed.
E4B_DEV void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(uint16_t(3))
      : "memory");
}

// ----------------------------------------------------------------- e4m3
// Two fp32 values -> two OCP E4M3 bytes, round to nearest even, magnitudes
// beyond 448 saturated to 448: the low byte holds lo, the high byte hi.
E4B_DEV uint32_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two E4M3 bytes (low byte first) -> their exact values.
E4B_DEV float2 f32x2_from_e4m3x2(uint32_t b) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(uint16_t(b)));
  const __half2 v = *reinterpret_cast<const __half2*>(&h);
  return __half22float2(v);
}

}  // namespace sm100
}  // namespace e4b
