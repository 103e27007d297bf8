// ptx.cuh - thin inline-PTX wrappers for sm_100a: mbarriers with bounded waits,
// TMA tensor/bulk copies, and the tcgen05 (5th-generation tensor core) family:
// tensor-memory allocation, MMA issue, commit, and TMEM <-> register moves.
// Written from the PTX ISA; every wait in this library goes through
// Bounded::wait so that no kernel can spin forever.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace attn156 {

// Codes recorded in the device error word (low 8 bits: status, high bits: site).
constexpr uint32_t kErrTimeout = 9u;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// A bounded waiter shared by all roles of one CTA.  If any wait of the CTA runs
// out, it raises `abort` (shared memory) so that every other role stops at its
// next wait instead of timing out one by one, and it records the failure in the
// device error word.
struct Bounded {
  volatile int* abort;      // shared-memory flag, 0 = running
  uint32_t* err;            // device error word (global memory)
  uint64_t limit_ns;

  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, uint32_t site) const {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
      for (int i = 0; i < 32; ++i)
        if (mbar_try_wait(bar, parity)) return true;
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort = 1;
        atomicCAS(err, 0u, kErrTimeout | (site << 8));
        return false;
      }
    }
  }
  // For warps that go on to issue warp-collective (.sync.aligned) tcgen05
  // instructions: every lane waits, and the warp proceeds only if all lanes saw
  // the barrier complete, so the warp never diverges on an abort.
  __device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, uint32_t site) const {
    const bool ok = wait(bar, parity, site);
    return __all_sync(0xffffffffu, ok) != 0;
  }
  __device__ __forceinline__ bool aborted() const { return *abort != 0; }
};

// ----------------------------------------------------------------------------
// TMA (bulk tensor copies) and plain bulk copies
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 4-D tiled load global -> shared, completion counted on `bar` in bytes.
// Coordinates are innermost first: (d, head, seq, batch).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* map, uint32_t bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// Contiguous bulk copy global -> shared (both 16-byte aligned, size multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Make generic-proxy writes to shared memory visible to the async proxy
// (tensor core operand reads, TMA stores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, commit
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 async op issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ----------------------------------------------------------------------------
// Fused MMA chains: one asm block issues all K-steps of a 128-row product, so
// the issuing thread spends about three instructions per tcgen05.mma.  The
// descriptors of step kk are the base descriptors with the start-address field
// (16-byte units, low 32 bits) advanced by: K-major 128B-swizzled tiles
// ((kk / 4) * 1024 + (kk % 4) * 2), i.e. 32 bytes per 16-element step inside a
// 64-column box and the next 16 KB box every four steps; MN-major tiles
// (kk * 128), i.e. 16 rows of 128 bytes per step.  Start addresses stay below
// 256 KB, so the low half never carries into the high half.  The first step
// accumulates iff `accumulate` is non-zero; later steps always accumulate.
// ----------------------------------------------------------------------------
// 8 chained K-steps, A K-major, B K-major (SS form).
__device__ __forceinline__ void mma_chain_kk8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                   uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .b32 alo, ahi, blo, bhi, al, bl;\n\t.reg .b64 ad, bd;\n\t.reg .pred pa, pt;\n\t"
      "mov.b64 {alo, ahi}, %1;\n\tmov.b64 {blo, bhi}, %2;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "add.u32 al, alo, 0;\n\tadd.u32 bl, blo, 0;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pa;\n\t"
      "add.u32 al, alo, 2;\n\tadd.u32 bl, blo, 2;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 4;\n\tadd.u32 bl, blo, 4;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 6;\n\tadd.u32 bl, blo, 6;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1024;\n\tadd.u32 bl, blo, 1024;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1026;\n\tadd.u32 bl, blo, 1026;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1028;\n\tadd.u32 bl, blo, 1028;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1030;\n\tadd.u32 bl, blo, 1030;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 4 chained K-steps, A K-major, B K-major (SS form).
__device__ __forceinline__ void mma_chain_kk4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                   uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .b32 alo, ahi, blo, bhi, al, bl;\n\t.reg .b64 ad, bd;\n\t.reg .pred pa, pt;\n\t"
      "mov.b64 {alo, ahi}, %1;\n\tmov.b64 {blo, bhi}, %2;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "add.u32 al, alo, 0;\n\tadd.u32 bl, blo, 0;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pa;\n\t"
      "add.u32 al, alo, 2;\n\tadd.u32 bl, blo, 2;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 4;\n\tadd.u32 bl, blo, 4;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 6;\n\tadd.u32 bl, blo, 6;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 8 chained K-steps, A K-major, B MN-major (SS form).
__device__ __forceinline__ void mma_chain_kmn8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                   uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .b32 alo, ahi, blo, bhi, al, bl;\n\t.reg .b64 ad, bd;\n\t.reg .pred pa, pt;\n\t"
      "mov.b64 {alo, ahi}, %1;\n\tmov.b64 {blo, bhi}, %2;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "add.u32 al, alo, 0;\n\tadd.u32 bl, blo, 0;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pa;\n\t"
      "add.u32 al, alo, 2;\n\tadd.u32 bl, blo, 128;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 4;\n\tadd.u32 bl, blo, 256;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 6;\n\tadd.u32 bl, blo, 384;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1024;\n\tadd.u32 bl, blo, 512;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1026;\n\tadd.u32 bl, blo, 640;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1028;\n\tadd.u32 bl, blo, 768;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1030;\n\tadd.u32 bl, blo, 896;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 8 chained K-steps, A MN-major, B MN-major (SS form).
__device__ __forceinline__ void mma_chain_mnmn8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                   uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .b32 alo, ahi, blo, bhi, al, bl;\n\t.reg .b64 ad, bd;\n\t.reg .pred pa, pt;\n\t"
      "mov.b64 {alo, ahi}, %1;\n\tmov.b64 {blo, bhi}, %2;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "add.u32 al, alo, 0;\n\tadd.u32 bl, blo, 0;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pa;\n\t"
      "add.u32 al, alo, 128;\n\tadd.u32 bl, blo, 128;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 256;\n\tadd.u32 bl, blo, 256;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 384;\n\tadd.u32 bl, blo, 384;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 512;\n\tadd.u32 bl, blo, 512;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 640;\n\tadd.u32 bl, blo, 640;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 768;\n\tadd.u32 bl, blo, 768;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 896;\n\tadd.u32 bl, blo, 896;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 8 chained K-steps, A K-major (16 KB boxes), B K-major in boxes of 16 rows
// (2 KB: a small N = 16 operand) (SS form).
__device__ __forceinline__ void mma_chain_kk8_b16(uint32_t d_tmem, uint64_t a_desc,
                                                  uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .b32 alo, ahi, blo, bhi, al, bl;\n\t.reg .b64 ad, bd;\n\t.reg .pred pa, pt;\n\t"
      "mov.b64 {alo, ahi}, %1;\n\tmov.b64 {blo, bhi}, %2;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "add.u32 al, alo, 0;\n\tadd.u32 bl, blo, 0;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pa;\n\t"
      "add.u32 al, alo, 2;\n\tadd.u32 bl, blo, 2;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 4;\n\tadd.u32 bl, blo, 4;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 6;\n\tadd.u32 bl, blo, 6;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1024;\n\tadd.u32 bl, blo, 128;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1026;\n\tadd.u32 bl, blo, 130;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1028;\n\tadd.u32 bl, blo, 132;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1030;\n\tadd.u32 bl, blo, 134;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 8 chained K-steps, A MN-major, B K-major in boxes of 16 rows (2 KB: a small
// N = 16 operand, the next 64-element K block 2 KB further on) (SS form).
__device__ __forceinline__ void mma_chain_mnk8_b16(uint32_t d_tmem, uint64_t a_desc,
                                                   uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .b32 alo, ahi, blo, bhi, al, bl;\n\t.reg .b64 ad, bd;\n\t.reg .pred pa, pt;\n\t"
      "mov.b64 {alo, ahi}, %1;\n\tmov.b64 {blo, bhi}, %2;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "add.u32 al, alo, 0;\n\tadd.u32 bl, blo, 0;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pa;\n\t"
      "add.u32 al, alo, 128;\n\tadd.u32 bl, blo, 2;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 256;\n\tadd.u32 bl, blo, 4;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 384;\n\tadd.u32 bl, blo, 6;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 512;\n\tadd.u32 bl, blo, 128;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 640;\n\tadd.u32 bl, blo, 130;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 768;\n\tadd.u32 bl, blo, 132;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 896;\n\tadd.u32 bl, blo, 134;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 8 chained K-steps, A from tensor memory (8 columns per step), B MN-major (TS form).
__device__ __forceinline__ void mma_chain_ts_mn8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                   uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .b32 blo, bhi, bl, at;\n\t.reg .b64 bd;\n\t.reg .pred pa, pt;\n\t"
      "mov.b64 {blo, bhi}, %2;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "add.u32 at, %1, 0;\n\tadd.u32 bl, blo, 0;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pa;\n\t"
      "add.u32 at, %1, 8;\n\tadd.u32 bl, blo, 128;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 16;\n\tadd.u32 bl, blo, 256;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 24;\n\tadd.u32 bl, blo, 384;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 32;\n\tadd.u32 bl, blo, 512;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 40;\n\tadd.u32 bl, blo, 640;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 48;\n\tadd.u32 bl, blo, 768;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 56;\n\tadd.u32 bl, blo, 896;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// As mma_chain_ts_mn8, with A's 16-bit pairs in two blocks of 32 columns 64
// apart (K-steps 0-3 from columns [0,32), K-steps 4-7 from [64,96)): the layout
// two thread groups leave when each writes its half of P beside its own scores.
__device__ __forceinline__ void mma_chain_ts_mn8_split64(uint32_t d_tmem, uint32_t a_tmem,
                                                         uint64_t b_desc, uint32_t idesc,
                                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .b32 blo, bhi, bl, at;\n\t.reg .b64 bd;\n\t.reg .pred pa, pt;\n\t"
      "mov.b64 {blo, bhi}, %2;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "add.u32 at, %1, 0;\n\tadd.u32 bl, blo, 0;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pa;\n\t"
      "add.u32 at, %1, 8;\n\tadd.u32 bl, blo, 128;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 16;\n\tadd.u32 bl, blo, 256;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 24;\n\tadd.u32 bl, blo, 384;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 64;\n\tadd.u32 bl, blo, 512;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 72;\n\tadd.u32 bl, blo, 640;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 80;\n\tadd.u32 bl, blo, 768;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 88;\n\tadd.u32 bl, blo, 896;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor for kind::f16 with 16-bit A/B of format `fmt`
// (0 = f16, 1 = bf16; A and B always the same) and f32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f32acc(int M, int N, bool a_mn_major,
                                                    bool b_mn_major, uint32_t fmt) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Instruction descriptor for kind::f16 with bf16 A/B and f32 accumulate.
// Fields: [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format,
// [15] A major (1 = MN-major), [16] B major, [17,23) N>>3, [24,29) M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
// Operand tiles are stored as "boxes" of R rows x 128 bytes (64 bf16), 1024-byte
// aligned, exactly as a TMA load with 128-byte swizzle writes them.
//  K-major:  rows = M (or N) index, the 128-byte row runs along K.
//            SBO = 1024 (next group of 8 rows); LBO unused (1).
//  MN-major: rows = K index, the 128-byte row runs along M (or N).
//            SBO = 1024 (next group of 8 K rows); LBO = distance between
//            consecutive 64-element blocks along M/N (the next box).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= uint64_t(1024u >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// ----------------------------------------------------------------------------
// TMEM <-> registers.  Each warp may touch only the 32 lanes of its quadrant
// (warp_id % 4).  Loads are fused with tcgen05.wait::ld in the same asm
// statement, so the outputs are complete when the statement ends; stores are
// fused with tcgen05.wait::st.
// ----------------------------------------------------------------------------
#define ATTN_R8(b) "=r"(r[b + 0]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), \
                   "=r"(r[b + 4]), "=r"(r[b + 5]), "=r"(r[b + 6]), "=r"(r[b + 7])
#define ATTN_W8(b) "r"(r[b + 0]), "r"(r[b + 1]), "r"(r[b + 2]), "r"(r[b + 3]), \
                   "r"(r[b + 4]), "r"(r[b + 5]), "r"(r[b + 6]), "r"(r[b + 7])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ATTN_R8(0), ATTN_R8(8), ATTN_R8(16), ATTN_R8(24)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ATTN_R8(0), ATTN_R8(8)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      ATTN_W8(0), ATTN_W8(8), ATTN_W8(16), ATTN_W8(24)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      ATTN_W8(0), ATTN_W8(8)
      : "memory");
}

// Generated wide TMEM moves (one tcgen05 instruction + its wait per call).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};\n\t"
      "tcgen05.wait::st.sync.aligned;"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
      : "memory");
}

#undef ATTN_R8
#undef ATTN_W8

// ----------------------------------------------------------------------------
// Register reallocation between warpgroups (all four warps of a warpgroup must
// execute the same instruction).
// ----------------------------------------------------------------------------
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Move this warpgroup from `From` registers per thread (its count at launch)
// to `To`: setmaxnreg.inc to grow, setmaxnreg.dec to shrink, chosen at compile
// time so the direction can never be wrong.
template <int From, int To>
__device__ __forceinline__ void regs_realloc() {
  static_assert(To % 8 == 0 && To >= 24 && To <= 256, "setmaxnreg count out of range");
  if constexpr (To > From) {
    regs_inc<To>();
  } else if constexpr (To < From) {
    regs_dec<To>();
  }
}

// Named barrier over `count` threads (ids 1..15; id 0 is __syncthreads).
// Programmatic dependent launch: a grid launched after this one with the
// programmatic-serialization attribute may start once every CTA of this grid
// has signalled (or exited); it must call griddep_wait() before it reads what
// this grid writes (the wait returns once this grid has completed and its
// memory operations are visible).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier over `count` threads that also ANDs a predicate across them; every
// participant gets the same answer, so a group can agree to stop together.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// TMA bulk reduce-add (fp32) of a shared-memory box into global memory.
__device__ __forceinline__ void tma_reduce_add_2d(const void* map, uint32_t src, int c0, int c1) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          map),
      "r"(src), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until the shared-memory sources of all committed bulk groups have been read.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until at most N of the committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ----------------------------------------------------------------------------
// Packed fp32 pairs (sm_100 f32x2 arithmetic) and helpers of the softmax
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ----------------------------------------------------------------------------
// Arithmetic helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Pack two floats to bf16x2 (round to nearest even); `lo` lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void red_add_f32(float* gptr, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(gptr), "f"(a) : "memory");
}

// The two 16-bit element formats of the operands and outputs.  pack2 rounds
// two floats to nearest-even and puts `lo` in bits 0..15; unpack2 widens a
// packed pair exactly.
struct ElemBF16 {
  static constexpr uint32_t kFmt = 1;  // kind::f16 operand format code
  __device__ static __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }
  __device__ static __forceinline__ void unpack2(uint32_t u, float& lo, float& hi) {
    lo = __uint_as_float(u << 16);
    hi = __uint_as_float(u & 0xffff0000u);
  }
};
struct ElemF16 {
  static constexpr uint32_t kFmt = 0;
  __device__ static __forceinline__ uint32_t pack2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
  }
  __device__ static __forceinline__ void unpack2(uint32_t u, float& lo, float& hi) {
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(u));
  }
};

__device__ __forceinline__ void red_add_v4(float* gptr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(gptr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ void st_global_v4(void* gptr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(gptr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ float4 ld_shared_v4(uint32_t saddr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(saddr)
               : "memory");
  return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

}  // namespace attn156
