// ptx_d256.cuh - fused tcgen05 product chains of the head_dim 256 forward
// (conventions as in ptx.cuh: one asm block issues every K-step; descriptor
// start addresses advance in 16-byte units).
#pragma once

#include <stdint.h>

namespace attn156 {

// 16 chained K-steps (K = 256), A K-major in 16 KB boxes (128 rows), B K-major in
// 8 KB boxes (64 rows) (SS form).
__device__ __forceinline__ void mma_chain_kk16_b8k(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
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
      "add.u32 al, alo, 1024;\n\tadd.u32 bl, blo, 512;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1026;\n\tadd.u32 bl, blo, 514;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1028;\n\tadd.u32 bl, blo, 516;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 1030;\n\tadd.u32 bl, blo, 518;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 2048;\n\tadd.u32 bl, blo, 1024;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 2050;\n\tadd.u32 bl, blo, 1026;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 2052;\n\tadd.u32 bl, blo, 1028;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 2054;\n\tadd.u32 bl, blo, 1030;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 3072;\n\tadd.u32 bl, blo, 1536;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 3074;\n\tadd.u32 bl, blo, 1538;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 3076;\n\tadd.u32 bl, blo, 1540;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "add.u32 al, alo, 3078;\n\tadd.u32 bl, blo, 1542;\n\t"
      "mov.b64 ad, {al, ahi};\n\tmov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 4 chained K-steps (K = 64), A from tensor memory (8 columns per step), B MN-major (TS form).
__device__ __forceinline__ void mma_chain_ts_mn4(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
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
      "}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 4 chained K-steps (K = 64), A from tensor memory in two 16-column pieces 32
// columns apart (steps at +0, +8, +32, +40), B MN-major (TS form).
__device__ __forceinline__ void mma_chain_ts_mn4_split32(uint32_t d_tmem, uint32_t a_tmem,
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
      "add.u32 at, %1, 32;\n\tadd.u32 bl, blo, 256;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "add.u32 at, %1, 40;\n\tadd.u32 bl, blo, 384;\n\t"
      "mov.b64 bd, {bl, bhi};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %3, pt;\n\t"
      "}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

}  // namespace attn156
