// diag.cu - test-only diagnostics of the building blocks the attention kernels
// rely on, each checked against a CPU product by the tests:
//   attn_diag_mma: one 128x128x128 bf16 product through tcgen05.mma in one of
//     the operand forms the kernels use (operands placed in shared memory with
//     the 128-byte swizzle by plain stores):
//       mode 0: C = A B^T, A and B K-major              (S = Q K^T;  S^T = K Q^T)
//       mode 1: C = A B,   A K-major, B MN-major         (dK += dS^T Q)
//       mode 2: C = A B,   A from tensor memory, B MN-major (O += P V; dV += P^T dO)
//       mode 3: C = A^T B, A MN-major, B MN-major        (dQ = dS K)
//       modes 4-7: the same four products through the fused multi-step
//       chains the kernels issue (mma_chain_*)
//   attn_diag_mma_pair: one 256x128x128 bf16 product issued for a pair of
//     CTAs (a cluster of two, tcgen05 cta_group::2); CTA r holds rows
//     [128 r, 128 r + 128) of A and C, and rows [64 r, 64 r + 64) of B (N x K):
//       mode 8:  C = A B^T, A and B K-major, placed by plain stores
//       mode 9:  C = A B,   A from tensor memory, B MN-major (CTA r: columns [64 r, +64))
//       mode 10: as mode 8, operands brought in by the pair's TMA loads whose
//                bytes are counted on the even CTA's mbarrier
//   attn_diag_tma: a TMA load of a (1, 128, 1, 128) bf16 tensor with the
//     same 4-D map and 128-byte swizzle as the kernels; the raw shared-memory
//     bytes are copied out so the test can check the placement.
//   attn_diag_mask_bounds, attn_diag_fwd_tile_ranges, attn_diag_bwd_qtile_ranges,
//   attn_diag_chunked_order, attn_diag_d256_work: host-only views of the index
//     arithmetic the kernels pick their work with (mask bounds per row and per
//     key, the key-tile range of a query tile and the query-tile range of a key
//     tile, the block order, the head_dim 256 backward's gradient per block);
//     they launch nothing, so the CPU tests check them exhaustively.
// Not part of the product library.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bwd256_sm100.cuh"
#include "bwd_sm100.cuh"
#include "common.cuh"
#include "fwd_sm100.cuh"
#include "ptx.cuh"
#include "ptx_pair.cuh"

using namespace attn156;

namespace {

__device__ uint32_t g_diag_err = 0;

constexpr int N = 128;
constexpr int kBox = 128 * 128;  // bytes of one 128-row x 64-col box

// byte offset of element (row, col) of a 128 x 128 bf16 tile stored as two
// 128-byte-swizzled boxes of 64 columns
__device__ __forceinline__ uint32_t swz(int row, int col) {
  const uint32_t box = uint32_t(col / 64);
  const uint32_t chunk = uint32_t((col % 64) / 8);
  return box * kBox + uint32_t(row) * 128 + ((chunk ^ uint32_t(row & 7)) << 4) +
         uint32_t(col % 8) * 2;
}

__global__ void __launch_bounds__(128, 1)
    diag_mma_kernel(int mode, const __nv_bfloat16* A, const __nv_bfloat16* Bm, float* C) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t& bar = *reinterpret_cast<uint64_t*>(smem + 4 * kBox);
  uint32_t& tslot = *reinterpret_cast<uint32_t*>(smem + 4 * kBox + 8);
  int& abort_flag = *reinterpret_cast<int*>(smem + 4 * kBox + 12);
  uint8_t* sa = smem;
  uint8_t* sb = smem + 2 * kBox;
  const int tid = threadIdx.x;
  const int warp = tid / 32;
  const uint32_t sa_u = smem_u32(sa), sb_u = smem_u32(sb);
  if ((sa_u & 1023u) != 0) return;

  // Place operands.  A and B are row-major 128 x 128 in global memory.
  //  A K-major (modes 0,1): smem row m holds A[m][0..127] (K along the row).
  //  A MN-major (mode 3): C = A^T B, so the M index is A's column; smem row = K index = A's row.
  //  B K-major (mode 0): C = A B^T, smem row n holds B[n][0..127].
  //  B MN-major (modes 1,2,3): C = A B, smem row = K index = B's row, N along the row.
  // In every case the smem tile is "row r, column c" = global element [r][c].
  for (int e = tid; e < N * N; e += blockDim.x) {
    const int r = e / N, c = e % N;
    *reinterpret_cast<__nv_bfloat16*>(sa + swz(r, c)) = A[e];
    *reinterpret_cast<__nv_bfloat16*>(sb + swz(r, c)) = Bm[e];
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tslot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const uint32_t lane_off = uint32_t(warp * 32) << 16;
  const int row = warp * 32 + (tid % 32);

  if (mode == 2 || mode == 6) {
    // A into tensor memory columns [128, 192): lane m holds A[m][k] packed in pairs.
    uint32_t w[32];
    for (int half = 0; half < 2; ++half) {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int k = half * 64 + 2 * c;
        const float lo = __bfloat162float(A[row * N + k]);
        const float hi = __bfloat162float(A[row * N + k + 1]);
        w[c] = pack_bf16x2(lo, hi);
      }
      tmem_st32(tmem + lane_off + 128 + half * 32, w);
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();

  Bounded bw{&abort_flag, &g_diag_err, 1000000000ull};
  if (tid == 0) {
    if (mode >= 4) {
      // the fused chains of the attention kernels
      if (mode == 4)
        mma_chain_kk8(tmem, sdesc_sw128(sa_u, 16), sdesc_sw128(sb_u, 16),
                      idesc_bf16_f32(128, 128, false, false), 0u);
      else if (mode == 5)
        mma_chain_kmn8(tmem, sdesc_sw128(sa_u, 16), sdesc_sw128(sb_u, kBox),
                       idesc_bf16_f32(128, 128, false, true), 0u);
      else if (mode == 6)
        mma_chain_ts_mn8(tmem, tmem + 128, sdesc_sw128(sb_u, kBox),
                         idesc_bf16_f32(128, 128, false, true), 0u);
      else
        mma_chain_mnmn8(tmem, sdesc_sw128(sa_u, kBox), sdesc_sw128(sb_u, kBox),
                        idesc_bf16_f32(128, 128, true, true), 0u);
    } else {
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = kk > 0 ? 1u : 0u;
        const uint32_t kmaj_off = (kk / 4) * kBox + (kk % 4) * 32;  // K-major: 16 K-elements
        const uint32_t mn_off = kk * 16 * 128;                      // MN-major: 16 K-rows
        if (mode == 0) {
          mma_bf16_ss(tmem, sdesc_sw128(sa_u + kmaj_off, 16), sdesc_sw128(sb_u + kmaj_off, 16),
                      idesc_bf16_f32(128, 128, false, false), acc);
        } else if (mode == 1) {
          mma_bf16_ss(tmem, sdesc_sw128(sa_u + kmaj_off, 16), sdesc_sw128(sb_u + mn_off, kBox),
                      idesc_bf16_f32(128, 128, false, true), acc);
        } else if (mode == 2) {
          mma_bf16_ts(tmem, tmem + 128 + kk * 8, sdesc_sw128(sb_u + mn_off, kBox),
                      idesc_bf16_f32(128, 128, false, true), acc);
        } else {
          mma_bf16_ss(tmem, sdesc_sw128(sa_u + mn_off, kBox), sdesc_sw128(sb_u + mn_off, kBox),
                      idesc_bf16_f32(128, 128, true, true), acc);
        }
      }
    }
    tc_commit(smem_u32(&bar));
  }
  __syncwarp();
  const bool ok = bw.wait_warp(smem_u32(&bar), 0, 1);
  tc_fence_after();
  if (ok) {
    for (int c0 = 0; c0 < N; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + c0, r);
#pragma unroll
      for (int c = 0; c < 32; ++c) C[row * N + c0 + c] = __uint_as_float(r[c]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------- CTA pair
// A is 256 x 128 (row-major), B is 128 x 128 (row-major: N x K for modes 8/10,
// K x N for mode 9), C is 256 x 128 fp32.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
    diag_mma_pair_kernel(int mode, const __nv_bfloat16* A, const __nv_bfloat16* Bm, float* C,
                         const __grid_constant__ CUtensorMap mapA,
                         const __grid_constant__ CUtensorMap mapB) {
  extern __shared__ __align__(1024) uint8_t smem[];
  // [A half: 2 boxes of 128 rows x 64 cols][B half: K-major 2 boxes of 64 rows, or one
  //  MN-major box of 128 K rows x 64 N cols][bars]
  constexpr int kAOff = 0, kBOff = 2 * kBox, kBarOff = 4 * kBox;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);  // 0: loads, 1: product done
  uint32_t& tslot = *reinterpret_cast<uint32_t*>(smem + kBarOff + 16);
  int& abort_flag = *reinterpret_cast<int*>(smem + kBarOff + 20);
  const int tid = threadIdx.x;
  const int warp = tid / 32;
  const uint32_t rank = cluster_ctarank();
  const uint32_t sa_u = smem_u32(smem + kAOff), sb_u = smem_u32(smem + kBOff);
  if ((sa_u & 1023u) != 0) return;
  const int row = warp * 32 + (tid % 32);  // this CTA's row of A / C
  if (tid == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (mode == 8 || mode == 9) {
    // A half: rows [128 rank, +128) of A, K-major, two 64-column boxes
    for (int e = tid; e < 128 * N; e += blockDim.x) {
      const int r = e / N, c = e % N;
      if (mode == 8)
        *reinterpret_cast<__nv_bfloat16*>(smem + kAOff + swz(r, c)) = A[(128 * rank + r) * N + c];
    }
    if (mode == 8) {
      // B half, K-major: rows [64 rank, +64) of B (N x K); boxes of 64 rows (8 KB)
      for (int e = tid; e < 64 * N; e += blockDim.x) {
        const int r = e / N, c = e % N;
        const uint32_t off = uint32_t(c / 64) * 8192 + uint32_t(r) * 128 +
                             ((uint32_t((c % 64) / 8) ^ uint32_t(r & 7)) << 4) + uint32_t(c % 8) * 2;
        *reinterpret_cast<__nv_bfloat16*>(smem + kBOff + off) = Bm[(64 * rank + r) * N + c];
      }
    } else {
      // B half, MN-major: all 128 K rows, N columns [64 rank, +64): one 128 x 64 box
      for (int e = tid; e < 128 * 64; e += blockDim.x) {
        const int r = e / 64, c = e % 64;
        *reinterpret_cast<__nv_bfloat16*>(smem + kBOff + swz(r, c)) = Bm[r * N + 64 * rank + c];
      }
    }
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(&tslot), 256);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers initialised and operands placed in both CTAs
  tc_fence_after();
  const uint32_t tmem = tslot;
  const uint32_t lane_off = uint32_t(warp * 32) << 16;
  if (mode == 9) {
    // A rows of this CTA into tensor memory columns [128, 192) as bf16 pairs
    uint32_t w[32];
    for (int half = 0; half < 2; ++half) {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int k = half * 64 + 2 * c;
        w[c] = pack_bf16x2(__bfloat162float(A[(128 * rank + row) * N + k]),
                           __bfloat162float(A[(128 * rank + row) * N + k + 1]));
      }
      tmem_st32(tmem + lane_off + 128 + half * 32, w);
    }
    tc_fence_before();
  }
  Bounded bw{&abort_flag, &g_diag_err, 1000000000ull};
  const uint32_t leader_load_bar = mapa_shared(smem_u32(&bars[0]), 0);
  if (mode == 10 && tid == 0) {
    if (rank == 0) mbar_arrive_expect_tx(smem_u32(&bars[0]), 2 * (2 * kBox + 2 * 8192));
    for (int x = 0; x < 2; ++x) {
      tma_load_4d_pair(sa_u + x * kBox, &mapA, leader_load_bar, x * 64, 0, 128 * int(rank), 0);
      tma_load_4d_pair(sb_u + x * 8192, &mapB, leader_load_bar, x * 64, 0, 64 * int(rank), 0);
    }
  }
  cluster_sync();  // mode 9: both CTAs' A rows are in tensor memory
  tc_fence_after();
  bool ok = true;
  if (rank == 0 && tid == 0) {
    if (mode == 10) ok = bw.wait(smem_u32(&bars[0]), 0, 3);
    if (ok) {
      tc_fence_after();
      const uint32_t id_kk = idesc_bf16_f32(256, 128, false, false);
      const uint32_t id_ts = idesc_bf16_f32(256, 128, false, true);
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = kk > 0 ? 1u : 0u;
        if (mode == 9) {
          mma2_bf16_ts(tmem, tmem + 128 + kk * 8, sdesc_sw128(sb_u + kk * 16 * 128, kBox), id_ts, acc);
        } else {
          const uint32_t a_off = (kk / 4) * kBox + (kk % 4) * 32;
          const uint32_t b_off = (kk / 4) * 8192 + (kk % 4) * 32;
          mma2_bf16_ss(tmem, sdesc_sw128(sa_u + a_off, 16), sdesc_sw128(sb_u + b_off, 16), id_kk, acc);
        }
      }
    }
    tc_commit_pair(smem_u32(&bars[1]), 0x3);
  }
  __syncwarp();
  ok = bw.wait_warp(smem_u32(&bars[1]), 0, 4);
  tc_fence_after();
  if (ok) {
    for (int c0 = 0; c0 < N; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + c0, r);
#pragma unroll
      for (int c = 0; c < 32; ++c) C[(128 * rank + row) * N + c0 + c] = __uint_as_float(r[c]);
    }
  }
  tc_fence_before();
  cluster_sync();  // no CTA leaves while its peer may still use its memory
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 256);
  }
}

__global__ void __launch_bounds__(32, 1)
    diag_tma_kernel(const __grid_constant__ CUtensorMap map, uint8_t* out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t& bar = *reinterpret_cast<uint64_t*>(smem + 2 * kBox);
  int& abort_flag = *reinterpret_cast<int*>(smem + 2 * kBox + 8);
  const uint32_t s = smem_u32(smem);
  if ((s & 1023u) != 0) return;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(smem_u32(&bar), 2 * kBox);
    tma_load_4d(s, &map, smem_u32(&bar), 0, 0, 0, 0);
    tma_load_4d(s + kBox, &map, smem_u32(&bar), 64, 0, 0, 0);
  }
  Bounded bw{&abort_flag, &g_diag_err, 1000000000ull};
  const bool ok = bw.wait(smem_u32(&bar), 0, 2);
  if (ok)
    for (int e = threadIdx.x; e < 2 * kBox; e += 32) out[e] = smem[e];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

extern "C" {

__attribute__((visibility("default"))) int attn_diag_mma(int mode, const void* A, const void* B,
                                                         float* C, void* stream) {
  if (mode < 0 || mode > 7 || !A || !B || !C) return 1;
  const int smem = 4 * kBox + 64;
  if (cudaFuncSetAttribute(diag_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return 2;
  diag_mma_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      mode, static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), C);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

// C (256 x 128 fp32) = the pair product of `mode` (8, 9 or 10) of A (256 x 128)
// and B (128 x 128), both row-major bf16.
__attribute__((visibility("default"))) int attn_diag_mma_pair(int mode, const void* A,
                                                              const void* B, float* C,
                                                              void* stream) {
  if (mode < 8 || mode > 10 || !A || !B || !C) return 1;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      fn == nullptr)
    return 2;
  // A as (D=128, H=1, S=256, B=1) with 128 x 64 boxes; B as (128, 1, 128, 1) with 64 x 64 boxes
  alignas(64) CUtensorMap mapA, mapB;
  const cuuint64_t dA[4] = {128, 1, 256, 1}, dB[4] = {128, 1, 128, 1};
  const cuuint64_t sA[3] = {256, 256, 256 * 256}, sB[3] = {256, 256, 128 * 256};
  const cuuint32_t bA[4] = {64, 1, 128, 1}, bB[4] = {64, 1, 64, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  auto enc = reinterpret_cast<EncodeTiledFn>(fn);
  if (enc(&mapA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(A), dA, sA, bA, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      enc(&mapB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(B), dB, sB, bB, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return 3;
  const int smem = 4 * kBox + 64;
  if (cudaFuncSetAttribute(diag_mma_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return 4;
  diag_mma_pair_kernel<<<2, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      mode, static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), C, mapA,
      mapB);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

__attribute__((visibility("default"))) int attn_diag_tma(const void* A, void* out, void* stream) {
  if (!A || !out) return 1;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      fn == nullptr)
    return 2;
  alignas(64) CUtensorMap map;
  const cuuint64_t dims[4] = {128, 1, 128, 1};
  const cuuint64_t strides[3] = {256, 256, 128 * 256};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  if (reinterpret_cast<EncodeTiledFn>(fn)(
          &map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(A), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return 3;
  const int smem = 2 * kBox + 64;
  if (cudaFuncSetAttribute(diag_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return 4;
  diag_tma_kernel<<<1, 32, smem, static_cast<cudaStream_t>(stream)>>>(map,
                                                                       static_cast<uint8_t*>(out));
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

__attribute__((visibility("default"))) int attn_diag_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  uint32_t w = 0;
  cudaMemcpyFromSymbol(&w, g_diag_err, sizeof(w));
  const uint32_t z = 0;
  cudaMemcpyToSymbol(g_diag_err, &z, sizeof(z));
  return int(w);
}

// Mask bounds of every query row (lo, hi: keys lo..hi visible, none if hi < lo)
// and of every key (qmin, qmax: the rows that see it, before clipping to
// [0, Sq)), as the kernels compute them.
__attribute__((visibility("default"))) int attn_diag_mask_bounds(int Sq, int Sk, int causal,
                                                                 int win_left, int win_right,
                                                                 int* lo, int* hi, int* qmin,
                                                                 int* qmax) {
  if (Sq < 0 || Sk < 0 || !lo || !hi || !qmin || !qmax) return 1;
  const MaskGeom g = MaskGeom::make(Sq, Sk, causal, win_left, win_right);
  for (int i = 0; i < Sq; ++i) {
    lo[i] = g.lo(i);
    hi[i] = g.hi(i);
  }
  for (int j = 0; j < Sk; ++j) {
    qmin[j] = g.qmin(j);
    qmax[j] = g.qmax(j);
  }
  return 0;
}

// Key-tile range [jlo, jhi) the forward visits for query tiles 0..n_tiles-1
// (rows r0 = t * BM .. min(r0 + BM - 1, Sq - 1)); *bm, *bn: its tile sizes.
__attribute__((visibility("default"))) int attn_diag_fwd_tile_ranges(int Sq, int Sk, int causal,
                                                                     int win_left, int win_right,
                                                                     int n_tiles, int* jlo,
                                                                     int* jhi, int* bm, int* bn) {
  if (Sq < 0 || Sk < 0 || n_tiles < 0 || !jlo || !jhi || !bm || !bn) return 1;
  const MaskGeom g = MaskGeom::make(Sq, Sk, causal, win_left, win_right);
  for (int t = 0; t < n_tiles; ++t) {
    const int r0 = t * fwd::BM;
    const int r1 = r0 + fwd::BM - 1 < Sq - 1 ? r0 + fwd::BM - 1 : Sq - 1;
    fwd::tile_range(g, r0, r1, jlo[t], jhi[t]);
  }
  *bm = fwd::BM;
  *bn = fwd::BN;
  return 0;
}

// Query-tile range [qlo, qhi) the backward visits for key tiles 0..n_tiles-1
// (keys n0 = t * BN .. min(n0 + BN - 1, Sk - 1)); *bm, *bn: its tile sizes.
__attribute__((visibility("default"))) int attn_diag_bwd_qtile_ranges(int Sq, int Sk, int causal,
                                                                      int win_left, int win_right,
                                                                      int n_tiles, int* qlo,
                                                                      int* qhi, int* bm, int* bn) {
  if (Sq < 0 || Sk < 0 || n_tiles < 0 || !qlo || !qhi || !bm || !bn) return 1;
  const MaskGeom g = MaskGeom::make(Sq, Sk, causal, win_left, win_right);
  for (int t = 0; t < n_tiles; ++t) {
    const int n0 = t * bwd::BN;
    const int n1 = n0 + bwd::BN - 1 < Sk - 1 ? n0 + bwd::BN - 1 : Sk - 1;
    bwd::qtile_range(g, n0, n1, qlo[t], qhi[t]);
  }
  *bm = bwd::BM;
  *bn = bwd::BN;
  return 0;
}

// (tile, head-batch) of every linear block index of an n_tiles x n_hb grid
// visited in chunked order.
__attribute__((visibility("default"))) int attn_diag_chunked_order(int n_tiles, int n_hb,
                                                                   int chunk, int* tile, int* hb) {
  if (n_tiles < 0 || n_hb < 0 || chunk < 1 || !tile || !hb) return 1;
  for (int lin = 0; lin < n_tiles * n_hb; ++lin) {
    const ChunkedOrder o = chunked_order(lin, n_tiles, n_hb, chunk);
    tile[lin] = o.tile;
    hb[lin] = o.hb;
  }
  return 0;
}

// (mode, tile) of every block index x of the head_dim 256 backward's grid
// (2 n_k + n_q per head); mode 0 dK, 1 dV, 2 dQ.
__attribute__((visibility("default"))) int attn_diag_d256_work(int n_k, int n_q, int causal,
                                                               int* mode, int* tile) {
  if (n_k < 0 || n_q < 0 || !mode || !tile) return 1;
  for (int x = 0; x < 2 * n_k + n_q; ++x) {
    const bwd256::D256Work w = bwd256::d256_work(x, n_k, n_q, causal);
    mode[x] = w.mode;
    tile[x] = w.tile;
  }
  return 0;
}

}  // extern "C"
