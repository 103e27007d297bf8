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
//   attn_diag_tma: a TMA load of a (1, 128, 1, 128) bf16 tensor with the
//     same 4-D map and 128-byte swizzle as the kernels; the raw shared-memory
//     bytes are copied out so the test can check the placement.
// Not part of the product library.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

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

__global__ void diag_exp2_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    float r0, r1;
    f2_unpack(f2_exp2_poly(f2_pack(x[i], x[i + 1])), r0, r1);
    y[i] = r0;
    y[i + 1] = r1;
  }
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

// y = the softmax's polynomial 2^x (pairs); n must be even.
__attribute__((visibility("default"))) int attn_diag_exp2(const float* x, float* y, int n,
                                                          void* stream) {
  if (!x || !y || n <= 0 || (n & 1)) return 1;
  const int pairs = n / 2;
  diag_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

__attribute__((visibility("default"))) int attn_diag_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  uint32_t w = 0;
  cudaMemcpyFromSymbol(&w, g_diag_err, sizeof(w));
  const uint32_t z = 0;
  cudaMemcpyToSymbol(g_diag_err, &z, sizeof(z));
  return int(w);
}

}  // extern "C"
