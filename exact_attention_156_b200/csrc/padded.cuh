// padded.cuh - padded batches: gather the real rows of a (B, S, H, D) batch
// into the packed layout of the variable-length kernels, and scatter packed
// results back with the padding rows of every output cleared.
//
// The pages name both upstream tests test_flash_attn_varlen and
// test_flash_attn_padded (FlashAttention-2 overview, lshu.cn, section 3.2):
// a padded batch holds B sequences of one padded length S, sequence b's real
// rows being 0 .. len[b] - 1.  Padding rows are never read (they may hold
// anything, non-finite values included), so the attention of a padded batch is
// exactly that of the packed batch of its real rows.  All kernels here are
// memory bound: one warp moves one row of H x D 16-bit elements (16 bytes per
// lane per step).
#pragma once

#include <math.h>
#include <stdint.h>

#include "common.cuh"

namespace attn156 {
namespace padded {

// cu[0] = 0, cu[b + 1] = cu[b] + len[b] for the B lengths, by one warp in
// chunks of 32.  A length outside [0, S] is recorded in the device error word
// (ATTN_ERR_SEQLENS) and taken as 0, so nothing of that sequence is read or
// written.  cu[B + 1] receives the number of malformed lengths (0 when valid).
__global__ void __launch_bounds__(32) seqlens_scan_kernel(const int* __restrict__ len, int B,
                                                          int S, int* __restrict__ cu,
                                                          uint32_t* err) {
  const int lane = threadIdx.x;
  int base = 0, bad = 0;
  if (lane == 0) cu[0] = 0;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    int x = 0;
    if (b < B) {
      x = len[b];
      if (x < 0 || x > S) {
        ++bad;
        x = 0;
      }
    }
    // inclusive warp scan
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (b < B) cu[b + 1] = base + x;
    base += __shfl_sync(0xffffffffu, x, 31);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, off);
  if (lane == 0) {
    cu[B + 1] = bad;
    if (bad) atomicCAS(err, 0u, kErrSeqlens);
  }
}

// Length of sequence b as scanned (malformed lengths read as 0).
__device__ __forceinline__ int scanned_len(const int* cu, int b) { return cu[b + 1] - cu[b]; }

// One warp per padded row (b, i) of a (B, S, NH, D) tensor: rows i < len[b]
// are copied to packed row cu[b] + i of a (rows_max, NH, D) tensor.  The
// first `tail` packed rows after the last real one are cleared, so that a
// kernel's ragged last tile reads zeros rather than stale workspace memory
// there (its mask gives those rows weight 0, and 0 x 0 stays 0).
template <int D>
__global__ void __launch_bounds__(256) pack_rows_kernel(const uint16_t* __restrict__ src,
                                                        uint16_t* __restrict__ dst,
                                                        const int* __restrict__ cu, int B, int S,
                                                        int NH, long long rows_max, int tail) {
  const long long gw = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const long long row_elems = (long long)NH * D;  // a multiple of 64
  if (gw < (long long)B * S) {
    const int b = int(gw / S);
    const int i = int(gw % S);
    if (i < scanned_len(cu, b)) {
      const uint4* s4 = reinterpret_cast<const uint4*>(src + gw * row_elems);
      uint4* d4 = reinterpret_cast<uint4*>(dst + ((long long)cu[b] + i) * row_elems);
      for (long long c = lane; c < row_elems / 8; c += 32) d4[c] = s4[c];
    }
  } else if (gw < (long long)B * S + tail) {
    const long long r = (long long)cu[B] + (gw - (long long)B * S);
    if (r < rows_max) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + r * row_elems);
      for (long long c = lane; c < row_elems / 8; c += 32) d4[c] = make_uint4(0, 0, 0, 0);
    }
  }
}

// One warp per padded row (b, i): packed row cu[b] + i back to padded row
// (b, i) for i < len[b]; padding rows are written as zeros.
template <int D>
__global__ void __launch_bounds__(256) unpack_rows_kernel(const uint16_t* __restrict__ src,
                                                          uint16_t* __restrict__ dst,
                                                          const int* __restrict__ cu, int B, int S,
                                                          int NH) {
  const long long gw = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (gw >= (long long)B * S) return;
  const long long row_elems = (long long)NH * D;
  const int b = int(gw / S);
  const int i = int(gw % S);
  uint4* d4 = reinterpret_cast<uint4*>(dst + gw * row_elems);
  if (i < scanned_len(cu, b)) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src + ((long long)cu[b] + i) * row_elems);
    for (long long c = lane; c < row_elems / 8; c += 32) d4[c] = s4[c];
  } else {
    for (long long c = lane; c < row_elems / 8; c += 32) d4[c] = make_uint4(0, 0, 0, 0);
  }
}

// LSE between the padded (B, H, S) layout and the packed (H, total) layout.
// Padded to packed: real rows only.  Packed to padded: padding rows get -inf
// (a row with no key, the convention for rows that attend to nothing).
__global__ void __launch_bounds__(256) pack_lse_kernel(const float* __restrict__ src,
                                                       float* __restrict__ dst,
                                                       const int* __restrict__ cu, int B, int S,
                                                       int H, long long total_max) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)B * H * S) return;
  const int i = int(t % S);
  const long long bh = t / S;
  const int h = int(bh % H);
  const int b = int(bh / H);
  if (i < scanned_len(cu, b)) dst[(long long)h * total_max + cu[b] + i] = src[t];
}

__global__ void __launch_bounds__(256) unpack_lse_kernel(const float* __restrict__ src,
                                                         float* __restrict__ dst,
                                                         const int* __restrict__ cu, int B, int S,
                                                         int H, long long total_max) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)B * H * S) return;
  const int i = int(t % S);
  const long long bh = t / S;
  const int h = int(bh % H);
  const int b = int(bh / H);
  dst[t] = i < scanned_len(cu, b) ? src[(long long)h * total_max + cu[b] + i] : -INFINITY;
}

}  // namespace padded
}  // namespace attn156
