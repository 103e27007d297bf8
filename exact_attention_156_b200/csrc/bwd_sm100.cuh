// bwd_sm100.cuh - recompute-based exact-attention backward for B200 (sm_100a).
//
// Method: the backward rebuilds the attention probabilities from Q, K and the
// forward's per-row log-sum-exp instead of storing them (flash-attn install
// guide, yfxerp.com, section 1, on the backward recomputing the attention
// scores; FlashAttention-2 overview, lshu.cn, section 2.1, second anti-pattern:
// the standard backward re-reads Q, K, V several times).  The gradient is the
// analytic one of O = softmax(scale Q K^T) V:
//   P = exp(scale S - LSE), dV = P^T dO, dP = dO V^T, Delta_i = rowsum(dO*O),
//   dS = P * (dP - Delta), dK = scale dS^T Q, dQ = scale dS K.
//
// Kernels:
//  1. bwd_pre: -Delta_i (fp32), -LSE in base 2 (padded rows: -inf so P = 0),
//     and zeroes the fp32 dQ accumulator.  Memory bound.  Both row values are
//     stored negated so the main kernel adds them with packed fp32 pairs.
//  2. bwd_main: one CTA per (128-key tile, key/value head, batch); K_j and V_j
//     stay in shared memory while the CTA streams the query tiles that can see
//     them, for every query head that reads this K/V head (one, or H / Hk with
//     grouped K/V heads), so dK_j and dV_j accumulate in tensor memory.
//     Transposed products put the key index on tensor-memory lanes:
//       S^T = K Q^T  and  dP^T = V dO^T   (M = keys, N = queries, K = D)
//       dV += P^T dO  (A = P^T from tensor memory)
//       dK += dS^T Q  (A = dS^T from shared memory, K-major)
//       dQ_tile = dS K (A = the same dS^T buffer read MN-major) -> fp32 TMA
//       bulk reduce-add through a dedicated two-slot staging ring
//     warps 0-7: P and dS in two groups of four (one thread = one key row and
//     64 of the tile's 128 query columns; each group keeps its half of P beside
//     its own scores and writes its half of dS^T); warps 8-11: drain dQ;
//     warp 12: MMA issue; warp 13: Q loads; warp 14: dO loads.
//     Q (with its row values) is double buffered, dO single buffered; the MMA
//     order dV(t), S(t+1), dQ(t), dK(t), dP(t+1) lets the next tile's P run
//     while the tensor core finishes this tile's gradients.
//  3. bwd_dq_finalize: dQ = scale * accumulator, rounded to the input format.
// Q, K, V, dO, P, dS and the gradients are bf16 or f16 (template parameter E);
// all accumulation is f32.
// Tensor memory (512 columns): dK [0,D) dV [D,2D) S^T/P^T [2D,2D+128) (P^T as
// 16-bit pairs in [2D,2D+32) and [2D+64,2D+96)), dP^T / dQ [2D+128, 2D+256).
#pragma once

#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "ptx.cuh"

namespace attn156 {
namespace bwd {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // key rows per CTA
// two compute WGs (64 query columns each), dQ-drain WG, control WG {MMA, Q load, dO load, idle}
constexpr int kThreads = 512;
constexpr int kDrainWarp0 = 8;
constexpr int kMmaWarp = 12;
constexpr int kLoadQWarp = 13;
constexpr int kLoadDOWarp = 14;
constexpr int kQStages = 2;
constexpr int kComputeThreads = 256;
// Register split after launch (128 per thread at launch: 512 x 128 = 65536):
// compute 2 x 128 x 136 + drain 128 x 160 + control 128 x 64 = 63488.
constexpr int kLaunchRegs = 128;
constexpr int kComputeRegs = 136;
constexpr int kDrainRegs = 160;
constexpr int kControlRegs = 64;
static_assert(128 * (2 * kComputeRegs + kDrainRegs + kControlRegs) <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

template <int D>
struct Cfg {
  static constexpr int kBoxBytes = 128 * 128;  // one 64-column bf16 box of 128 rows
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kDQChunk = 32;                 // fp32 columns per reduce-add box
  static constexpr int kDQChunks = D / kDQChunk;
  static constexpr int kDQBufBytes = BM * kDQChunk * 4;  // 16 KB, 128-byte rows
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kTileBytes;
  static constexpr int kQOff = kVOff + kTileBytes;                  // [kQStages] Q tiles
  static constexpr int kDOOff = kQOff + kQStages * kTileBytes;      // one dO tile
  static constexpr int kDSOff = kDOOff + kTileBytes;                // dS^T, 128 x 128 bf16
  static constexpr int kDQOff = kDSOff + BN * BM * 2;               // [2] dQ staging boxes
  static constexpr int kLseOff = kDQOff + 2 * kDQBufBytes;          // [kQStages][BM] -LSE*log2e
  static constexpr int kDeltaOff = kLseOff + kQStages * BM * 4;     // [kQStages][BM] -Delta
  static constexpr int kBarOff = kDeltaOff + kQStages * BM * 4;
  static constexpr int kBarKV = 0;
  static constexpr int kBarQFull = 1;
  static constexpr int kBarQEmpty = kBarQFull + kQStages;
  static constexpr int kBarDOFull = kBarQEmpty + kQStages;
  static constexpr int kBarDOEmpty = kBarDOFull + 1;
  static constexpr int kBarS = kBarDOEmpty + 1;
  static constexpr int kBarDP = kBarS + 1;
  static constexpr int kBarP = kBarDP + 1;
  static constexpr int kBarDS = kBarP + 1;
  static constexpr int kBarDSEmpty = kBarDS + 1;
  static constexpr int kBarDQFull = kBarDSEmpty + 1;
  static constexpr int kBarDQEmpty = kBarDQFull + 1;
  static constexpr int kBarDone = kBarDQEmpty + 1;
  static constexpr int kNumBars = kBarDone + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr uint32_t kColDK = 0;
  static constexpr uint32_t kColDV = D;
  static constexpr uint32_t kColS = 2 * D;
  static constexpr uint32_t kColDP = 2 * D + 128;
  static_assert(kSmemBytes <= 232448, "shared memory exceeds the 227 KB per block of sm_100");
  static_assert(kDQOff % 1024 == 0 && kDOOff % 1024 == 0 && kDSOff % 1024 == 0,
                "128-byte-swizzled buffers need 1024-byte alignment");
};

struct Params {
  uint16_t* dk;  // 16-bit elements (bf16 or f16, as the kernel's element format)
  uint16_t* dv;
  const float* nlse2;   // [B*H][Sq_pad] -LSE * log2(e); -inf for padding rows
  const float* ndelta;  // [B*H][Sq_pad] -Delta
  float* dq_acc;       // [B*H][Sq_pad][D]
  int B, H, Sq, Sk, Sq_pad;  // packed sequences: Sq, Sk are the largest lengths
  // Packed variable-length sequences (null for the (B, S, H, D) layout): sequence
  // b is rows cu_q[b] .. cu_q[b+1]-1 of Q/dO and cu_k[b] .. cu_k[b+1]-1 of K/V.
  // The row values and the dQ accumulator then hold, per query head, R rows
  // (varlen_rows): query i of sequence b is row rv_start(cu_q, b) + i, each
  // sequence starting on a 16-byte boundary and followed by >= 128 padding rows.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k, R;
  int compact;  // packed batches: blockIdx.x numbers the key tiles that have work (compact_tile)
  int order_chunk;  // (B, S, H, D) batches: K/V-head-batch combinations per block-order chunk
  int Hk;  // key/value heads: the CTA's K/V head is shared by H / Hk query heads
  float scale;
  float scale_log2;
  int causal, win_left, win_right;
  uint32_t* err;
  uint64_t timeout_ns;
};

// ---------------------------------------------------------------------------
// 1. preprocess: one warp per kPreRows consecutive rows of (b, h, padded query
//    axis); the loads of all its rows are issued before any is reduced, so that
//    enough bytes are in flight to keep HBM busy.
// ---------------------------------------------------------------------------
constexpr int kPreRows = 4;  // divides Sq_pad (a multiple of 128) and the packed R

// One lane's share of a row of O or dO: D / 32 16-bit elements in D / 64 words.
template <int D>
__device__ __forceinline__ void load_row_words(const uint16_t* __restrict__ src,
                                               uint32_t (&w)[D / 64]) {
  const int lane = threadIdx.x % 32;
  if constexpr (D == 256) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + lane * 8);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (D == 128) {
    const uint2 v = *reinterpret_cast<const uint2*>(src + lane * 4);
    w[0] = v.x; w[1] = v.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(src + lane * 2);
  }
}

// Lane sums of O∘dO for kPreRows rows, reduced over the warp; every lane gets
// all kPreRows dot products.
template <int D, class E>
__device__ __forceinline__ void rows_dot(const uint32_t (&ow)[kPreRows][D / 64],
                                         const uint32_t (&dw)[kPreRows][D / 64],
                                         float (&dot)[kPreRows]) {
#pragma unroll
  for (int r = 0; r < kPreRows; ++r) {
    dot[r] = 0.f;
#pragma unroll
    for (int t = 0; t < D / 64; ++t) {
      float a0, a1, c0, c1;
      E::unpack2(ow[r][t], a0, a1);
      E::unpack2(dw[r][t], c0, c1);
      dot[r] = fmaf(a0, c0, dot[r]);
      dot[r] = fmaf(a1, c1, dot[r]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int r = 0; r < kPreRows; ++r) dot[r] += __shfl_xor_sync(0xffffffffu, dot[r], off);
}

template <int D, class E>
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(
    const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
    const float* __restrict__ lse, float* __restrict__ nlse2, float* __restrict__ ndelta,
    float* __restrict__ dq_acc, int B, int H, int Sq, int Sq_pad) {
  const long long g0 = ((long long)blockIdx.x * 8 + threadIdx.x / 32) * kPreRows;
  const int lane = threadIdx.x % 32;
  if (g0 >= (long long)B * H * Sq_pad) return;
  // the warp's rows share (b, h): Sq_pad is a multiple of kPreRows
  const int i0 = int(g0 % Sq_pad);
  const long long bh = g0 / Sq_pad;
  const int h = int(bh % H);
  const int b = int(bh / H);
  uint32_t ow[kPreRows][D / 64], dw[kPreRows][D / 64];
#pragma unroll
  for (int r = 0; r < kPreRows; ++r) {
    if (i0 + r < Sq) {
      const size_t base = ((size_t(b) * Sq + i0 + r) * H + h) * D;
      load_row_words<D>(o + base, ow[r]);
      load_row_words<D>(dout + base, dw[r]);
    } else {
#pragma unroll
      for (int t = 0; t < D / 64; ++t) ow[r][t] = dw[r][t] = 0u;
    }
  }
  float dot[kPreRows];
  rows_dot<D, E>(ow, dw, dot);
  if (lane < kPreRows) {
    // lane r writes row r (dot is warp-uniform after the reduction)
    float dr = dot[0];
#pragma unroll
    for (int r = 1; r < kPreRows; ++r)
      if (lane == r) dr = dot[r];
    const int i = i0 + lane;
    float nl2 = -INFINITY;  // padding rows and rows that see no key: P = 0
    if (i < Sq) {
      const float l = lse[size_t(bh) * Sq + i];
      if (l != -INFINITY) nl2 = -l * 1.4426950408889634f;
    }
    nlse2[g0 + lane] = nl2;
    ndelta[g0 + lane] = -dr;
  }
  // (no accumulator to clear when dQ is written whole rather than reduced into)
  if (dq_acc == nullptr) return;
  float4* acc = reinterpret_cast<float4*>(dq_acc + size_t(g0) * D);
  for (int c = lane; c < kPreRows * D / 4; c += 32) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------
// 3. dQ finalize: dq[b, i, h, :] = 16-bit(scale * acc[b, h, i, :]); 8 elements per thread
// ---------------------------------------------------------------------------
template <int D, class E>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                          uint16_t* __restrict__ dq, int B,
                                                          int H, int Sq, int Sq_pad, float scale) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  constexpr int kVec = D / 8;
  const long long total = (long long)B * Sq * H * kVec;
  if (t >= total) return;
  const int v = int(t % kVec);
  long long r = t / kVec;  // (b, i, h) in BSHD order
  const int h = int(r % H);
  r /= H;
  const int i = int(r % Sq);
  const int b = int(r / Sq);
  const float4* src =
      reinterpret_cast<const float4*>(dq_acc + ((size_t(b) * H + h) * Sq_pad + i) * D + v * 8);
  const float4 a = src[0];
  const float4 c = src[1];
  uint4 w;
  w.x = E::pack2(a.x * scale, a.y * scale);
  w.y = E::pack2(a.z * scale, a.w * scale);
  w.z = E::pack2(c.x * scale, c.y * scale);
  w.w = E::pack2(c.z * scale, c.w * scale);
  *reinterpret_cast<uint4*>(dq + ((size_t(b) * Sq + i) * H + h) * D + v * 8) = w;
}

// ---------------------------------------------------------------------------
// Packed variable-length batches: the preprocess and the dQ finalize.
// ---------------------------------------------------------------------------
// First row of sequence b in the per-head row-value / dQ-accumulator layout
// of packed batches: cu[b] + 132 b rounded up to a multiple of 4 (16 bytes of
// fp32, the alignment of the bulk copies that read the row values).  Sequence
// b's block then has at least Lq_b + 128 rows before sequence b + 1 starts, so
// a ragged query tile never reaches another sequence's rows.
constexpr int kRvGap = BM + 4;
__device__ __forceinline__ long long rv_start(const int* cu, int b) {
  return ((long long)cu[b] + (long long)kRvGap * b + 3) & ~3ll;
}

// Largest b in [0, B) with key(b) <= x for a key non-decreasing in b (true
// for valid boundaries); callers re-check the sequence, so malformed
// boundaries cannot steer an access.
template <class KeyFn>
__device__ __forceinline__ int find_seq(int B, long long x, KeyFn key) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (key(mid) <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// One warp per kPreRows rows of the [H][R] row-value layout: Delta and
// -LSE*log2(e) of query rows, neutral values (P = 0) for the padding rows, dQ
// accumulator zeroed.  Sequence blocks start at multiples of 4 rows, so the
// warp's rows lie in one sequence's block and one search finds it.
template <int D, class E>
__global__ void __launch_bounds__(256) attn_bwd_pre_varlen_kernel(
    const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
    const float* __restrict__ lse, float* __restrict__ nlse2, float* __restrict__ ndelta,
    float* __restrict__ dq_acc, const int* __restrict__ cu_q, const int* __restrict__ cu_k, int B,
    int H, int total_q, int total_k, int max_q, int max_k, int R, uint32_t* err) {
  static_assert(kPreRows == 4, "sequence blocks are aligned to 4 rows");
  const long long g0 = ((long long)blockIdx.x * 8 + threadIdx.x / 32) * kPreRows;
  const int lane = threadIdx.x % 32;
  if (g0 >= (long long)H * R) return;
  const int h = int(g0 / R);
  const long long y0 = g0 % R;
  const int b = find_seq(B, y0, [&](int c) { return rv_start(cu_q, c); });
  const SeqSpan sp = seq_span(cu_q, cu_k, b, total_q, total_k, max_q, max_k);
  if (!sp.ok && lane == 0 && h == 0) atomicCAS(err, 0u, kErrSeqlens);
  const long long i0 = y0 - rv_start(cu_q, b);  // query index of the first row in the sequence
  uint32_t ow[kPreRows][D / 64], dw[kPreRows][D / 64];
#pragma unroll
  for (int r = 0; r < kPreRows; ++r) {
    const long long i = i0 + r;
    if (sp.ok && i >= 0 && i < sp.Lq) {
      const size_t base = ((size_t(sp.q0) + size_t(i)) * H + h) * D;
      load_row_words<D>(o + base, ow[r]);
      load_row_words<D>(dout + base, dw[r]);
    } else {
#pragma unroll
      for (int t = 0; t < D / 64; ++t) ow[r][t] = dw[r][t] = 0u;
    }
  }
  float dot[kPreRows];
  rows_dot<D, E>(ow, dw, dot);
  if (lane < kPreRows) {
    float dr = dot[0];
#pragma unroll
    for (int r = 1; r < kPreRows; ++r)
      if (lane == r) dr = dot[r];
    const long long i = i0 + lane;
    float nl2 = -INFINITY;
    if (sp.ok && i >= 0 && i < sp.Lq) {
      const float l = lse[size_t(h) * total_q + size_t(sp.q0) + size_t(i)];
      if (l != -INFINITY) nl2 = -l * 1.4426950408889634f;
    }
    nlse2[g0 + lane] = nl2;
    ndelta[g0 + lane] = -dr;
  }
  float4* acc = reinterpret_cast<float4*>(dq_acc + size_t(g0) * D);
  for (int c = lane; c < kPreRows * D / 4; c += 32) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dq[x, h, :] = 16-bit(scale * acc[h][rv_start(b) + i]) for packed row x =
// cu_q[b] + i; 8 elements per thread.
template <int D, class E>
__global__ void __launch_bounds__(256) attn_bwd_dq_varlen_kernel(
    const float* __restrict__ dq_acc, uint16_t* __restrict__ dq, const int* __restrict__ cu_q,
    const int* __restrict__ cu_k, int B, int H, int total_q, int total_k, int max_q, int max_k,
    int R, float scale) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  constexpr int kVec = D / 8;
  if (t >= (long long)total_q * H * kVec) return;
  const int v = int(t % kVec);
  const long long r = t / kVec;  // (x, h) in packed (row, head) order
  const int h = int(r % H);
  const long long x = r / H;
  const int b = find_seq(B, x, [&](int c) { return (long long)cu_q[c]; });
  const SeqSpan sp = seq_span(cu_q, cu_k, b, total_q, total_k, max_q, max_k);
  // rows of malformed sequences are left untouched
  if (!sp.ok || x < sp.q0 || x >= (long long)sp.q0 + sp.Lq) return;
  const float4* src = reinterpret_cast<const float4*>(
      dq_acc + (size_t(h) * R + size_t(rv_start(cu_q, b) + (x - sp.q0))) * D + v * 8);
  const float4 a = src[0];
  const float4 c = src[1];
  uint4 w;
  w.x = E::pack2(a.x * scale, a.y * scale);
  w.y = E::pack2(a.z * scale, a.w * scale);
  w.z = E::pack2(c.x * scale, c.y * scale);
  w.w = E::pack2(c.z * scale, c.w * scale);
  *reinterpret_cast<uint4*>(dq + (size_t(x) * H + h) * D + v * 8) = w;
}

// ---------------------------------------------------------------------------
// 2. main backward kernel
// ---------------------------------------------------------------------------
// Query-tile range [qlo, qhi) that can see keys [n0, n1]; empty if qhi <= qlo.
__host__ __device__ __forceinline__ void qtile_range(const MaskGeom& g, int n0, int n1, int& qlo, int& qhi) {
  const int a = max(0, g.qmin(n0));
  const int z = min(g.Sq - 1, g.qmax(n1));
  if (n0 >= g.Sk || z < a) {
    qlo = 0;
    qhi = 0;
    return;
  }
  qlo = a / BM;
  qhi = z / BM + 1;
}

// E: element format of Q, K, V, dO, P, dS and the gradients (ElemBF16 or ElemF16).
template <int D, class E, bool kVarlen>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmDO,
                         const __grid_constant__ CUtensorMap tmDQ, const Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  auto bar = [&](int idx) { return smem_u32(&bars[idx]); };
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(p.err, 0u, 8u);
    return;
  }

  // Grid: (key tile, K/V head, batch), visited in chunked order
  // (chunked_order): key tile 0 (the most query tiles when causal) of every K/V
  // head of a chunk whose Q, dO and dQ accumulator fit in L2 together, then
  // key tile 1, ...
  int kt = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;  // hk: key/value head
  if (p.order_chunk > 1) {
    const int lin = int(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    const ChunkedOrder o =
        chunked_order(lin, int(gridDim.x), int(gridDim.y * gridDim.z), p.order_chunk);
    kt = o.tile;
    hk = o.hb % int(gridDim.y);
    b = o.hb / int(gridDim.y);
  }
  const int cidx = kt;  // compact grids: the tile's index in the compact numbering
  if constexpr (kVarlen) {
    if (p.compact) {
      // one CTA per key tile that has work, low key tiles (the heaviest when
      // causal) first
      b = compact_tile(p.cu_q, p.cu_k, p.B, p.total_q, p.total_k, p.Sq, p.Sk, true, BN,
                       cidx, kt);
      if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 32)
        compact_check(p.cu_q, p.cu_k, p.B, p.total_q, p.total_k, p.Sq, p.Sk, true, BN,
                      (long long)gridDim.x, p.err);
      if (b < 0) return;
    }
  }
  const int group = p.H / p.Hk;  // query heads sharing this K/V head
  // This sequence's lengths, first rows, TMA batch coordinate and row-value base.
  int Lq = p.Sq, Lk = p.Sk, q_row0 = 0, k_row0 = 0, bc = b;
  if constexpr (kVarlen) {
    const SeqSpan sp = seq_span(p.cu_q, p.cu_k, b, p.total_q, p.total_k, p.Sq, p.Sk);
    if (!sp.ok && threadIdx.x == 0) atomicCAS(p.err, 0u, kErrSeqlens);
    Lq = sp.Lq;  // 0 for a malformed sequence: nothing is read or written
    Lk = sp.Lk;
    q_row0 = sp.q0;
    k_row0 = sp.k0;
    bc = 0;
  }
  // first row of query head h's row values / dQ accumulator rows
  auto rv_base = [&](int h) -> long long {
    return kVarlen ? (long long)h * p.R + rv_start(p.cu_q, b) : ((long long)b * p.H + h) * p.Sq_pad;
  };
  const MaskGeom g = MaskGeom::make(Lq, Lk, p.causal, p.win_left, p.win_right);
  const int n0 = kt * BN;
  // No key of this sequence falls in this CTA (shorter sequences of a packed
  // batch): nothing to compute or write.
  if (n0 >= Lk) return;
  const int n1 = min(n0 + BN - 1, Lk - 1);
  int qlo, qhi;
  qtile_range(g, n0, n1, qlo, qhi);
  const int nq_head = qhi - qlo;  // query tiles per query head
  // Work item t of this CTA: query head hk * group + t / nq_head, query tile
  // qlo + t % nq_head.  dK and dV of the K/V head accumulate over all of them.
  const int nq = nq_head * group;
  auto item_head = [&](int t) { return hk * group + t / nq_head; };
  auto item_row0 = [&](int t) { return (qlo + t % nq_head) * BM; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) {
      uint32_t count = 1;
      if (i == C::kBarP || i == C::kBarDS) count = kComputeThreads;
      if (i == C::kBarDQEmpty) count = 128;
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Bounded bw{abort_flag, p.err, p.timeout_ns};
  auto q_addr = [&](int s) { return sbase + C::kQOff + s * C::kTileBytes; };
  const uint32_t do_addr = sbase + C::kDOOff;
  const uint32_t k_addr = sbase + C::kKOff;
  const uint32_t v_addr = sbase + C::kVOff;
  const uint32_t ds_addr = sbase + C::kDSOff;
  int q_loads0 = 0, q_loads1 = 0;  // Q loads issued per slot (slot 0, slot 1)
  int do_loads = 0;
  bool drain_issued = false;

  // ------------------------------------------------------------ teardown
  // Inlined at the end of every role (each role returns after it), so that
  // each role's code is register-allocated on its own.
  auto finish = [&]() {
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
      const uint64_t drain_ns = 2000000000ull;
      auto settle = [&](uint32_t bb, uint32_t parity) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bb, parity))
          if (globaltimer_ns() - t0 > drain_ns) break;
      };
      if (warp == kLoadQWarp && lane == 0 && nq > 0) {
        if (q_loads0 > 0) settle(bar(C::kBarQFull + 0), (q_loads0 - 1) & 1);
        if (q_loads1 > 0) settle(bar(C::kBarQFull + 1), (q_loads1 - 1) & 1);
        settle(bar(C::kBarKV), 0);
      }
      if (warp == kLoadDOWarp && lane == 0 && do_loads > 0)
        settle(bar(C::kBarDOFull), (do_loads - 1) & 1);
      if (warp == kMmaWarp && lane == 0) {
        tc_commit(bar(C::kBarDone));
        settle(bar(C::kBarDone), 0);
      }
      tc_fence_before();
      __syncthreads();
    }
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  };

  if (warp < kDrainWarp0) {
    regs_realloc<kLaunchRegs, kComputeRegs>();
    // ------------------------------------------------------------ P and dS
    // Two groups of four warps: group grp owns query columns [64 grp, 64 grp + 64)
    // of every key row (one thread = one key row per group).  Each group writes
    // its half of P as 16-bit pairs into the first 32 of its own 64 score
    // columns, and its half of dS^T into its own 64-column box.
    const int grp = warp / 4;
    const int quad = warp % 4;
    const int r = quad * 32 + lane;  // key row within the tile
    const int kk_idx = n0 + r;       // key index
    const int cb = 64 * grp;         // first query column of this group
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS + uint32_t(cb);
    const uint32_t tDP = tmem + lane_off + C::kColDP + uint32_t(cb);
    const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
    const int qmin_k = g.qmin(kk_idx);
    const int qmax_k = min(g.qmax(kk_idx), Lq - 1);
    const bool key_ok = kk_idx < Lk;
    // rows of the dS^T buffer: 128 bytes per 64 columns, 16-byte chunks swizzled by row % 8
    const uint32_t ds_row = ds_addr + uint32_t(grp) * C::kBoxBytes + uint32_t(r) * 128;
    const uint32_t sw = uint32_t(r & 7);
    bool ok = true;
    for (int t = 0; t < nq; ++t) {
      const int s = t % kQStages;
      const int i0 = item_row0(t);
      const float4* nl = reinterpret_cast<const float4*>(smem + C::kLseOff + s * BM * 4 + cb * 4);
      const float4* nd = reinterpret_cast<const float4*>(smem + C::kDeltaOff + s * BM * 4 + cb * 4);
      // P = 2^(scale*log2e*S - LSE*log2e), kept as 16-bit pairs (what dV uses) for dS too
      if (!bw.wait_warp(bar(C::kBarS), t & 1, 27)) { ok = false; break; }
      tc_fence_after();
      uint32_t pw[32];
      {
        uint32_t rr[64];
        tmem_ld64(tS, rr);
        const bool full = key_ok && n0 + BN - 1 <= Lk - 1 && i0 + BM - 1 <= Lq - 1 &&
                          i0 >= g.qmin(n0 + BN - 1) && i0 + BM - 1 <= g.qmax(n0);
        if (full) {
          // every entry visible: no mask
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 l4 = nl[c / 4];
            const uint64_t x0 = f2_fma(f2_pack(__uint_as_float(rr[c]), __uint_as_float(rr[c + 1])),
                                       sl2, f2_pack(l4.x, l4.y));
            const uint64_t x1 = f2_fma(
                f2_pack(__uint_as_float(rr[c + 2]), __uint_as_float(rr[c + 3])), sl2,
                f2_pack(l4.z, l4.w));
            float a0, a1, a2, a3;
            f2_unpack(x0, a0, a1);
            f2_unpack(x1, a2, a3);
            pw[c / 2] = E::pack2(ex2_approx(a0), ex2_approx(a1));
            pw[c / 2 + 1] = E::pack2(ex2_approx(a2), ex2_approx(a3));
          }
        } else {
          const int c_lo = key_ok ? qmin_k - i0 - cb : (1 << 30);
          const int c_hi = qmax_k - i0 - cb;
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 l4 = nl[c / 4];
            const uint64_t x0 = f2_fma(f2_pack(__uint_as_float(rr[c]), __uint_as_float(rr[c + 1])),
                                       sl2, f2_pack(l4.x, l4.y));
            const uint64_t x1 = f2_fma(
                f2_pack(__uint_as_float(rr[c + 2]), __uint_as_float(rr[c + 3])), sl2,
                f2_pack(l4.z, l4.w));
            float a[4];
            f2_unpack(x0, a[0], a[1]);
            f2_unpack(x1, a[2], a[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              a[e] = ex2_approx(a[e]);
              if (c + e < c_lo || c + e > c_hi) a[e] = 0.f;
            }
            pw[c / 2] = E::pack2(a[0], a[1]);
            pw[c / 2 + 1] = E::pack2(a[2], a[3]);
          }
        }
      }
      tmem_st32(tS, pw);
      tc_fence_before();
      mbar_arrive(bar(C::kBarP));

      // dS = P * (dP - Delta) -> 16-bit, written swizzled for the dK and dQ products
      if (!bw.wait_warp(bar(C::kBarDP), t & 1, 28)) { ok = false; break; }
      tc_fence_after();
      uint32_t rr[64];
      tmem_ld64(tDP, rr);
      if (t > 0 && !bw.wait_warp(bar(C::kBarDSEmpty), (t - 1) & 1, 29)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < 64; c += 8) {
        const float4 d0 = nd[c / 4];
        const float4 d1 = nd[c / 4 + 1];
        const float dl[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float pl, ph;
          E::unpack2(pw[c / 2 + e], pl, ph);
          const uint64_t p2 = f2_pack(pl, ph);
          const uint64_t gd = f2_add(
              f2_pack(__uint_as_float(rr[c + 2 * e]), __uint_as_float(rr[c + 2 * e + 1])),
              f2_pack(dl[2 * e], dl[2 * e + 1]));
          float a0, a1;
          f2_unpack(f2_mul(p2, gd), a0, a1);
          w[e] = E::pack2(a0, a1);
        }
        const uint32_t chunk = uint32_t(c / 8);
        st_shared_v4(ds_row + ((chunk ^ sw) << 4), w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(C::kBarDS));
    }
    // epilogue: group 0 writes dK = scale * acc, group 1 dV = acc (16-bit), once the
    // last dK product is done
    if (ok && nq > 0) ok = bw.wait_warp(bar(C::kBarDSEmpty), (nq - 1) & 1, 30);
    if (ok) {
      tc_fence_after();
      const size_t orow =
          ((kVarlen ? size_t(k_row0) + kk_idx : size_t(b) * p.Sk + size_t(kk_idx)) * p.Hk + hk) * D;
      const uint32_t col = grp == 0 ? C::kColDK : C::kColDV;
      const float mul = grp == 0 ? p.scale : 1.0f;
      uint16_t* outp = grp == 0 ? p.dk : p.dv;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t rr[32];
        if (nq > 0) {
          tmem_ld32(tmem + lane_off + col + c0, rr);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) rr[c] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = E::pack2(__uint_as_float(rr[2 * c]) * mul, __uint_as_float(rr[2 * c + 1]) * mul);
        if (key_ok) {
          uint8_t* dst = reinterpret_cast<uint8_t*>(outp + orow + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            st_global_v4(dst + 16 * v, w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
    }
    finish();
    return;
  }
  if (warp < kMmaWarp) {
    regs_realloc<kLaunchRegs, kDrainRegs>();
    // ------------------------------------------------------------ dQ drain
    // TMEM -> registers (then the tensor memory is handed back at once) ->
    // 32-column fp32 boxes (128-byte swizzle) in a two-slot staging ring ->
    // one TMA reduce-add per box into the fp32 accumulator.
    const int quad = warp % 4;
    const int r = quad * 32 + lane;  // query row within the tile
    const uint32_t tDQ = tmem + (uint32_t(quad * 32) << 16) + C::kColDP;
    const uint32_t sw = uint32_t(r & 7);
    const bool leader = (warp == kDrainWarp0 && lane == 0);
    if (leader) tma_prefetch_desc(&tmDQ);
    int n = 0;  // boxes issued so far
    for (int t = 0; t < nq; ++t) {
      // all four drain warps continue or stop together (they meet at named barriers)
      if (!named_bar_and(1, 128, bw.wait(bar(C::kBarDQFull), t & 1, 31))) break;
      tc_fence_after();
      uint32_t rr[D];
      if constexpr (D == 128) {
        uint32_t (&lo)[64] = *reinterpret_cast<uint32_t(*)[64]>(&rr[0]);
        uint32_t (&hi)[64] = *reinterpret_cast<uint32_t(*)[64]>(&rr[64]);
        tmem_ld64(tDQ, lo);
        tmem_ld64(tDQ + 64, hi);
      } else {
        tmem_ld64(tDQ, rr);
      }
      // tensor memory is free again: the MMA warp may start dP of the next tile
      tc_fence_before();
      mbar_arrive(bar(C::kBarDQEmpty));
      const int row0 = int(rv_base(item_head(t)) + item_row0(t));
#pragma unroll
      for (int c = 0; c < C::kDQChunks; ++c, ++n) {
        const uint32_t buf = sbase + C::kDQOff + uint32_t(n & 1) * C::kDQBufBytes;
        // the reduce that last read this slot (two boxes ago) must have finished reading
        if (leader && n >= 2) bulk_wait_read<1>();
        named_bar_sync(1, 128);
        const uint32_t row = buf + uint32_t(r) * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          st_shared_v4(row + ((uint32_t(k) ^ sw) << 4), rr[c * 32 + 4 * k], rr[c * 32 + 4 * k + 1],
                       rr[c * 32 + 4 * k + 2], rr[c * 32 + 4 * k + 3]);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader) {
          tma_reduce_add_2d(&tmDQ, buf, c * C::kDQChunk, row0);
          bulk_commit();
          drain_issued = true;
        }
      }
    }
    if (leader && drain_issued) bulk_wait_all();
    finish();
    return;
  }
  regs_realloc<kLaunchRegs, kControlRegs>();
  if (warp == kLoadQWarp) {
    // ------------------------------------------------------------ K, V, Q (+ row values)
    if (lane == 0 && nq > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(C::kBarKV), 2 * C::kTileBytes);
      for (int x = 0; x < C::kBoxes; ++x) {
        tma_load_4d(k_addr + x * C::kBoxBytes, &tmK, bar(C::kBarKV), x * 64, hk, k_row0 + n0, bc);
        tma_load_4d(v_addr + x * C::kBoxBytes, &tmV, bar(C::kBarKV), x * 64, hk, k_row0 + n0, bc);
      }
      for (int t = 0; t < nq; ++t) {
        const int s = t % kQStages;
        const int u = t / kQStages;
        if (u > 0 && !bw.wait(bar(C::kBarQEmpty + s), (u - 1) & 1, 20)) break;
        const int i0 = item_row0(t);
        const int h = item_head(t);
        const uint32_t fb = bar(C::kBarQFull + s);
        mbar_arrive_expect_tx(fb, C::kTileBytes + 2 * BM * 4);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_4d(q_addr(s) + x * C::kBoxBytes, &tmQ, fb, x * 64, h, q_row0 + i0, bc);
        const size_t roff = size_t(rv_base(h) + i0);
        bulk_load(sbase + C::kLseOff + s * BM * 4, p.nlse2 + roff, BM * 4, fb);
        bulk_load(sbase + C::kDeltaOff + s * BM * 4, p.ndelta + roff, BM * 4, fb);
        if (s == 0) ++q_loads0; else ++q_loads1;
      }
    }
  } else if (warp == kLoadDOWarp) {
    // ------------------------------------------------------------ dO
    if (lane == 0 && nq > 0) {
      tma_prefetch_desc(&tmDO);
      for (int t = 0; t < nq; ++t) {
        if (t > 0 && !bw.wait(bar(C::kBarDOEmpty), (t - 1) & 1, 32)) break;
        const int i0 = item_row0(t);
        mbar_arrive_expect_tx(bar(C::kBarDOFull), C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_4d(do_addr + x * C::kBoxBytes, &tmDO, bar(C::kBarDOFull), x * 64, item_head(t),
                      q_row0 + i0, bc);
        do_loads++;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && nq > 0) {
      constexpr uint32_t id_s = idesc_f32acc(BN, BM, false, false, E::kFmt);  // S^T, dP^T
      constexpr uint32_t id_dv = idesc_f32acc(BN, D, false, true, E::kFmt);   // dV, dK
      constexpr uint32_t id_dq = idesc_f32acc(BM, D, true, true, E::kFmt);    // dQ
      auto issue_kmajor = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
        if constexpr (D == 128)
          mma_chain_kk8(tmem + d_col, sdesc_sw128(a_base, 16), sdesc_sw128(b_base, 16), id_s, 0u);
        else
          mma_chain_kk4(tmem + d_col, sdesc_sw128(a_base, 16), sdesc_sw128(b_base, 16), id_s, 0u);
      };
      bool ok = bw.wait(bar(C::kBarKV), 0, 21);
      if (ok) ok = bw.wait(bar(C::kBarQFull + 0), 0, 22);
      if (ok) {
        tc_fence_after();
        issue_kmajor(C::kColS, k_addr, q_addr(0));
        tc_commit(bar(C::kBarS));
        ok = bw.wait(bar(C::kBarDOFull), 0, 33);
      }
      if (ok) {
        tc_fence_after();
        issue_kmajor(C::kColDP, v_addr, do_addr);
        tc_commit(bar(C::kBarDP));
      }
      for (int t = 0; ok && t < nq; ++t) {
        const int s = t % kQStages;
        const bool more = t + 1 < nq;
        // dV += P^T dO   (A = P^T in tensor memory, K = query index)
        if (!bw.wait(bar(C::kBarP), t & 1, 23)) { ok = false; break; }
        tc_fence_after();
        mma_chain_ts_mn8_split64(tmem + C::kColDV, tmem + C::kColS,
                                 sdesc_sw128(do_addr, C::kBoxBytes), id_dv, t > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarDOEmpty));
        // next S^T: overwrites P^T only after dV has read it (same issue order)
        if (more) {
          const int s1 = (t + 1) % kQStages;
          if (!bw.wait(bar(C::kBarQFull + s1), ((t + 1) / kQStages) & 1, 25)) { ok = false; break; }
          tc_fence_after();
          issue_kmajor(C::kColS, k_addr, q_addr(s1));
          tc_commit(bar(C::kBarS));
        }
        if (!bw.wait(bar(C::kBarDS), t & 1, 24)) { ok = false; break; }
        tc_fence_after();
        // dQ_tile = dS K  (A = dS read MN-major: rows of the buffer are keys = K index)
        mma_chain_mnmn8(tmem + C::kColDP, sdesc_sw128(ds_addr, C::kBoxBytes),
                        sdesc_sw128(k_addr, C::kBoxBytes), id_dq, 0u);
        tc_commit(bar(C::kBarDQFull));
        // dK += dS^T Q   (A = dS^T in shared memory, K-major over the query index)
        mma_chain_kmn8(tmem + C::kColDK, sdesc_sw128(ds_addr, 16),
                       sdesc_sw128(q_addr(s), C::kBoxBytes), id_dv, t > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarQEmpty + s));
        tc_commit(bar(C::kBarDSEmpty));
        if (more) {
          // dP^T of the next tile reuses the dQ columns once the drain has read them
          if (!bw.wait(bar(C::kBarDQEmpty), t & 1, 26)) { ok = false; break; }
          if (!bw.wait(bar(C::kBarDOFull), (t + 1) & 1, 34)) { ok = false; break; }
          tc_fence_after();
          issue_kmajor(C::kColDP, v_addr, do_addr);
          tc_commit(bar(C::kBarDP));
        }
      }
    }
  }
  finish();
}

}  // namespace bwd
}  // namespace attn156
