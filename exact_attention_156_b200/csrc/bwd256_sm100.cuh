// bwd256_sm100.cuh - recompute-based exact-attention backward at head_dim 256
// on B200 (sm_100a).
//
// Method: as the head_dim 64/128 backward (flash-attn install guide,
// yfxerp.com, section 1: the backward recomputes the attention scores from Q,
// K and the forward's log-sum-exp); the gradient is the analytic one:
//   P = exp(scale S - LSE), dV = P^T dO, dP = dO V^T, dS = P * (dP - Delta),
//   dK = scale dS^T Q, dQ = scale dS K.
//
// B200 mapping.  At head_dim 256 one 128-row accumulator of a gradient takes
// 256 of the 512 tensor-memory columns, and one 128-row tile of Q, K, V or dO
// takes 64 KB of shared memory, so dK and dV cannot share a CTA (their
// accumulators alone fill tensor memory).  Each CTA accumulates ONE gradient
// tile in tensor memory, over 64-wide steps of the other sequence axis:
//   mode dK (CTA = 128 keys):    X = K Q^T, Y = V dO^T, Z = dS^T = P^T (Y - Delta)
//                                dK += Z Q
//   mode dV (CTA = 128 keys):    X = K Q^T,             Z = P^T
//                                dV += Z dO
//   mode dQ (CTA = 128 queries): X = Q K^T, Y = dO V^T, Z = dS = P (Y - Delta)
//                                dQ += Z K   (written as float32; the dQ
//                                finalize kernel scales and rounds it)
// X and Y are M = 128, N = 64, K = 256 products of two shared-memory operands;
// Z (16-bit) is written by the compute warps into tensor memory over X, and
// the accumulation Z B (M = 128, N = 256, K = 64) reads it from there, so Z
// never touches shared memory (a tensor-memory A operand is as fast as a
// shared-memory one only at N = 256).  X and Y are double-buffered in tensor memory,
// so the products of step t + 1 run while the compute warps form Z of step t.
// The three modes are one launch (blockIdx.x picks mode and tile); they share
// nothing but their inputs, so their CTAs run side by side.  The scores are
// recomputed three times (once per gradient) instead of once: the price of
// fitting head_dim 256 into one SM's tensor and shared memory.
//
// Roles (384 threads): warps 0-3 / 4-7 compute Z for columns [0,32) / [32,64)
// of every step (one thread = one accumulator row = one TMEM lane in each
// group; each group writes its Z over its own X columns, so the groups never
// wait for each other) and write half of the gradient tile; warp 8 issues the
// tcgen05 products; warp 9 loads the two resident 128-row tiles and then the
// first streamed operand (two slots, with the step's row values in dK / dV
// mode); warp 10 loads the second streamed operand (one slot; two in dV mode).
// Steps are issued in pairs: the accumulations of steps t - 1 and t, then the
// products X, Y of steps t + 1 and t + 2, so a slot's next load overlaps an
// accumulation and the other step's products instead of stalling the tensor
// core (15% faster than one step at a time on B1 H16 S8192 causal).
// Tensor memory: accumulator [0,256), X0 [256,320), X1 [320,384),
// Y0 [384,448), Y1 [448,512); the Z of a group (16-bit pairs) overwrites the
// first 16 of that group's 32 columns of its X buffer.
#pragma once

#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "ptx.cuh"
#include "ptx_d256.cuh"

namespace attn156 {
namespace bwd256 {

constexpr int D = 256;
constexpr int BR = 128;  // accumulator rows per CTA (keys, or queries in dQ mode)
constexpr int BC = 64;   // columns per step (queries, or keys in dQ mode)
constexpr int kThreads = 384;
constexpr int kMmaWarp = 8;
constexpr int kLoad1Warp = 9;
constexpr int kLoad2Warp = 10;
constexpr int kComputeThreads = 256;  // two groups: columns [0,32) and [32,64) of a step
constexpr int kModeDK = 0, kModeDV = 1, kModeDQ = 2;

// The gradient (mode) and tile of block index x of one head, for n_k key tiles
// and n_q query tiles: in threes, the dK and dV tiles of key tile l and the dQ
// tile of the l-th heaviest query tile (with a causal mask low key tiles see
// the most queries and high query tiles the most keys), then the remaining
// tiles of the longer axis, dK and dV alternating.  The 2 n_k + n_q indices
// name every (mode, tile) once.
struct D256Work {
  int mode, tile;
};
__host__ __device__ __forceinline__ D256Work d256_work(int bx, int n_k, int n_q, int causal) {
  const int nmin = n_k < n_q ? n_k : n_q;
  D256Work w;
  if (bx < 3 * nmin) {
    const int l = bx / 3, m = bx % 3;
    w.mode = m == 0 ? kModeDK : (m == 1 ? kModeDV : kModeDQ);
    w.tile = (m == 2 && causal) ? n_q - 1 - l : l;
  } else if (n_k > nmin) {
    const int r = bx - 3 * nmin;
    w.mode = r & 1 ? kModeDV : kModeDK;
    w.tile = nmin + (r >> 1);
  } else {
    w.mode = kModeDQ;
    const int q = nmin + (bx - 3 * nmin);
    w.tile = causal ? n_q - 1 - q : q;
  }
  return w;
}

struct Cfg {
  static constexpr int kRBox = BR * 128;        // 128 rows x 64 columns (16 KB)
  static constexpr int kRBytes = 4 * kRBox;     // a resident 128 x 256 tile (64 KB)
  static constexpr int kSBox = BC * 128;        // 64 rows x 64 columns (8 KB)
  static constexpr int kSBytes = 4 * kSBox;     // a streamed 64 x 256 tile (32 KB)
  static constexpr int kR1Off = 0;
  static constexpr int kR2Off = kRBytes;                 // dV mode: second slot of operand 2
  static constexpr int kS1Off = 2 * kRBytes;             // [2] streamed operand 1
  static constexpr int kS2Off = kS1Off + 2 * kSBytes;    // streamed operand 2 (slot 0)
  static constexpr int kRowOff = kS2Off + kSBytes;       // [2 slots][2][BC] f32 row values
  static constexpr int kBarOff = kRowOff + 2 * 2 * BC * 4;
  static constexpr int kBarR = 0;
  static constexpr int kBarS1Full = 1;                   // [2]
  static constexpr int kBarS1Empty = kBarS1Full + 2;     // [2]
  static constexpr int kBarS2Full = kBarS1Empty + 2;     // [2]
  static constexpr int kBarS2Empty = kBarS2Full + 2;     // [2]
  static constexpr int kBarX = kBarS2Empty + 2;          // [2] X (and Y) of a buffer done
  static constexpr int kBarZ = kBarX + 2;                // Z written (256 arrivals)
  static constexpr int kBarAcc = kBarZ + 1;              // last accumulation done
  static constexpr int kBarDone = kBarAcc + 1;
  static constexpr int kNumBars = kBarDone + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr uint32_t kColAcc = 0;
  __device__ static constexpr uint32_t col_x(int t) { return 256u + uint32_t(t & 1) * 64u; }
  __device__ static constexpr uint32_t col_y(int t) { return 384u + uint32_t(t & 1) * 64u; }
  static_assert(kSmemBytes <= 232448, "shared memory exceeds the 227 KB per block of sm_100");
  static_assert(kS1Off % 1024 == 0 && kS2Off % 1024 == 0 && kRowOff % 16 == 0,
                "swizzled tiles need 1024-byte alignment, bulk copies 16");
};

struct Params {
  uint16_t* dk;  // 16-bit elements (bf16 or f16, as the kernel's element format)
  uint16_t* dv;
  float* dq_acc;        // [B*H][Sq_pad][256]: dS K (unscaled), row by row
  const float* nlse2;   // [B*H][Sq_pad] -LSE * log2(e); -inf for padding rows
  const float* ndelta;  // [B*H][Sq_pad] -Delta
  int B, H, Hk, Sq, Sk, Sq_pad;
  int n_ktiles, n_qtiles;  // ceil(Sk / 128), ceil(Sq / 128)
  int order_chunk;         // head-batch combinations per block-order chunk (chunked_order)
  float scale;
  float scale_log2;
  int causal, win_left, win_right;
  uint32_t* err;
  uint64_t timeout_ns;
};

// E: element format of Q, K, V, dO and the gradients (ElemBF16 or ElemF16).
// Tensor maps: the four inputs with 128-row boxes (resident tiles) and with
// 64-row boxes (streamed tiles), all 64 columns wide with 128-byte swizzle.
template <class E>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ128,
                         const __grid_constant__ CUtensorMap tmK128,
                         const __grid_constant__ CUtensorMap tmV128,
                         const __grid_constant__ CUtensorMap tmDO128,
                         const __grid_constant__ CUtensorMap tmQ64,
                         const __grid_constant__ CUtensorMap tmK64,
                         const __grid_constant__ CUtensorMap tmV64,
                         const __grid_constant__ CUtensorMap tmDO64, const Params p) {
  using C = Cfg;
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

  // Block index x (per head): the gradient and tile of d256_work.  y: the
  // query head (dQ) or key/value head (dK, dV; CTAs with y >= Hk have nothing
  // to do).  The (x, head) pairs are visited in chunked order over the heads
  // (chunked_order).
  int bx = blockIdx.x, hy = blockIdx.y, b = blockIdx.z;  // hy: dQ query head, dK/dV K/V head
  if (p.order_chunk > 1) {
    const int lin = int(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    const ChunkedOrder o =
        chunked_order(lin, int(gridDim.x), int(gridDim.y * gridDim.z), p.order_chunk);
    bx = o.tile;
    hy = o.hb % int(gridDim.y);
    b = o.hb / int(gridDim.y);
  }
  const D256Work work = d256_work(bx, p.n_ktiles, p.n_qtiles, p.causal);
  const int mode = work.mode, tile = work.tile;
  const int group = p.H / p.Hk;
  if (mode != kModeDQ && hy >= p.Hk) return;
  const MaskGeom g = MaskGeom::make(p.Sq, p.Sk, p.causal, p.win_left, p.win_right);
  const int r0 = tile * BR;   // first accumulator row (key, or query in dQ mode)
  const int r1 = mode == kModeDQ ? min(r0 + BR - 1, p.Sq - 1) : min(r0 + BR - 1, p.Sk - 1);
  // steps [slo, shi) of 64 columns per head, over nheads heads
  int slo = 0, shi = 0;
  if (mode == kModeDQ) {
    const int klo = g.lo(r0), khi = g.hi(r1);
    if (khi >= klo && khi >= 0) {
      slo = klo / BC;
      shi = khi / BC + 1;
    }
  } else {
    const int a = max(0, g.qmin(r0));
    const int z = min(p.Sq - 1, g.qmax(r1));
    if (z >= a) {
      slo = a / BC;
      shi = z / BC + 1;
    }
  }
  const int per_head = shi - slo;
  const int n = mode == kModeDQ ? per_head : per_head * group;
  // step t: head and first column
  auto step_head = [&](int t) { return mode == kModeDQ ? hy : hy * group + t / per_head; };
  auto step_col0 = [&](int t) { return (slo + (mode == kModeDQ ? t : t % per_head)) * BC; };
  const int hk_dq = hy / group;  // dQ mode: the key/value head of this query head

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i)
      mbar_init(bar(i), i == C::kBarZ ? uint32_t(kComputeThreads) : 1u);
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
  const bool has_y = mode != kModeDV;
  auto s1_addr = [&](int t) { return sbase + C::kS1Off + uint32_t(t & 1) * C::kSBytes; };
  // operand 2: one slot in dK / dQ mode (read only by Y), two in dV mode (read
  // by the accumulation, like operand 1)
  auto s2_slot = [&](int t) { return has_y ? 0 : (t & 1); };
  auto s2_phase = [&](int t) { return has_y ? (t & 1) : ((t >> 1) & 1); };
  auto s2_addr = [&](int t) {
    return sbase + (s2_slot(t) == 0 ? uint32_t(C::kS2Off) : uint32_t(C::kR2Off));
  };
  int loads1 = 0, loads2 = 0;  // streamed loads issued (loader threads only)

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
      if (warp == kLoad1Warp && lane == 0 && n > 0) {
        settle(bar(C::kBarR), 0);
        for (int t = loads1 - 2 > 0 ? loads1 - 2 : 0; t < loads1; ++t)
          settle(bar(C::kBarS1Full + (t & 1)), (t >> 1) & 1);
      }
      if (warp == kLoad2Warp && lane == 0) {
        const int depth = has_y ? 1 : 2;
        for (int t = loads2 - depth > 0 ? loads2 - depth : 0; t < loads2; ++t)
          settle(bar(C::kBarS2Full + s2_slot(t)), s2_phase(t));
      }
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

  if (warp < 8) {
    // ------------------------------------------------------------ Z and the epilogue
    const int grp = warp / 4;  // columns [32 grp, 32 grp + 32) of every step
    const int quad = warp % 4;
    const int r = quad * 32 + lane;
    const int ri = r0 + r;  // this thread's key (dK, dV) or query (dQ)
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
    // dQ mode: this row's values are fixed for the whole CTA
    float nl_row = -INFINITY, nd_row = 0.f;
    if (mode == kModeDQ && ri < p.Sq) {
      const size_t rv = (size_t(b) * p.H + hy) * p.Sq_pad + ri;
      nl_row = p.nlse2[rv];
      nd_row = p.ndelta[rv];
    }
    // visible columns of this row, relative to a step's first column
    int vis_lo, vis_hi;
    if (mode == kModeDQ) {
      vis_lo = ri < p.Sq ? g.lo(ri) : (1 << 30);
      vis_hi = g.hi(ri);
    } else {
      vis_lo = ri < p.Sk ? max(0, g.qmin(ri)) : (1 << 30);
      vis_hi = min(g.qmax(ri), p.Sq - 1);
    }
    // the whole 128 x 64 block is visible (no mask needed) for a step at c0 iff
    const int row_lo_max = mode == kModeDQ ? g.lo(r1) : max(0, g.qmin(r1));
    const int row_hi_min = mode == kModeDQ ? g.hi(r0) : min(g.qmax(r0), p.Sq - 1);
    const bool rows_valid = mode == kModeDQ ? (r0 + BR - 1 < p.Sq) : (r0 + BR - 1 < p.Sk);
    bool ok = true;
    for (int t = 0; t < n; ++t) {
      if (!bw.wait_warp(bar(C::kBarX + (t & 1)), (t >> 1) & 1, 60)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tX = tmem + lane_off + C::col_x(t) + uint32_t(grp * 32);
      uint32_t xr[32];
      tmem_ld32(tX, xr);
      uint32_t yr[32];
      if (has_y) tmem_ld32(tmem + lane_off + C::col_y(t) + uint32_t(grp * 32), yr);
      const int c0 = step_col0(t);
      const float* rows =
          reinterpret_cast<const float*>(smem + C::kRowOff) + (t & 1) * 2 * BC + grp * 32;
      const bool full = rows_valid && c0 >= row_lo_max && c0 + BC - 1 <= row_hi_min;
      const int c_lo = vis_lo - c0 - grp * 32, c_hi = vis_hi - c0 - grp * 32;
      uint32_t zw[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float nl0, nl1, nd0, nd1;
        if (mode == kModeDQ) {
          nl0 = nl1 = nl_row;
          nd0 = nd1 = nd_row;
        } else {
          nl0 = rows[c];
          nl1 = rows[c + 1];
          nd0 = rows[BC + c];
          nd1 = rows[BC + c + 1];
        }
        float a0, a1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(xr[c]), __uint_as_float(xr[c + 1])), sl2,
                         f2_pack(nl0, nl1)),
                  a0, a1);
        a0 = ex2_approx(a0);
        a1 = ex2_approx(a1);
        if (!full) {
          if (c < c_lo || c > c_hi) a0 = 0.f;
          if (c + 1 < c_lo || c + 1 > c_hi) a1 = 0.f;
        }
        // P rounded to the 16-bit format (what dV uses); dS is formed from it
        const uint32_t pw = E::pack2(a0, a1);
        if (has_y) {
          float q0, q1;
          E::unpack2(pw, q0, q1);
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(q0, q1),
                           f2_add(f2_pack(__uint_as_float(yr[c]), __uint_as_float(yr[c + 1])),
                                  f2_pack(nd0, nd1))),
                    d0, d1);
          zw[c / 2] = E::pack2(d0, d1);
        } else {
          zw[c / 2] = pw;
        }
      }
      // Z of this group's 32 columns -> 16 columns at the start of its own X
      // columns (the other group's X is never touched)
      tmem_st16(tX, zw);
      tc_fence_before();
      mbar_arrive(bar(C::kBarZ));
    }
    // epilogue: dK = scale acc, dV = acc (16-bit); dQ: acc as float32 rows
    if (ok && n > 0) ok = bw.wait_warp(bar(C::kBarAcc), 0, 61);
    if (ok) {
      tc_fence_after();
      const bool row_ok = mode == kModeDQ ? ri < p.Sq : ri < p.Sk;
#pragma unroll 1
      for (int c0 = grp * (D / 2); c0 < (grp + 1) * (D / 2); c0 += 32) {
        uint32_t rr[32];
        if (n > 0) {
          tmem_ld32(tmem + lane_off + C::kColAcc + c0, rr);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) rr[c] = 0u;
        }
        if (!row_ok) continue;
        if (mode == kModeDQ) {
          float* dst = p.dq_acc + ((size_t(b) * p.H + hy) * p.Sq_pad + ri) * D + c0;
#pragma unroll
          for (int v = 0; v < 8; ++v)
            st_global_v4(dst + 4 * v, rr[4 * v], rr[4 * v + 1], rr[4 * v + 2], rr[4 * v + 3]);
        } else {
          const float mul = mode == kModeDK ? p.scale : 1.0f;
          uint16_t* outp = mode == kModeDK ? p.dk : p.dv;
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = E::pack2(__uint_as_float(rr[2 * c]) * mul, __uint_as_float(rr[2 * c + 1]) * mul);
          uint8_t* dst = reinterpret_cast<uint8_t*>(
              outp + ((size_t(b) * p.Sk + size_t(ri)) * p.Hk + hy) * D + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            st_global_v4(dst + 16 * v, w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
    }
    finish();
    return;
  }

  // resident tiles and streamed operands of this mode
  const CUtensorMap* mR1 = mode == kModeDQ ? &tmQ128 : &tmK128;
  const CUtensorMap* mR2 = mode == kModeDQ ? &tmDO128 : &tmV128;
  const CUtensorMap* mS1 = mode == kModeDQ ? &tmK64 : &tmQ64;
  const CUtensorMap* mS2 = mode == kModeDQ ? &tmV64 : &tmDO64;

  if (warp == kLoad1Warp) {
    // ------------------------------------------------------------ residents, operand 1 (+ row values)
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(mR1);
      tma_prefetch_desc(mS1);
      const int rh = mode == kModeDQ ? hy : hy;  // head coordinate of the resident tiles
      mbar_arrive_expect_tx(bar(C::kBarR), (has_y ? 2 : 1) * C::kRBytes);
      for (int x = 0; x < 4; ++x) {
        tma_load_4d(sbase + C::kR1Off + x * C::kRBox, mR1, bar(C::kBarR), x * 64, rh, r0, b);
        if (has_y)
          tma_load_4d(sbase + C::kR2Off + x * C::kRBox, mR2, bar(C::kBarR), x * 64, rh, r0, b);
      }
      for (int t = 0; t < n; ++t) {
        if (t >= 2 && !bw.wait(bar(C::kBarS1Empty + (t & 1)), ((t >> 1) - 1) & 1, 62)) break;
        const uint32_t fb = bar(C::kBarS1Full + (t & 1));
        const int c0 = step_col0(t);
        const int sh = mode == kModeDQ ? hk_dq : step_head(t);
        const bool rows = mode != kModeDQ;
        mbar_arrive_expect_tx(fb, C::kSBytes + (rows ? 2 * BC * 4 : 0));
        for (int x = 0; x < 4; ++x)
          tma_load_4d(s1_addr(t) + x * C::kSBox, mS1, fb, x * 64, sh, c0, b);
        if (rows) {
          const size_t rv = (size_t(b) * p.H + sh) * p.Sq_pad + c0;
          const uint32_t dst = sbase + C::kRowOff + (t & 1) * 2 * BC * 4;
          bulk_load(dst, p.nlse2 + rv, BC * 4, fb);
          bulk_load(dst + BC * 4, p.ndelta + rv, BC * 4, fb);
        }
        ++loads1;
      }
    }
  } else if (warp == kLoad2Warp) {
    // ------------------------------------------------------------ operand 2
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(mS2);
      const int depth = has_y ? 1 : 2;
      for (int t = 0; t < n; ++t) {
        if (t >= depth && !bw.wait(bar(C::kBarS2Empty + s2_slot(t)), s2_phase(t) ^ 1, 63)) break;
        const uint32_t fb = bar(C::kBarS2Full + s2_slot(t));
        const int sh = mode == kModeDQ ? hk_dq : step_head(t);
        mbar_arrive_expect_tx(fb, C::kSBytes);
        for (int x = 0; x < 4; ++x)
          tma_load_4d(s2_addr(t) + x * C::kSBox, mS2, fb, x * 64, sh, step_col0(t), b);
        ++loads2;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ tcgen05 issue
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_xy = idesc_f32acc(BR, BC, false, false, E::kFmt);
      constexpr uint32_t id_acc = idesc_f32acc(BR, D, false, true, E::kFmt);
      bool ok = bw.wait(bar(C::kBarR), 0, 64);
      auto issue_xy = [&](int t) -> bool {
        if (!bw.wait(bar(C::kBarS1Full + (t & 1)), (t >> 1) & 1, 65)) return false;
        tc_fence_after();
        mma_chain_kk16_b8k(tmem + C::col_x(t), sdesc_sw128(sbase + C::kR1Off, 16),
                           sdesc_sw128(s1_addr(t), 16), id_xy, 0u);
        if (has_y) {
          if (!bw.wait(bar(C::kBarS2Full + s2_slot(t)), s2_phase(t), 66)) return false;
          tc_fence_after();
          mma_chain_kk16_b8k(tmem + C::col_y(t), sdesc_sw128(sbase + C::kR2Off, 16),
                             sdesc_sw128(s2_addr(t), 16), id_xy, 0u);
          tc_commit(bar(C::kBarS2Empty + s2_slot(t)));
        }
        tc_commit(bar(C::kBarX + (t & 1)));
        return true;
      };
      if (ok) ok = issue_xy(0);
      if (ok && n > 1) ok = issue_xy(1);
      for (int t = 0; ok && t < n; ++t) {
        if (!bw.wait(bar(C::kBarZ), t & 1, 67)) break;
        uint32_t bsrc;
        if (has_y) {
          bsrc = s1_addr(t);  // dK: Q, dQ: K (already waited for by X)
        } else {
          if (!bw.wait(bar(C::kBarS2Full + s2_slot(t)), s2_phase(t), 68)) break;
          bsrc = s2_addr(t);  // dV: dO
        }
        tc_fence_after();
        // acc += Z B: A = Z (tensor memory, K = the step's 64 columns), B MN-major
        // (rows = the step's columns, 128-byte rows along the 256 head dims)
        mma_chain_ts_mn4_split32(tmem + C::kColAcc, tmem + C::col_x(t),
                                 sdesc_sw128(bsrc, C::kSBox), id_acc, t > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarS1Empty + (t & 1)));
        if (!has_y) tc_commit(bar(C::kBarS2Empty + s2_slot(t)));
        if (t == n - 1) tc_commit(bar(C::kBarAcc));
        // steps go in pairs: after the accumulations of steps t - 1 and t, the
        // products of t + 1 and t + 2, so each slot's next load overlaps an
        // accumulation and the other pair member's products
        if (t & 1) {
          if (ok && t + 1 < n) ok = issue_xy(t + 1);
          if (ok && t + 2 < n) ok = issue_xy(t + 2);
        }
      }
    }
  }
  finish();
}

}  // namespace bwd256
}  // namespace attn156
