// bwd_sm100.cuh - recompute-based exact-attention backward for B200 (sm_100a).
//
// Method: the backward rebuilds the attention probabilities from Q, K and the
// forward's per-row log-sum-exp instead of storing them (flash-attn install
// guide, yfxerp.com, section 1: "the backward recomputes the attention
// scores"; FlashAttention-2 overview, lshu.cn, section 2.1, second anti-pattern:
// the standard backward re-reads Q, K, V several times).  The gradient is the
// analytic one of O = softmax(scale Q K^T) V:
//   P = exp(scale S - LSE), dV = P^T dO, dP = dO V^T, Delta_i = rowsum(dO*O),
//   dS = P * (dP - Delta), dK = scale dS^T Q, dQ = scale dS K.
//
// Kernels:
//  1. bwd_pre: Delta_i (fp32), LSE in base 2 (padded rows: +inf so P = 0),
//     and zeroes the fp32 dQ accumulator.  Memory bound.
//  2. bwd_main: one CTA per (128-key tile, head, batch); K_j and V_j stay in
//     shared memory while the CTA streams the query tiles that can see them.
//     Transposed products put the key index on tensor-memory lanes:
//       S^T = K Q^T  and  dP^T = V dO^T   (M = keys, N = queries, K = D)
//       dV += P^T dO  (A = P^T from tensor memory)
//       dK += dS^T Q  (A = dS^T from shared memory, K-major)
//       dQ_tile = dS K (A = the same dS^T buffer read MN-major) -> fp32 atomics
//     warps 0-3: P and dS (one thread = one key row); warps 4-7: drain dQ
//     from tensor memory into the fp32 accumulator with vector reductions;
//     warp 8: MMA issue; warp 9: TMA / bulk loads.
//  3. bwd_dq_finalize: dQ = bf16(scale * accumulator).
// Tensor memory (512 columns): dK [0,D) dV [D,2D) S^T/P^T [2D,2D+128)
// dP^T / dQ [2D+128, 2D+256).
#pragma once

#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "ptx.cuh"

namespace attn156 {
namespace bwd {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // key rows per CTA
constexpr int kThreads = 384;  // compute WG, dQ-drain WG, control WG {MMA, TMA, 2 idle}
constexpr int kDrainWarp0 = 4;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kStages = 2;
// Register split after launch (168 per thread at launch: 384 x 168 = 64512):
// compute 128 x 240 + drain 128 x 144 + control 128 x 120 = 64512.
constexpr int kLaunchRegs = 168;
constexpr int kComputeRegs = 240;
constexpr int kDrainRegs = 144;
constexpr int kControlRegs = 120;
static_assert(128 * (kComputeRegs + kDrainRegs + kControlRegs) <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

template <int D>
struct Cfg {
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kTileBytes;
  // stage s = [Q_s | dO_s]; once the MMAs of a stage are done, the whole stage
  // (128 x D fp32 bytes) holds the dQ tile on its way to the TMA reduce-add.
  static constexpr int kStageOff = kVOff + kTileBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kDSOff = kStageOff + kStages * kStageBytes;  // dS^T, 128 x 128 bf16
  static constexpr int kLseOff = kDSOff + BN * BM * 2;             // [kStages][BM] fp32
  static constexpr int kDeltaOff = kLseOff + kStages * BM * 4;     // [kStages][BM] fp32
  static constexpr int kBarOff = kDeltaOff + kStages * BM * 4;
  static constexpr int kBarKV = 0;
  static constexpr int kBarFull = 1;
  static constexpr int kBarEmpty = kBarFull + kStages;
  static constexpr int kBarS = kBarEmpty + kStages;
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
  static_assert(kStageBytes == BM * D * 4, "a stage must hold one fp32 dQ tile");
};

struct Params {
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* lse2;   // [B*H][Sq_pad] LSE * log2(e); +inf for padding rows
  const float* delta;  // [B*H][Sq_pad]
  float* dq_acc;       // [B*H][Sq_pad][D]
  int B, H, Sq, Sk, Sq_pad;
  float scale;
  float scale_log2;
  int causal, win_left, win_right;
  uint32_t* err;
  uint64_t timeout_ns;
};

// ---------------------------------------------------------------------------
// 1. preprocess: one warp per (b, h, row of the padded query axis)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ delta,
    float* __restrict__ dq_acc, int B, int H, int Sq, int Sq_pad) {
  const long long gw = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const long long rows = (long long)B * H * Sq_pad;
  if (gw >= rows) return;
  const int i = int(gw % Sq_pad);
  const long long bh = gw / Sq_pad;
  const int h = int(bh % H);
  const int b = int(bh / H);
  float dot = 0.f;
  if (i < Sq) {
    const size_t base = ((size_t(b) * Sq + i) * H + h) * D;
    constexpr int kPer = D / 32;  // bf16 elements per lane (2 or 4)
    if constexpr (kPer == 4) {
      const uint2 ov = *reinterpret_cast<const uint2*>(o + base + lane * 4);
      const uint2 dv = *reinterpret_cast<const uint2*>(dout + base + lane * 4);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float2 a = __bfloat1622float2(o2[t]);
        const float2 c = __bfloat1622float2(d2[t]);
        dot = fmaf(a.x, c.x, dot);
        dot = fmaf(a.y, c.y, dot);
      }
    } else {
      const __nv_bfloat162 ov = *reinterpret_cast<const __nv_bfloat162*>(o + base + lane * 2);
      const __nv_bfloat162 dv = *reinterpret_cast<const __nv_bfloat162*>(dout + base + lane * 2);
      const float2 a = __bfloat1622float2(ov);
      const float2 c = __bfloat1622float2(dv);
      dot = fmaf(a.x, c.x, dot);
      dot = fmaf(a.y, c.y, dot);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  if (lane == 0) {
    const size_t r = size_t(bh) * Sq_pad + i;
    float l2 = INFINITY;  // padding rows and rows that see no key: P = 0
    if (i < Sq) {
      const float l = lse[size_t(bh) * Sq + i];
      if (l != -INFINITY) l2 = l * 1.4426950408889634f;
    }
    lse2[r] = l2;
    delta[r] = dot;
  }
  float4* acc = reinterpret_cast<float4*>(dq_acc + (size_t(bh) * Sq_pad + i) * D);
  for (int c = lane; c < D / 4; c += 32) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------
// 3. dQ finalize: dq[b, i, h, :] = bf16(scale * acc[b, h, i, :]); 8 elements per thread
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                          __nv_bfloat16* __restrict__ dq, int B,
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
  w.x = pack_bf16x2(a.x * scale, a.y * scale);
  w.y = pack_bf16x2(a.z * scale, a.w * scale);
  w.z = pack_bf16x2(c.x * scale, c.y * scale);
  w.w = pack_bf16x2(c.z * scale, c.w * scale);
  *reinterpret_cast<uint4*>(dq + ((size_t(b) * Sq + i) * H + h) * D + v * 8) = w;
}

// ---------------------------------------------------------------------------
// 2. main backward kernel
// ---------------------------------------------------------------------------
// Query-tile range [qlo, qhi) that can see keys [n0, n1]; empty if qhi <= qlo.
__device__ __forceinline__ void qtile_range(const MaskGeom& g, int n0, int n1, int& qlo, int& qhi) {
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

template <int D>
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

  const int kt = blockIdx.x;  // key tile; low indices see the most query tiles when causal
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * p.H + h;
  const MaskGeom g = MaskGeom::make(p.Sq, p.Sk, p.causal, p.win_left, p.win_right);
  const int n0 = kt * BN;
  const int n1 = min(n0 + BN - 1, p.Sk - 1);
  int qlo, qhi;
  qtile_range(g, n0, n1, qlo, qhi);
  const int nq = qhi - qlo;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) {
      uint32_t count = 1;
      if (i == C::kBarP || i == C::kBarDS || i == C::kBarDQEmpty) count = 128;
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
  auto stage_addr = [&](int s) { return sbase + C::kStageOff + s * C::kStageBytes; };
  auto q_addr = [&](int s) { return stage_addr(s); };
  auto do_addr = [&](int s) { return stage_addr(s) + C::kTileBytes; };
  const uint32_t k_addr = sbase + C::kKOff;
  const uint32_t v_addr = sbase + C::kVOff;
  const uint32_t ds_addr = sbase + C::kDSOff;
  int load_count[kStages] = {0, 0};
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
      if (warp == kLoadWarp && lane == 0 && nq > 0) {
        for (int s = 0; s < kStages; ++s) {
          if (load_count[s] == 0) continue;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(bar(C::kBarFull + s), (load_count[s] - 1) & 1))
            if (globaltimer_ns() - t0 > drain_ns) break;
        }
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bar(C::kBarKV), 0))
          if (globaltimer_ns() - t0 > drain_ns) break;
      }
      if (warp == kMmaWarp && lane == 0) {
        tc_commit(bar(C::kBarDone));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bar(C::kBarDone), 0))
          if (globaltimer_ns() - t0 > drain_ns) break;
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
    const int quad = warp % 4;
    const int r = quad * 32 + lane;  // key row within the tile
    const int kk_idx = n0 + r;       // key index
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS;
    const uint32_t tDP = tmem + lane_off + C::kColDP;
    const float sl2 = p.scale_log2;
    const int qmin_k = g.qmin(kk_idx);
    const int qmax_k = min(g.qmax(kk_idx), p.Sq - 1);
    const bool key_ok = kk_idx < p.Sk;
    // rows of the dS^T buffer: 128 bytes per 64 columns, 16-byte chunks swizzled by row % 8
    const uint32_t ds_row = ds_addr + uint32_t(r) * 128;
    const uint32_t sw = uint32_t(r & 7);
    bool ok = true;
    for (int t = 0; t < nq; ++t) {
      const int s = t % kStages;
      const int i0 = (qlo + t) * BM;
      const float4* lse2 = reinterpret_cast<const float4*>(smem + C::kLseOff + s * BM * 4);
      const float4* dlt = reinterpret_cast<const float4*>(smem + C::kDeltaOff + s * BM * 4);
      if (!bw.wait_warp(bar(C::kBarS), t & 1, 27)) { ok = false; break; }
      tc_fence_after();
      float pr[BM];
      {
        uint32_t rr[BM];
        tmem_ld128(tS, rr);
#pragma unroll
        for (int c = 0; c < BM; c += 4) {
          const float4 l4 = lse2[c / 4];
          pr[c + 0] = ex2_approx(fmaf(__uint_as_float(rr[c + 0]), sl2, -l4.x));
          pr[c + 1] = ex2_approx(fmaf(__uint_as_float(rr[c + 1]), sl2, -l4.y));
          pr[c + 2] = ex2_approx(fmaf(__uint_as_float(rr[c + 2]), sl2, -l4.z));
          pr[c + 3] = ex2_approx(fmaf(__uint_as_float(rr[c + 3]), sl2, -l4.w));
        }
      }
      const bool full = key_ok && n0 + BN - 1 <= p.Sk - 1 && i0 + BM - 1 <= p.Sq - 1 &&
                        i0 >= g.qmin(n0 + BN - 1) && i0 + BM - 1 <= g.qmax(n0);
      if (!full) {
        const int c_lo = key_ok ? qmin_k - i0 : (1 << 30);
        const int c_hi = qmax_k - i0;
#pragma unroll
        for (int c = 0; c < BM; ++c)
          if (c < c_lo || c > c_hi) pr[c] = 0.f;
      }
      {
        uint32_t w[BM / 2];
#pragma unroll
        for (int c = 0; c < BM / 2; ++c) w[c] = pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
        tmem_st64(tS, w);
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarP));

      if (!bw.wait_warp(bar(C::kBarDP), t & 1, 28)) { ok = false; break; }
      if (t > 0 && !bw.wait_warp(bar(C::kBarDSEmpty), (t - 1) & 1, 29)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < BM; c0 += 64) {
        uint32_t rr[64];
        tmem_ld64(tDP + c0, rr);
#pragma unroll
        for (int cc = 0; cc < 64; cc += 8) {
          const float4 d0 = dlt[(c0 + cc) / 4];
          const float4 d1 = dlt[(c0 + cc) / 4 + 1];
          const float dl[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float a0 = pr[c0 + cc + e] * (__uint_as_float(rr[cc + e]) - dl[e]);
            const float a1 = pr[c0 + cc + e + 1] * (__uint_as_float(rr[cc + e + 1]) - dl[e + 1]);
            w[e / 2] = pack_bf16x2(a0, a1);
          }
          const int col = c0 + cc;  // first of 8 columns in this 16-byte chunk
          const uint32_t box = uint32_t(col / 64);
          const uint32_t chunk = uint32_t((col % 64) / 8);
          st_shared_v4(ds_row + box * C::kBoxBytes + ((chunk ^ sw) << 4), w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(C::kBarDS));
    }
    // epilogue: dK = scale * acc, dV = acc (bf16)
    if (ok && nq > 0) ok = bw.wait_warp(bar(C::kBarDQFull), (nq - 1) & 1, 30);
    if (ok) {
      tc_fence_after();
      const size_t orow = ((size_t(b) * p.Sk + size_t(kk_idx)) * p.H + h) * D;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? C::kColDK : C::kColDV;
        const float mul = which == 0 ? p.scale : 1.0f;
        __nv_bfloat16* outp = which == 0 ? p.dk : p.dv;
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
            w[c] = pack_bf16x2(__uint_as_float(rr[2 * c]) * mul, __uint_as_float(rr[2 * c + 1]) * mul);
          if (key_ok) {
            uint8_t* dst = reinterpret_cast<uint8_t*>(outp + orow + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              st_global_v4(dst + 16 * v, w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
      }
    }
    finish();
    return;
  }
  if (warp < kMmaWarp) {
    regs_realloc<kLaunchRegs, kDrainRegs>();
    // ------------------------------------------------------------ dQ drain
    // TMEM -> registers -> the finished Q/dO stage (as four 128x32 fp32 boxes,
    // 128-byte swizzle) -> one TMA reduce-add per box into the fp32 accumulator.
    const int quad = warp % 4;
    const int r = quad * 32 + lane;  // query row within the tile
    const uint32_t tDQ = tmem + (uint32_t(quad * 32) << 16) + C::kColDP;
    const uint32_t sw = uint32_t(r & 7);
    const bool leader = (warp == kDrainWarp0 && lane == 0);
    if (leader) tma_prefetch_desc(&tmDQ);
    for (int t = 0; t < nq; ++t) {
      const int s = t % kStages;
      // all four drain warps continue or stop together (they meet at named barriers)
      if (!named_bar_and(1, 128, bw.wait(bar(C::kBarDQFull), t & 1, 31))) break;
      tc_fence_after();
      const uint32_t stg = stage_addr(s) + uint32_t(r) * 128;
      auto stage_cols = [&](const uint32_t(&rr)[64], int c_base) {
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const int col = c_base + c;
          const uint32_t box = uint32_t(col / 32);
          const uint32_t chunk = uint32_t((col % 32) / 4);
          st_shared_v4(stg + box * (128 * 128) + ((chunk ^ sw) << 4), rr[c], rr[c + 1],
                       rr[c + 2], rr[c + 3]);
        }
      };
      uint32_t rr[64];
      tmem_ld64(tDQ, rr);
      if constexpr (D == 128) {
        stage_cols(rr, 0);
        tmem_ld64(tDQ + 64, rr);
      }
      // tensor memory is free again: the MMA warp may start dP of the next tile
      tc_fence_before();
      mbar_arrive(bar(C::kBarDQEmpty));
      stage_cols(rr, D - 64);
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (leader) {
        const int row0 = bh * p.Sq_pad + (qlo + t) * BM;
#pragma unroll
        for (int box = 0; box < D / 32; ++box)
          tma_reduce_add_2d(&tmDQ, stage_addr(s) + box * (128 * 128), box * 32, row0);
        bulk_commit();
        bulk_wait_read_all();  // the stage may be refilled once the reduce has read it
        mbar_arrive(bar(C::kBarEmpty + s));
        drain_issued = true;
      }
    }
    if (leader && drain_issued) bulk_wait_all();
    finish();
    return;
  }
  regs_realloc<kLaunchRegs, kControlRegs>();
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ loads
    if (lane == 0 && nq > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar(C::kBarKV), 2 * C::kTileBytes);
      for (int x = 0; x < C::kBoxes; ++x) {
        tma_load_4d(k_addr + x * C::kBoxBytes, &tmK, bar(C::kBarKV), x * 64, h, n0, b);
        tma_load_4d(v_addr + x * C::kBoxBytes, &tmV, bar(C::kBarKV), x * 64, h, n0, b);
      }
      for (int t = 0; t < nq; ++t) {
        const int s = t % kStages;
        const int u = t / kStages;
        if (u > 0 && !bw.wait(bar(C::kBarEmpty + s), (u - 1) & 1, 20)) break;
        const int i0 = (qlo + t) * BM;
        const uint32_t fb = bar(C::kBarFull + s);
        mbar_arrive_expect_tx(fb, 2 * C::kTileBytes + 2 * BM * 4);
        for (int x = 0; x < C::kBoxes; ++x) {
          tma_load_4d(q_addr(s) + x * C::kBoxBytes, &tmQ, fb, x * 64, h, i0, b);
          tma_load_4d(do_addr(s) + x * C::kBoxBytes, &tmDO, fb, x * 64, h, i0, b);
        }
        const size_t roff = size_t(bh) * p.Sq_pad + i0;
        bulk_load(sbase + C::kLseOff + s * BM * 4, p.lse2 + roff, BM * 4, fb);
        bulk_load(sbase + C::kDeltaOff + s * BM * 4, p.delta + roff, BM * 4, fb);
        load_count[s]++;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && nq > 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(BN, BM, false, false);   // S^T, dP^T
      constexpr uint32_t id_dv = idesc_bf16_f32(BN, D, false, true);    // dV, dK
      constexpr uint32_t id_dq = idesc_bf16_f32(BM, D, true, true);     // dQ
      auto issue_kmajor = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
        if constexpr (D == 128)
          mma_chain_kk8(tmem + d_col, sdesc_sw128(a_base, 16), sdesc_sw128(b_base, 16), id_s, 0u);
        else
          mma_chain_kk4(tmem + d_col, sdesc_sw128(a_base, 16), sdesc_sw128(b_base, 16), id_s, 0u);
      };
      bool ok = bw.wait(bar(C::kBarKV), 0, 21);
      if (ok) ok = bw.wait(bar(C::kBarFull + 0), 0, 22);
      if (ok) {
        tc_fence_after();
        issue_kmajor(C::kColS, k_addr, q_addr(0));
        tc_commit(bar(C::kBarS));
        issue_kmajor(C::kColDP, v_addr, do_addr(0));
        tc_commit(bar(C::kBarDP));
      }
      for (int t = 0; ok && t < nq; ++t) {
        const int s = t % kStages;
        // dV += P^T dO   (A = P^T in tensor memory, K = query index)
        if (!bw.wait(bar(C::kBarP), t & 1, 23)) { ok = false; break; }
        tc_fence_after();
        mma_chain_ts_mn8(tmem + C::kColDV, tmem + C::kColS,
                         sdesc_sw128(do_addr(s), C::kBoxBytes), id_dv, t > 0 ? 1u : 0u);
        // dK += dS^T Q   (A = dS^T in shared memory, K-major over the query index)
        if (!bw.wait(bar(C::kBarDS), t & 1, 24)) { ok = false; break; }
        tc_fence_after();
        mma_chain_kmn8(tmem + C::kColDK, sdesc_sw128(ds_addr, 16),
                       sdesc_sw128(q_addr(s), C::kBoxBytes), id_dv, t > 0 ? 1u : 0u);
        // next S^T while this tile's dQ is formed and drained
        const bool more = t + 1 < nq;
        const int s1 = (t + 1) % kStages;
        if (more) {
          if (!bw.wait(bar(C::kBarFull + s1), ((t + 1) / kStages) & 1, 25)) { ok = false; break; }
          tc_fence_after();
          issue_kmajor(C::kColS, k_addr, q_addr(s1));
          tc_commit(bar(C::kBarS));
        }
        // dQ_tile = dS K  (A = dS read MN-major: rows of the buffer are keys = K index)
        mma_chain_mnmn8(tmem + C::kColDP, sdesc_sw128(ds_addr, C::kBoxBytes),
                        sdesc_sw128(k_addr, C::kBoxBytes), id_dq, 0u);
        tc_commit(bar(C::kBarDQFull));
        tc_commit(bar(C::kBarDSEmpty));
        if (more) {
          if (!bw.wait(bar(C::kBarDQEmpty), t & 1, 26)) { ok = false; break; }
          tc_fence_after();
          issue_kmajor(C::kColDP, v_addr, do_addr(s1));
          tc_commit(bar(C::kBarDP));
        }
      }
    }
  }
  finish();
}

}  // namespace bwd
}  // namespace attn156
