// fwd256_sm100.cuh - exact-attention forward for head_dim 256 on B200 (sm_100a).
//
// Method: as the head_dim 64/128 forward (FlashAttention-2 overview, lshu.cn,
// section 2.2: tiles of Q, K, V, online softmax, the score matrix never
// written out).  The pages ask for control over particular head_dims (the
// pptc.cn page, section 6.1) and require head_dim to be a multiple of 8 (the
// yfxerp.com page, section 3.3); 256 is the largest of the usual sizes.
//
// B200 mapping.  At head_dim 256 one O accumulator takes 256 of the 512
// tensor-memory columns, so a CTA owns one 128-row query tile (two, as at
// head_dim 128, would need all 512 columns for O alone).  To keep the tensor
// core busy while the softmax works, the key tiles are 64 keys wide and S is
// double-buffered:
//   S(t) = Q K_t^T     (M = 128, N = 64, K = 256: 16 chained steps)
//   O   += P(t) V_t    (M = 128, N = 256, K = 64: P read from tensor memory)
// so S(t+1) runs while the softmax works on S(t), and per 64-key tile the
// products take about as long as the softmax.  Tensor memory: S0 [0,64),
// S1 [64,128), O [128,384); P(t) (16-bit pairs) overwrites the first 32
// columns of its S buffer.
//  * warps 0-3: softmax, one thread = one query row (= one TMEM lane); the
//    running max is only raised when it grows by more than 2^8, so O is
//    rescaled rarely (O and l share the stale max, O/l is unchanged);
//  * warp 4: one thread issues the tcgen05 products; warp 5: one thread loads
//    Q once (four 128 x 64 boxes) and then the K tiles into a ring of 2 slots
//    of 32 KB (four 64 x 64 boxes each), warp 6 the V tiles into a ring of 3
//    (a K slot is refilled as soon as S has read it; a V slot after P V);
//  * epilogue: O / l in the input format and LSE = (m + log2 l) ln 2, after a
//    barrier committed once behind the last P V (with S double-buffered the
//    per-tile O barrier can be two phases behind when the softmax gets there).
#pragma once

#include <cuda.h>
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"
#include "ptx_d256.cuh"

namespace attn156 {
namespace fwd256 {

constexpr int D = 256;
constexpr int BM = 128;  // query rows per CTA (= TMEM lanes)
constexpr int BN = 64;   // keys per K/V tile
constexpr int kThreads = 224;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;   // Q and K
constexpr int kLoadVWarp = 6;  // V
constexpr float kRescaleThreshold = 8.0f;

struct Cfg {
  static constexpr int kQBox = BM * 128;          // 128 rows x 64 columns (16 KB)
  static constexpr int kKVBox = BN * 128;         // 64 rows x 64 columns (8 KB)
  static constexpr int kBoxes = D / 64;           // 4 boxes across head_dim
  static constexpr int kQBytes = kBoxes * kQBox;  // 64 KB
  static constexpr int kTileBytes = kBoxes * kKVBox;  // 32 KB
  static constexpr int kKSlots = 2;
  static constexpr int kVSlots = 3;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQBytes;
  static constexpr int kVOff = kKOff + kKSlots * kTileBytes;
  static constexpr int kBarOff = kVOff + kVSlots * kTileBytes;
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kKSlots;
  static constexpr int kBarVFull = kBarKEmpty + kKSlots;
  static constexpr int kBarVEmpty = kBarVFull + kVSlots;
  static constexpr int kBarS = kBarVEmpty + kVSlots;  // [2]
  static constexpr int kBarP = kBarS + 2;
  static constexpr int kBarO = kBarP + 1;
  static constexpr int kBarOFinal = kBarO + 1;
  static constexpr int kBarDone = kBarOFinal + 1;
  static constexpr int kNumBars = kBarDone + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  __device__ static constexpr uint32_t col_s(int t) { return uint32_t(t & 1) * BN; }
  static constexpr uint32_t kColO = 2 * BN;
  static_assert(kSmemBytes <= 232448, "shared memory exceeds the 227 KB per block of sm_100");
};

struct Params {
  uint16_t* o;
  float* lse;
  int B, H, Sq, Sk, Hk;
  float scale_log2;
  int causal, win_left, win_right;
  int num_mblocks;  // ceil(Sq / 128)
  uint32_t* err;
  uint64_t timeout_ns;
};

template <class E>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const Params p) {
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

  // causal launches the query tiles with the most keys first
  const int mb = p.causal ? (p.num_mblocks - 1 - int(blockIdx.x)) : int(blockIdx.x);
  const int h = blockIdx.y;
  const int hk = h / (p.H / p.Hk);
  const int b = blockIdx.z;
  const MaskGeom g = MaskGeom::make(p.Sq, p.Sk, p.causal, p.win_left, p.win_right);
  const int r0 = mb * BM;
  const int r1 = min(r0 + BM - 1, p.Sq - 1);
  // key tiles [jlo, jhi) that rows r0..r1 can see
  int jlo = 0, jhi = 0;
  {
    const int klo = g.lo(r0);
    const int khi = g.hi(r1);
    if (khi >= klo && khi >= 0) {
      jlo = klo / BN;
      jhi = khi / BN + 1;
    }
  }
  const int n_kv = jhi - jlo;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) mbar_init(bar(i), i == C::kBarP ? 128u : 1u);
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
  auto k_addr = [&](int s) { return sbase + C::kKOff + s * C::kTileBytes; };
  auto v_addr = [&](int s) { return sbase + C::kVOff + s * C::kTileBytes; };
  int k_loads = 0, v_loads = 0;  // tiles issued by this loader (loader threads only)

  auto finish = [&]() {
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
      const uint64_t drain_ns = 2000000000ull;
      // the last tile each loader issued into each slot has landed
      auto settle_ring = [&](int full0, int slots, int issued) {
        for (int t = issued - slots > 0 ? issued - slots : 0; t < issued; ++t) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(bar(full0 + t % slots), (t / slots) & 1))
            if (globaltimer_ns() - t0 > drain_ns) break;
        }
      };
      if (warp == kLoadVWarp && lane == 0) settle_ring(C::kBarVFull, C::kVSlots, v_loads);
      if (warp == kLoadWarp && lane == 0) {
        settle_ring(C::kBarKFull, C::kKSlots, k_loads);
        if (n_kv > 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(bar(C::kBarQ), 0))
            if (globaltimer_ns() - t0 > drain_ns) break;
        }
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

  if (warp < 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int row = warp * 32 + lane;
    const int i = r0 + row;
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::kColO;
    const int lo_i = g.lo(i);
    const int hi_i = g.hi(i);
    const int tile_lo_max = g.lo(r1);  // largest row lower bound in the tile
    const int tile_hi_min = g.hi(r0);  // smallest row upper bound
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int t = 0; t < n_kv; ++t) {
      const int n0 = (jlo + t) * BN;
      const uint32_t tS = tmem + lane_off + C::col_s(t);
      if (!bw.wait_warp(bar(C::kBarS + (t & 1)), (t >> 1) & 1, 80)) { ok = false; break; }
      tc_fence_after();
      float s[BN];
      {
        uint32_t rr[BN];
        tmem_ld64(tS, rr);
        const bool full = (n0 >= tile_lo_max) && (n0 + BN - 1 <= tile_hi_min);
        const int c_lo = lo_i - n0;
        const int c_hi = hi_i - n0;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          s[c] = (full || (c >= c_lo && c <= c_hi)) ? __uint_as_float(rr[c]) : -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        float acc = s[a];
#pragma unroll
        for (int q = 1; q < 7; q += 2) acc = max3f(acc, s[8 * q + a], s[8 * (q + 1) + a]);
        mx8[a] = fmaxf(acc, s[56 + a]);
      }
      const float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]),
                             fmaxf(mx8[6], mx8[7]));
      const float m_cand = mx * sl2;
      const bool bump = m_cand > m_run + kRescaleThreshold;
      const float m_new = bump ? m_cand : m_run;
      const float alpha = bump ? ex2_approx(m_run - m_new) : 1.0f;
      const float m_eff = (m_new == -INFINITY) ? 0.0f : m_new;
      const uint64_t scale2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m_eff, -m_eff);
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN / 2; ++c) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), scale2, negm2), x0, x1);
        const uint64_t p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
        acc2[c & 3] = f2_add(acc2[c & 3], p2);
        float p0, p1;
        f2_unpack(p2, p0, p1);
        pk[c] = E::pack2(p0, p1);
      }
      tmem_st32(tS, pk);
      float sum;
      {
        float lo, hi2;
        f2_unpack(f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3])), lo, hi2);
        sum = lo + hi2;
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
      // S(t) was issued after P V(t - 2), so kBarO is at most one phase behind here
      if (t > 0 && __any_sync(0xffffffffu, bump)) {
        if (!bw.wait_warp(bar(C::kBarO), (t - 1) & 1, 81)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t rr[32];
          tmem_ld32(tO + c0, rr);
#pragma unroll
          for (int c = 0; c < 32; ++c) rr[c] = __float_as_uint(__uint_as_float(rr[c]) * alpha);
          tmem_st32(tO + c0, rr);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarP));
    }
    // epilogue: O / l in the input format, LSE (natural log)
    if (ok && n_kv > 0) ok = bw.wait_warp(bar(C::kBarOFinal), 0, 82);
    if (ok && r0 < p.Sq) {
      const bool row_ok = i < p.Sq;
      const size_t orow = ((size_t(b) * p.Sq + size_t(i)) * p.H + h) * D;
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.0f;
      if (n_kv > 0) tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t rr[32];
        if (n_kv > 0) {
          tmem_ld32(tO + c0, rr);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) rr[c] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = E::pack2(__uint_as_float(rr[2 * c]) * inv_l, __uint_as_float(rr[2 * c + 1]) * inv_l);
        if (row_ok) {
          uint8_t* dst = reinterpret_cast<uint8_t*>(p.o + orow + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            st_global_v4(dst + 16 * v, w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      if (row_ok)
        p.lse[(size_t(b) * p.H + h) * p.Sq + i] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
    }
    finish();
    return;
  }
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA: Q, then K_t
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_arrive_expect_tx(bar(C::kBarQ), C::kQBytes);
      for (int x = 0; x < C::kBoxes; ++x)
        tma_load_4d(sbase + C::kQOff + x * C::kQBox, &tmQ, bar(C::kBarQ), x * 64, h, r0, b);
      for (int t = 0; t < n_kv; ++t) {
        const int s = t % C::kKSlots;
        const int u = t / C::kKSlots;
        if (u > 0 && !bw.wait(bar(C::kBarKEmpty + s), (u - 1) & 1, 83)) break;
        const uint32_t fb = bar(C::kBarKFull + s);
        mbar_arrive_expect_tx(fb, C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_4d(k_addr(s) + x * C::kKVBox, &tmK, fb, x * 64, hk, (jlo + t) * BN, b);
        ++k_loads;
      }
    }
  } else if (warp == kLoadVWarp) {
    // ------------------------------------------------------------ TMA: V_t
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmV);
      for (int t = 0; t < n_kv; ++t) {
        const int s = t % C::kVSlots;
        const int u = t / C::kVSlots;
        if (u > 0 && !bw.wait(bar(C::kBarVEmpty + s), (u - 1) & 1, 88)) break;
        const uint32_t fb = bar(C::kBarVFull + s);
        mbar_arrive_expect_tx(fb, C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_4d(v_addr(s) + x * C::kKVBox, &tmV, fb, x * 64, hk, (jlo + t) * BN, b);
        ++v_loads;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ tcgen05 issue
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t idesc_s = idesc_f32acc(BM, BN, false, false, E::kFmt);
      constexpr uint32_t idesc_o = idesc_f32acc(BM, D, false, true, E::kFmt);
      const uint64_t q_desc = sdesc_sw128(sbase + C::kQOff, 16);
      bool ok = bw.wait(bar(C::kBarQ), 0, 84);
      // S(t) into buffer t % 2 once K_t has landed (its slot is handed back when
      // S(t) completes); S(t + 2) reuses the buffer once P V(t), which reads
      // P(t) from it, has been issued.
      auto issue_s = [&](int t) -> bool {
        const int s = t % C::kKSlots;
        if (!bw.wait(bar(C::kBarKFull + s), (t / C::kKSlots) & 1, 85)) return false;
        tc_fence_after();
        mma_chain_kk16_b8k(tmem + C::col_s(t), q_desc, sdesc_sw128(k_addr(s), 16), idesc_s, 0u);
        tc_commit(bar(C::kBarS + (t & 1)));
        tc_commit(bar(C::kBarKEmpty + s));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_kv > 1) ok = issue_s(1);
      for (int t = 0; ok && t < n_kv; ++t) {
        const int s = t % C::kVSlots;
        if (!bw.wait(bar(C::kBarP), t & 1, 86)) break;
        if (!bw.wait(bar(C::kBarVFull + s), (t / C::kVSlots) & 1, 87)) break;
        tc_fence_after();
        mma_chain_ts_mn4(tmem + C::kColO, tmem + C::col_s(t), sdesc_sw128(v_addr(s), C::kKVBox),
                         idesc_o, t > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarO));
        tc_commit(bar(C::kBarVEmpty + s));
        if (t == n_kv - 1) tc_commit(bar(C::kBarOFinal));
        if (t + 2 < n_kv) ok = issue_s(t + 2);
      }
    }
  }
  finish();
}

}  // namespace fwd256
}  // namespace attn156
