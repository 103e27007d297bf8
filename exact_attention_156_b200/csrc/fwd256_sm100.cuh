// fwd256_sm100.cuh - exact-attention forward for head_dim 256 on B200 (sm_100a).
//
// Method: as the head_dim 64/128 forward (FlashAttention-2 overview, lshu.cn,
// section 2.2: tiles of Q, K, V, online softmax, the score matrix never
// written out).  The pages ask for control over particular head_dims (the
// pptc.cn page, section 6.1) and require head_dim to be a multiple of 8 (the
// yfxerp.com page, section 3.3); 256 is the largest of the usual sizes.
//
// B200 mapping.  At head_dim 256 one O accumulator takes 256 of the 512
// tensor-memory columns, so a CTA owns one 128-row query tile, and the other
// 256 columns hold two 128-key score buffers, S0 and S1:
//   S(t) = Q K_t^T     (M = 128, N = 128, K = 256: two chains of 8 steps)
//   O   += P(t) V_t    (M = 128, N = 256, K = 128: P read from tensor memory)
// The tensor core computes S(t + 1) while the softmax works on S(t), and per
// key tile the products (2048 tensor-core cycles) outlast the softmax, so the
// tensor core, not the exponentials, sets the pace.  Tensor memory: S0 [0,128),
// S1 [128,256), O [256,512); P(t) (16-bit pairs) overwrites the first 64
// columns of its S buffer.
//  * warps 0-3 / 4-7: softmax of key columns [0,64) / [64,128) of each score
//    tile, one thread = one query row (= one TMEM lane) in each group; the two
//    halves of a row agree on its running max through shared memory at a
//    named barrier that also carries every thread's wait status, so both
//    groups stop together if a wait runs out.  The running max is only raised
//    when it grows by more than 2^8, so O is rescaled rarely (O and l share
//    the stale max, O/l is unchanged); each group rescales and writes its own
//    128 columns of O;
//  * warp 8: one thread issues the tcgen05 products; warp 9: one thread loads
//    Q once (four 128 x 64 boxes) and then, per key tile, the halves
//    K[:, 0:128], K[:, 128:256], V[:, 0:128], V[:, 128:256] into a ring of four
//    32 KB slots in the order the products read them (a slot is handed back as
//    soon as the product reading it is done).  With four slots the two halves
//    of every V tile land in adjacent slots, so P V is one N = 256 product per
//    16 keys: a tensor-memory A operand costs a fixed ~107 cycles per
//    instruction up to N = 128 (measured), so two N = 128 halves would take
//    1.6x as long as one N = 256 product;
//  * epilogue: O / l in the input format and LSE = (m + log2 l) ln 2, after a
//    barrier committed once behind the last P V.
#pragma once

#include <cuda.h>
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"

namespace attn156 {
namespace fwd256 {

constexpr int D = 256;
constexpr int BM = 128;  // query rows per CTA (= TMEM lanes)
constexpr int BN = 128;  // keys per K/V tile
constexpr int kThreads = 384;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kSoftmaxThreads = 256;
constexpr int kBarRowMax = 1;  // named barrier ids (0 is __syncthreads)
constexpr int kBarRowSum = 2;
constexpr float kRescaleThreshold = 8.0f;

struct Cfg {
  static constexpr int kBox = 128 * 128;          // 128 rows x 64 columns of 16-bit (16 KB)
  static constexpr int kQBytes = 4 * kBox;        // 64 KB
  static constexpr int kSlotBytes = 2 * kBox;     // 128 rows x 128 columns (32 KB)
  static constexpr int kSlots = 4;  // even: a V tile's halves stay adjacent
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQBytes;
  static constexpr int kRedOff = kRingOff + kSlots * kSlotBytes;  // [2][2][128] f32 row maxima
  static constexpr int kBarOff = kRedOff + 2 * 2 * BM * 4;
  static constexpr int kBarQ = 0;
  static constexpr int kBarFull = 1;
  static constexpr int kBarEmpty = kBarFull + kSlots;
  static constexpr int kBarS = kBarEmpty + kSlots;  // [2]
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
  int order_chunk;  // head-batch combinations per block-order chunk (chunked_order)
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

  // causal launches the query tiles with the most keys first, in chunked
  // order over the heads (chunked_order)
  int x = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (p.order_chunk > 1) {
    const int lin = int(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    const ChunkedOrder o =
        chunked_order(lin, int(gridDim.x), int(gridDim.y * gridDim.z), p.order_chunk);
    x = o.tile;
    h = o.hb % int(gridDim.y);
    b = o.hb / int(gridDim.y);
  }
  const int mb = p.causal ? (p.num_mblocks - 1 - x) : x;
  const int hk = h / (p.H / p.Hk);
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
    for (int i = 0; i < C::kNumBars; ++i)
      mbar_init(bar(i), i == C::kBarP ? uint32_t(kSoftmaxThreads) : 1u);
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
  auto slot_addr = [&](int s) { return sbase + C::kRingOff + s * C::kSlotBytes; };
  int loads = 0;  // ring loads issued (load thread only)

  auto finish = [&]() {
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
      const uint64_t drain_ns = 2000000000ull;
      if (warp == kLoadWarp && lane == 0) {
        // the last load issued into each slot has landed
        for (int L = loads - C::kSlots > 0 ? loads - C::kSlots : 0; L < loads; ++L) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(bar(C::kBarFull + L % C::kSlots), (L / C::kSlots) & 1))
            if (globaltimer_ns() - t0 > drain_ns) break;
        }
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

  if (warp < 8) {
    // ------------------------------------------------------------ softmax + epilogue
    const int grp = warp / 4;  // key columns [64 grp, 64 grp + 64) of each tile
    const int quad = warp % 4;
    const int row = quad * 32 + lane;
    const int i = r0 + row;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::kColO + uint32_t(grp) * 128u;
    const int lo_i = g.lo(i);
    const int hi_i = g.hi(i);
    const int tile_lo_max = g.lo(r1);  // largest row lower bound in the tile
    const int tile_hi_min = g.hi(r0);  // smallest row upper bound
    const float sl2 = p.scale_log2;
    float* red = reinterpret_cast<float*>(smem + C::kRedOff);  // [buf][grp][row]
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;      // every wait of this thread so far completed
    bool alive = true;   // no row-max barrier has told the groups to stop
    for (int t = 0; t < n_kv; ++t) {
      const int n0 = (jlo + t) * BN + grp * 64;  // first key of this group's columns
      const uint32_t tS = tmem + lane_off + C::col_s(t);
      const bool s_ok = bw.wait_warp(bar(C::kBarS + (t & 1)), (t >> 1) & 1, 80);
      float s[64];
      if (s_ok) {
        tc_fence_after();
        uint32_t rr[64];
        tmem_ld64(tS + uint32_t(grp) * 64u, rr);
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(rr[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = -INFINITY;
      }
      const int t0 = (jlo + t) * BN;
      const bool full = (t0 >= tile_lo_max) && (t0 + BN - 1 <= tile_hi_min);
      if (!full) {
        const int c_lo = lo_i - n0;
        const int c_hi = hi_i - n0;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < c_lo || c > c_hi) s[c] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        float acc = s[a];
#pragma unroll
        for (int q = 1; q < 7; q += 2) acc = max3f(acc, s[8 * q + a], s[8 * (q + 1) + a]);
        mx8[a] = fmaxf(acc, s[56 + a]);
      }
      float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]),
                       fmaxf(mx8[6], mx8[7]));
      // the other half of this row: exchange the maxima (buffer t % 2, so a
      // slow partner still reading tile t - 1's value is never overwritten)
      red[((t & 1) * 2 + grp) * BM + row] = mx;
      if (!named_bar_and(kBarRowMax, kSoftmaxThreads, ok && s_ok)) {
        ok = false;
        alive = false;
        break;
      }
      mx = fmaxf(mx, red[((t & 1) * 2 + (grp ^ 1)) * BM + row]);
      const float m_cand = mx * sl2;
      const bool bump = m_cand > m_run + kRescaleThreshold;
      const float m_new = bump ? m_cand : m_run;
      const float alpha = bump ? ex2_approx(m_run - m_new) : 1.0f;
      const float m_eff = (m_new == -INFINITY) ? 0.0f : m_new;
      const uint64_t scale2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m_eff, -m_eff);
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), scale2, negm2), x0, x1);
        const uint64_t p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
        acc2[c & 3] = f2_add(acc2[c & 3], p2);
        float p0, p1;
        f2_unpack(p2, p0, p1);
        pk[c] = E::pack2(p0, p1);
      }
      // P of this group's 64 keys -> 32 columns; the other group's scores in
      // those columns were read before the row-max barrier
      tmem_st32(tS + uint32_t(grp) * 32u, pk);
      float sum;
      {
        float lo, hi2;
        f2_unpack(f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3])), lo, hi2);
        sum = lo + hi2;
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
      // S(t) was issued after P V(t - 2), so kBarO is at most one phase behind
      // here.  A wait that runs out is carried to the next row-max barrier, so
      // both groups stop at the same tile.
      if (t > 0 && __any_sync(0xffffffffu, bump)) {
        if (bw.wait_warp(bar(C::kBarO), (t - 1) & 1, 81)) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t rr[32];
            tmem_ld32(tO + c0, rr);
#pragma unroll
            for (int c = 0; c < 32; ++c) rr[c] = __float_as_uint(__uint_as_float(rr[c]) * alpha);
            tmem_st32(tO + c0, rr);
          }
        } else {
          ok = false;
        }
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarP));
    }
    // epilogue: O / l in the input format, LSE (natural log)
    bool fin_ok = ok;
    if (fin_ok && n_kv > 0) fin_ok = bw.wait_warp(bar(C::kBarOFinal), 0, 82);
    // The row sum is split between the groups: exchange it.  Every softmax
    // thread gets here unless the loop broke at a row-max barrier, which all of
    // them then left together.  Buffer n_kv % 2 was last read at tile n_kv - 2,
    // before the partner passed the last row-max barrier.
    if (alive) {
      const int buf = n_kv & 1;
      red[(buf * 2 + grp) * BM + row] = l_run;
      fin_ok = named_bar_and(kBarRowSum, kSoftmaxThreads, fin_ok);
      l_run += red[(buf * 2 + (grp ^ 1)) * BM + row];
    }
    if (alive && fin_ok && r0 < p.Sq) {
      const bool row_ok = i < p.Sq;
      const size_t orow = ((size_t(b) * p.Sq + size_t(i)) * p.H + h) * D + size_t(grp) * 128;
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.0f;
      if (n_kv > 0) tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
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
      if (row_ok && grp == 0)
        p.lse[(size_t(b) * p.H + h) * p.Sq + i] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
    }
    finish();
    return;
  }
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA: Q, then K/V halves
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(C::kBarQ), C::kQBytes);
      for (int x = 0; x < 4; ++x)
        tma_load_4d(sbase + C::kQOff + x * C::kBox, &tmQ, bar(C::kBarQ), x * 64, h, r0, b);
      // Ring order = the order the products read them: K(0), then per tile t
      // K(t + 1) (if any) and V(t), each as two 128-column halves.
      bool lok = true;
      auto load_half = [&](const CUtensorMap* map, int t, int d0) {
        const int L = loads;
        const int s = L % C::kSlots;
        const int u = L / C::kSlots;
        if (u > 0 && !bw.wait(bar(C::kBarEmpty + s), (u - 1) & 1, 83)) return false;
        const int key0 = (jlo + t) * BN;
        const uint32_t fb = bar(C::kBarFull + s);
        mbar_arrive_expect_tx(fb, C::kSlotBytes);
        tma_load_4d(slot_addr(s), map, fb, d0, hk, key0, b);
        tma_load_4d(slot_addr(s) + C::kBox, map, fb, d0 + 64, hk, key0, b);
        ++loads;
        return true;
      };
      lok = load_half(&tmK, 0, 0) && load_half(&tmK, 0, 128);
      for (int t = 0; lok && t < n_kv; ++t) {
        if (t + 1 < n_kv) lok = load_half(&tmK, t + 1, 0) && load_half(&tmK, t + 1, 128);
        if (lok) lok = load_half(&tmV, t, 0) && load_half(&tmV, t, 128);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ tcgen05 issue
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t idesc_s = idesc_f32acc(BM, BN, false, false, E::kFmt);
      constexpr uint32_t idesc_o = idesc_f32acc(BM, D, false, true, E::kFmt);
      bool ok = bw.wait(bar(C::kBarQ), 0, 84);
      auto slot_of = [&](int L) { return L % C::kSlots; };
      // ring positions of the K and V halves of key tile t (the loader's order)
      auto pos_k = [&](int t) { return t == 0 ? 0 : 4 * t - 2; };
      auto pos_v = [&](int t) { return t + 1 < n_kv ? 4 * t + 4 : 4 * t + 2; };
      auto ready = [&](int L) {
        return bw.wait(bar(C::kBarFull + slot_of(L)), (L / C::kSlots) & 1, 85);
      };
      // S(t) into buffer t % 2 from the two K halves; each slot is handed back
      // when the products reading it complete.
      auto issue_s = [&](int t) -> bool {
        const int L = pos_k(t);
        if (!ready(L)) return false;
        tc_fence_after();
        mma_chain_kk8(tmem + C::col_s(t), sdesc_sw128(sbase + C::kQOff, 16),
                      sdesc_sw128(slot_addr(slot_of(L)), 16), idesc_s, 0u);
        tc_commit(bar(C::kBarEmpty + slot_of(L)));
        if (!ready(L + 1)) return false;
        tc_fence_after();
        mma_chain_kk8(tmem + C::col_s(t), sdesc_sw128(sbase + C::kQOff + 2 * C::kBox, 16),
                      sdesc_sw128(slot_addr(slot_of(L + 1)), 16), idesc_s, 1u);
        tc_commit(bar(C::kBarS + (t & 1)));
        tc_commit(bar(C::kBarEmpty + slot_of(L + 1)));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_kv > 1) ok = issue_s(1);
      for (int t = 0; ok && t < n_kv; ++t) {
        if (!bw.wait(bar(C::kBarP), t & 1, 86)) break;
        // V(t)'s halves sit in adjacent slots (L even): one N = 256 product whose
        // four 64-column boxes lie 16 KB apart
        const int L = pos_v(t);
        if (!ready(L) || !ready(L + 1)) break;
        tc_fence_after();
        mma_chain_ts_mn8(tmem + C::kColO, tmem + C::col_s(t),
                         sdesc_sw128(slot_addr(slot_of(L)), C::kBox), idesc_o, t > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarEmpty + slot_of(L)));
        tc_commit(bar(C::kBarEmpty + slot_of(L + 1)));
        tc_commit(bar(C::kBarO));
        if (t == n_kv - 1) tc_commit(bar(C::kBarOFinal));
        if (t + 2 < n_kv) ok = issue_s(t + 2);
      }
    }
  }
  finish();
}

}  // namespace fwd256
}  // namespace attn156
