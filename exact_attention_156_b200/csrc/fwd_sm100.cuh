// fwd_sm100.cuh - fused exact-attention forward for B200 (sm_100a).
//
// Method (FlashAttention-2 overview, lshu.cn, section 2.2): tile Q, K and V;
// for one Q tile, stream K/V tiles through on-chip memory, compute the local
// Q K^T, update a running row max m_i and row sum l_i (online softmax), and
// accumulate the weighted sum of V; the N x N score matrix never reaches HBM,
// and the next tile is fetched while the current one is computed.
//
// B200 mapping (a re-design, not the pages' Ampere/Hopper kernel):
//  * CTA = 2 query tiles of 128 rows (same batch/head) sharing one K/V stream.
//  * warp 9 (one thread) issues TMA loads: both Q tiles once, then K_j, V_j
//    into a ring of shared-memory slots (mbarrier full/empty pairs).
//  * warp 8 (one thread) issues tcgen05 MMAs: S_k = Q_k K_j^T into tensor
//    memory, and O_k += P_k V_j with P_k read from tensor memory.  The order
//    PV_0(j), S_0(j+1), PV_1(j), S_1(j+1) lets the softmax of one tile overlap
//    the tensor-core work of the other.
//  * warps 10-11 idle; after set-up the control warpgroup (8-11) gives registers
//    to the two softmax warpgroups (setmaxnreg).
//  * warps 0-3 / 4-7: softmax of tile 0 / tile 1; one thread owns one query row
//    (= one TMEM lane), so the row max and row sum need no shuffles.  Scores
//    are scaled by scale*log2(e) and exponentiated with ex2.  The running max
//    is only raised when it grows by more than 2^8 (factor 256), so O is
//    rescaled rarely; since O and l share the stale max, O/l is unchanged.
//  * epilogue: O/l in the input format and LSE = (m + log2 l) * ln 2 (natural log).
//  * Q, K, V, P and O are bf16 or f16 (template parameter E); accumulation is f32.
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D)
// O1 [256+D, 256+2D); P_k (16-bit pairs) overwrites the first 64 columns of S_k.
#pragma once

#include <cuda.h>
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"

namespace attn156 {
namespace fwd {

constexpr int BM = 128;  // query rows per tile (= TMEM lanes)
constexpr int BN = 128;  // keys per K/V tile
constexpr int NQ = 2;    // query tiles per CTA
constexpr int kThreads = 384;  // 3 warpgroups: softmax 0, softmax 1, {MMA, TMA, 2 idle}
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
// Register split after launch (168 per thread at launch: 384 x 168 = 64512):
// softmax warpgroups 2 x 128 x 216 + control warpgroup 128 x 64 = 63488.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 64;
static_assert(128 * (2 * kSoftmaxRegs + kControlRegs) <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 2^8 between rescales

template <int D>
struct Cfg {
  static constexpr int kBoxBytes = BM * 128;          // one 128-row x 64-col bf16 box
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = BM * D * 2;       // Q, K or V tile
  static constexpr int kStages = (D == 128) ? 4 : 8;  // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = NQ * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // barrier indices
  static constexpr int kBarQ = 0;
  static constexpr int kBarFull = 1;
  static constexpr int kBarEmpty = kBarFull + kStages;
  static constexpr int kBarS = kBarEmpty + kStages;
  static constexpr int kBarP = kBarS + NQ;
  static constexpr int kBarO = kBarP + NQ;
  static constexpr int kBarDone = kBarO + NQ;
  static constexpr int kNumBars = kBarDone + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base (4 B) + abort (4 B)
  static constexpr int kSmemBytes = kMiscOff + 16;
  // tensor-memory columns of S_k and O_k
  __device__ static constexpr uint32_t col_s(int k) { return uint32_t(k) * 128u; }
  __device__ static constexpr uint32_t col_o(int k) { return 256u + uint32_t(k) * D; }
};

struct Params {
  uint16_t* o;  // 16-bit elements (bf16 or f16, as the kernel's element format)
  float* lse;
  int B, H, Sq, Sk;  // packed sequences: Sq, Sk are the largest lengths
  // Packed variable-length sequences (null for the (B, S, H, D) layout):
  // sequence b is rows cu_q[b] .. cu_q[b+1]-1 of Q/O and cu_k[b] .. cu_k[b+1]-1
  // of K/V, of total_q / total_k rows; LSE is then (H, total_q).
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  int Hk;            // key/value heads (H a multiple of Hk; query head h reads h / (H / Hk))
  float scale_log2;  // scale * log2(e)
  int causal, win_left, win_right;
  int num_mblocks;   // ceil(Sq / (NQ * BM))
  int compact;       // packed batches: blockIdx.x numbers the tiles that have work (compact_tile)
  int order_chunk;   // (B, S, H, D) batches: head-batch combinations per block-order chunk
  uint32_t* err;
  uint64_t timeout_ns;
};

// Key-tile range [jlo, jhi) for query rows [r0, r1]; empty if jhi <= jlo.
__host__ __device__ __forceinline__ void tile_range(const MaskGeom& g, int r0, int r1, int& jlo, int& jhi) {
  const int klo = g.lo(r0);
  const int khi = g.hi(r1);
  if (r0 >= g.Sq || khi < klo || khi < 0) {
    jlo = 0;
    jhi = 0;
    return;
  }
  jlo = klo / BN;
  jhi = khi / BN + 1;
}

// E: element format of Q, K, V, P and O (ElemBF16 or ElemF16).
template <int D, class E, bool kVarlen>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  auto bar = [&](int idx) { return smem_u32(&bars[idx]); };

  // The swizzled operand layout needs a 1024-byte aligned base.
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(p.err, 0u, 8u);  // launch/config error
    return;
  }

  // Grid: (query-tile pair, head, batch), visited in chunked order
  // (chunked_order): pair 0 (the heaviest when causal) of every head of a chunk
  // of heads whose K/V fit in L2 together, then pair 1, ...
  int pr = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (p.order_chunk > 1) {
    const int lin = int(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    const ChunkedOrder o =
        chunked_order(lin, int(gridDim.x), int(gridDim.y * gridDim.z), p.order_chunk);
    pr = o.tile;
    h = o.hb % int(gridDim.y);
    b = o.hb / int(gridDim.y);
  }
  int mb = p.causal ? (p.num_mblocks - 1 - pr) : pr;
  const int hk = h / (p.H / p.Hk);  // the key/value head this query head reads
  if constexpr (kVarlen) {
    if (p.compact) {
      // one CTA per query-tile pair that has work, the heaviest pairs first
      int tile = 0;
      b = compact_tile(p.cu_q, p.cu_k, p.B, p.total_q, p.total_k, p.Sq, p.Sk, false, NQ * BM,
                       pr, tile);
      if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 32)
        compact_check(p.cu_q, p.cu_k, p.B, p.total_q, p.total_k, p.Sq, p.Sk, false, NQ * BM,
                      (long long)gridDim.x, p.err);
      if (b < 0) return;
      const int pairs =
          (seq_span(p.cu_q, p.cu_k, b, p.total_q, p.total_k, p.Sq, p.Sk).Lq + NQ * BM - 1) /
          (NQ * BM);
      mb = p.causal ? pairs - 1 - tile : tile;
    }
  }
  // This sequence's lengths, first rows and TMA batch coordinate.
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
  const MaskGeom g = MaskGeom::make(Lq, Lk, p.causal, p.win_left, p.win_right);

  int r0[NQ], jlo[NQ], jhi[NQ];
  bool valid[NQ];
  int ju_lo = 1 << 30, ju_hi = 0;
#pragma unroll
  for (int k = 0; k < NQ; ++k) {
    r0[k] = (mb * NQ + k) * BM;
    valid[k] = r0[k] < Lq;
    const int r1 = min(r0[k] + BM - 1, Lq - 1);
    tile_range(g, r0[k], r1, jlo[k], jhi[k]);
    if (jhi[k] > jlo[k]) {
      ju_lo = min(ju_lo, jlo[k]);
      ju_hi = max(ju_hi, jhi[k]);
    }
  }
  const bool any_work = ju_hi > ju_lo;
  // No query row of this sequence falls in this CTA (shorter sequences of a
  // packed batch): nothing to compute or write.
  if (!valid[0] && !valid[1]) return;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) {
      uint32_t count = 1;
      if (i >= C::kBarP && i < C::kBarP + NQ) count = 128;  // every softmax thread arrives
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
  auto q_addr = [&](int k) { return sbase + C::kQOff + k * C::kTileBytes; };
  auto kv_addr = [&](int s) { return sbase + C::kKVOff + s * C::kTileBytes; };
  int load_count[C::kStages];  // loads issued per slot (load thread only)
#pragma unroll
  for (int s = 0; s < C::kStages; ++s) load_count[s] = 0;

  // ------------------------------------------------------------ teardown
  // Inlined at the end of every role (each role returns after it), so that
  // each role's code is register-allocated on its own.
  auto finish = [&]() {
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
      // Drain what may still be in flight before the shared and tensor memory go away.
      const uint64_t drain_ns = 2000000000ull;
      if (warp == kLoadWarp && lane == 0) {
        for (int s = 0; s < C::kStages; ++s) {
          if (load_count[s] == 0) continue;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(bar(C::kBarFull + s), (load_count[s] - 1) & 1))
            if (globaltimer_ns() - t0 > drain_ns) break;
        }
        if (any_work) {
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
    regs_realloc<kLaunchRegs, kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax + epilogue
    const int k = warp / 4;            // query tile of this warpgroup
    const int quad = warp % 4;         // TMEM lane quadrant
    const int row = quad * 32 + lane;  // row within the tile
    const int i = r0[k] + row;         // query index
    const int n_k = jhi[k] - jlo[k];
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::col_s(k);
    const uint32_t tO = tmem + lane_off + C::col_o(k);
    const int lo_i = g.lo(i);
    const int hi_i = g.hi(i);
    const int r1 = min(r0[k] + BM - 1, Lq - 1);
    const int tile_lo_max = g.lo(r1);  // largest row lower bound in this tile
    const int tile_hi_min = g.hi(r0[k]);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;

    for (int t = 0; t < n_k; ++t) {
      const int j = jlo[k] + t;
      if (!bw.wait_warp(bar(C::kBarS + k), t & 1, 10 + k)) { ok = false; break; }
      tc_fence_after();
      float s[BN];
      {
        uint32_t r[BN];
        tmem_ld128(tS, r);
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(r[c]);
      }
      const int n0 = j * BN;
      const bool full = (n0 >= tile_lo_max) && (n0 + BN - 1 <= tile_hi_min);
      if (!full) {
        const int c_lo = lo_i - n0;
        const int c_hi = hi_i - n0;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c < c_lo || c > c_hi) s[c] = -INFINITY;
      }
      // row max: 8 independent chains of 3-input max, then a small tree
      float mx8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        float acc = s[a];
#pragma unroll
        for (int q = 1; q < 15; q += 2) acc = max3f(acc, s[8 * q + a], s[8 * (q + 1) + a]);
        mx8[a] = fmaxf(acc, s[120 + a]);
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
      uint64_t acc2[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) acc2[a] = 0ull;  // (+0.0f, +0.0f)
      // p = 2^(s * scale * log2(e) - m): the scale and subtract as f32x2 pairs,
      // the exponentials on MUFU (ex2(-inf) is exactly 0 for masked scores).
      // P goes to tensor memory as 16-bit pairs in two 64-column halves
      // (columns [0,32) and [32,64) of S_k).
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int e = half * 64 + 2 * c;
          const uint64_t x2 = f2_fma(f2_pack(s[e], s[e + 1]), scale2, negm2);
          float x0, x1;
          f2_unpack(x2, x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          acc2[c & 3] = f2_add(acc2[c & 3], f2_pack(p0, p1));
          pk[c] = E::pack2(p0, p1);
        }
        tmem_st32(tS + half * 32, pk);
      }
      float row_sum;
      {
        const uint64_t t2 = f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3]));
        float lo, hi;
        f2_unpack(t2, lo, hi);
        row_sum = lo + hi;
      }
      l_run = l_run * alpha + row_sum;
      m_run = m_new;
      // Rescale O when this warp raised any row's max (rare after the first tile).
      if (t > 0 && __any_sync(0xffffffffu, bump)) {
        if (!bw.wait_warp(bar(C::kBarO + k), (t - 1) & 1, 12 + k)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tO + c0, r);
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
          tmem_st32(tO + c0, r);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarP + k));
    }

    // Epilogue: O = O / l (input format), LSE = (m + log2 l) ln 2.
    if (valid[k] && ok) {
      const bool row_ok = i < Lq;
      const size_t orow =
          ((kVarlen ? size_t(q_row0) + i : size_t(b) * p.Sq + size_t(i)) * p.H + h) * D;
      if (n_k > 0) {
        ok = bw.wait_warp(bar(C::kBarO + k), (n_k - 1) & 1, 14 + k);
      }
      if (ok) {
        tc_fence_after();
        const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          if (n_k > 0) {
            tmem_ld32(tO + c0, r);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = E::pack2(__uint_as_float(r[2 * c]) * inv_l, __uint_as_float(r[2 * c + 1]) * inv_l);
          if (row_ok) {
            uint8_t* dst = reinterpret_cast<uint8_t*>(p.o + orow + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              st_global_v4(dst + 16 * v, w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
        if (row_ok) {
          const float lse = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
          const size_t lrow = kVarlen ? size_t(h) * p.total_q + q_row0 + i
                                     : (size_t(b) * p.H + h) * p.Sq + i;
          p.lse[lrow] = lse;
        }
      }
    }
    finish();
    return;
  }

  regs_realloc<kLaunchRegs, kControlRegs>();
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && any_work) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int nq = 0;
      for (int k = 0; k < NQ; ++k) nq += (valid[k] && jhi[k] > jlo[k]) ? 1 : 0;
      mbar_arrive_expect_tx(bar(C::kBarQ), nq * C::kTileBytes);
      for (int k = 0; k < NQ; ++k) {
        if (!(valid[k] && jhi[k] > jlo[k])) continue;
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_4d(q_addr(k) + x * C::kBoxBytes, &tmQ, bar(C::kBarQ), x * 64, h,
                      q_row0 + r0[k], bc);
      }
      const int nloads = 2 * (ju_hi - ju_lo);
      for (int L = 0; L < nloads; ++L) {
        const int s = L % C::kStages;
        const int u = L / C::kStages;
        if (u > 0 && !bw.wait(bar(C::kBarEmpty + s), (u - 1) & 1, 1)) break;
        const int j = ju_lo + L / 2;
        const void* map = (L & 1) ? static_cast<const void*>(&tmV) : static_cast<const void*>(&tmK);
        mbar_arrive_expect_tx(bar(C::kBarFull + s), C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_4d(kv_addr(s) + x * C::kBoxBytes, map, bar(C::kBarFull + s), x * 64, hk,
                      k_row0 + j * BN, bc);
        load_count[s]++;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && any_work) {
      constexpr uint32_t idesc_qk = idesc_f32acc(BM, BN, false, false, E::kFmt);
      constexpr uint32_t idesc_pv = idesc_f32acc(BM, D, false, true, E::kFmt);
      auto in_range = [&](int k, int j) { return j >= jlo[k] && j < jhi[k]; };
      auto issue_s = [&](int k, int s) {
        if constexpr (D == 128)
          mma_chain_kk8(tmem + C::col_s(k), sdesc_sw128(q_addr(k), 16), sdesc_sw128(kv_addr(s), 16),
                        idesc_qk, 0u);
        else
          mma_chain_kk4(tmem + C::col_s(k), sdesc_sw128(q_addr(k), 16), sdesc_sw128(kv_addr(s), 16),
                        idesc_qk, 0u);
        tc_commit(bar(C::kBarS + k));
      };
      auto issue_pv = [&](int k, int s, bool acc) {
        mma_chain_ts_mn8(tmem + C::col_o(k), tmem + C::col_s(k),
                         sdesc_sw128(kv_addr(s), C::kBoxBytes), idesc_pv, acc ? 1u : 0u);
        tc_commit(bar(C::kBarO + k));
      };
      auto slot_of = [&](int L) { return L % C::kStages; };
      auto phase_of = [&](int L) { return (L / C::kStages) & 1; };

      bool ok = bw.wait(bar(C::kBarQ), 0, 2);
      int L = 0;
      if (ok) ok = bw.wait(bar(C::kBarFull + slot_of(L)), phase_of(L), 3);
      if (ok) {
        tc_fence_after();
        for (int k = 0; k < NQ; ++k)
          if (in_range(k, ju_lo)) issue_s(k, slot_of(L));
        tc_commit(bar(C::kBarEmpty + slot_of(L)));
        ++L;
      }
      for (int j = ju_lo; ok && j < ju_hi; ++j) {
        const int Lv = L++;
        const bool have_next = j + 1 < ju_hi;
        const int Lk = have_next ? L++ : -1;
        if (!bw.wait(bar(C::kBarFull + slot_of(Lv)), phase_of(Lv), 4)) { ok = false; break; }
        tc_fence_after();
        bool k_ready = false;
        for (int k = 0; k < NQ; ++k) {
          if (in_range(k, j)) {
            const int t = j - jlo[k];
            if (!bw.wait(bar(C::kBarP + k), t & 1, 5)) { ok = false; break; }
            tc_fence_after();
            issue_pv(k, slot_of(Lv), t > 0);
          }
          if (have_next && in_range(k, j + 1)) {
            if (!k_ready) {
              if (!bw.wait(bar(C::kBarFull + slot_of(Lk)), phase_of(Lk), 6)) { ok = false; break; }
              tc_fence_after();
              k_ready = true;
            }
            issue_s(k, slot_of(Lk));
          }
        }
        if (!ok) break;
        tc_commit(bar(C::kBarEmpty + slot_of(Lv)));
        if (have_next) {
          if (!k_ready) {
            if (!bw.wait(bar(C::kBarFull + slot_of(Lk)), phase_of(Lk), 7)) { ok = false; break; }
            tc_fence_after();
          }
          tc_commit(bar(C::kBarEmpty + slot_of(Lk)));
        }
      }
    }
  }
  finish();
}

}  // namespace fwd
}  // namespace attn156
