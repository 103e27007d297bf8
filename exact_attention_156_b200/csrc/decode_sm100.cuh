// decode_sm100.cuh - exact attention of a few new query rows per sequence
// against a K/V cache (decode), for B200 (sm_100a).
//
// Method: the pages name flash_attn_with_kvcache as the KV-cache entry point
// (FlashAttention-2 overview, lshu.cn, section 3.3) without further detail;
// the arithmetic is the same exact attention (section 2.1 three steps, section
// 2.2 tiling with a running max and sum), over the first cache_seqlens[b] rows
// of the cache.
//
// B200 mapping: decode reads every cached K/V byte once and does little math
// per byte (memory bound), so the aim is to keep HBM busy:
//  * CTA = (key split, K/V head, batch).  All query rows that read this K/V
//    head (H / Hk heads x Sq new positions, at most 128) form one 128-row tile,
//    loaded with one TMA box, so the cache is streamed from HBM once per K/V
//    head rather than once per query head.
//  * the split's 128-key K tiles and V tiles stream through two shared-memory
//    rings of their own (TMA, mbarrier full/empty pairs, one loader warp
//    each): a K slot is handed back as soon as S = Q K^T has read it and a V
//    slot once O += P V has, so the next tiles are in flight while the
//    softmax works (one ring of K+V pairs would hold each K tile through the
//    softmax and P V); tcgen05 computes both products in tensor memory (the
//    tensor core is mostly idle: rows that are not query rows are padding);
//  * warps 0-3: online softmax (one thread = one row), warp 4: MMA issue,
//    warp 5: K loads (and Q), warp 6: V loads; S is double-buffered in tensor
//    memory, so the products of one tile (S of the next, P V of the previous)
//    run under the softmax of the other;
//  * each CTA writes its rows' normalised partial O (fp32) and log-sum-exp for
//    its split; attn_decode_combine_kernel merges the splits:
//    LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.
// Cache rows past a sequence's length are real memory (possibly stale or
// non-finite): their scores are masked, and their V rows are zeroed in shared
// memory before P V reads them (0 * NaN would otherwise poison O).
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O [256,256+D); P
// (16-bit pairs) overwrites the first 64 columns of its S.
#pragma once

#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "ptx.cuh"

namespace attn156 {
namespace dec {

constexpr int BM = 128;  // rows of the query tile (= TMEM lanes)
constexpr int BN = 128;  // keys per K/V tile
constexpr int kThreads = 224;
constexpr int kMmaWarp = 4;
constexpr int kLoadKWarp = 5;
constexpr int kLoadVWarp = 6;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct Cfg {
  static constexpr int kBoxBytes = BN * 128;  // 128 rows x 64 columns
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = BN * D * 2;
  static constexpr int kSlots = (D == 128) ? 3 : 6;  // slots of each of the K and V rings
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kTileBytes;                      // K ring
  static constexpr int kVOff = kKOff + kSlots * kTileBytes;     // V ring
  static constexpr int kBarOff = kVOff + kSlots * kTileBytes;
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kSlots;
  static constexpr int kBarVFull = kBarKEmpty + kSlots;
  static constexpr int kBarVEmpty = kBarVFull + kSlots;
  static constexpr int kBarS = kBarVEmpty + kSlots;  // [2]: per S buffer
  static constexpr int kBarP = kBarS + 2;
  static constexpr int kBarO = kBarP + 1;
  // committed once, after the last P V: the epilogue's wait.  (A parity wait on
  // kBarO could alias: with S double-buffered the softmax only knows that
  // P V(n - 3) is done when it gets there, so kBarO may be two phases behind.)
  static constexpr int kBarOFinal = kBarO + 1;
  static constexpr int kBarDone = kBarOFinal + 1;
  static constexpr int kNumBars = kBarDone + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  __device__ static constexpr uint32_t col_s(int t) { return uint32_t(t & 1) * 128u; }
  static constexpr uint32_t kColO = 256;
  static_assert(kSmemBytes <= 232448, "shared memory exceeds the 227 KB per block of sm_100");
};

struct Params {
  const int* seqlens;    // [B] valid cache rows per sequence (device)
  float* opart;          // [B][H][Sq][nsplit][D] normalised partial O
  float* lsepart;        // [B][H][Sq][nsplit] partial log-sum-exp (natural log)
  int B, Sq, Smax, H, Hk;
  int group;             // H / Hk query heads per K/V head
  int nsplit;            // key splits
  int tiles_per_split;   // 128-key tiles per split
  float scale_log2;      // scale * log2(e)
  int causal;
  uint32_t* err;
  uint64_t timeout_ns;
};

// E: element format of Q, K, V and P (ElemBF16 or ElemF16).
template <int D, class E>
__global__ void __launch_bounds__(kThreads, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
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
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(p.err, 0u, 8u);
    return;
  }
  // the combine grid may be scheduled now; it waits for this grid to finish
  griddep_launch_dependents();

  const int split = blockIdx.x;
  const int g = blockIdx.y;  // K/V head
  const int b = blockIdx.z;
  const int L = min(max(p.seqlens[b], 0), p.Smax);  // valid cache rows
  const int rows = p.group * p.Sq;                   // query rows of the tile (<= 128)
  const int n_tiles = (L + BN - 1) / BN;
  const int j0 = split * p.tiles_per_split;
  const int j1 = min(j0 + p.tiles_per_split, n_tiles);
  const int n_kv = j1 > j0 ? j1 - j0 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) mbar_init(bar(i), i == C::kBarP ? 128u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Query tile rows past `rows` are never loaded: zero them once so that they
  // stay finite padding.
  for (int e = threadIdx.x; e < C::kTileBytes / 16; e += kThreads)
    reinterpret_cast<uint4*>(smem + C::kQOff)[e] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
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

  auto finish = [&]() {
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
      const uint64_t drain_ns = 2000000000ull;
      if (warp == kMmaWarp && lane == 0) {
        tc_commit(bar(C::kBarDone));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bar(C::kBarDone), 0))
          if (globaltimer_ns() - t0 > drain_ns) break;
      }
      if ((warp == kLoadKWarp || warp == kLoadVWarp) && lane == 0 && n_kv > 0) {
        // every issued load lands within microseconds; give them time before
        // the shared memory goes away
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000ull) {
        }
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
    // ------------------------------------------------------------ softmax + partial output
    const int r = warp * 32 + lane;  // tile row = query position i * group + head offset
    const bool row_ok = r < rows;
    const int i = r / p.group;                  // new-query index (0 .. Sq-1)
    const int h = g * p.group + r % p.group;    // query head
    // last visible key of this row (inclusive); keys are 0 .. L-1
    const int hi = p.causal ? min(L - 1, L - p.Sq + i) : L - 1;
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::kColO;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int t = 0; t < n_kv; ++t) {
      const int j = j0 + t;
      const int n0 = j * BN;
      const uint32_t tS = tmem + lane_off + C::col_s(t);
      if (!bw.wait_warp(bar(C::kBarS + (t & 1)), (t >> 1) & 1, 40)) { ok = false; break; }
      tc_fence_after();
      float s[BN];
      {
        uint32_t rr[BN];
        tmem_ld128(tS, rr);
        const int c_hi = hi - n0;  // columns > c_hi are not visible
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = (c > c_hi) ? -INFINITY : __uint_as_float(rr[c]);
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
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};  // four independent partial sums
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int e = half * 64 + 2 * c;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), scale2, negm2), x0, x1);
          const uint64_t p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          acc2[c & 3] = f2_add(acc2[c & 3], p2);
          float p0, p1;
          f2_unpack(p2, p0, p1);
          pk[c] = E::pack2(p0, p1);
        }
        tmem_st32(tS + half * 32, pk);
      }
      float sum;
      {
        float lo, hi2;
        f2_unpack(f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3])), lo, hi2);
        sum = lo + hi2;
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
      if (t > 0 && __any_sync(0xffffffffu, bump)) {
        if (!bw.wait_warp(bar(C::kBarO), (t - 1) & 1, 41)) { ok = false; break; }
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
      // V rows past the sequence (this thread's row r of the slot's V tile)
      // hold no value of this sequence: zero them, once the tile has landed,
      // before P V reads them.  (The slot cannot be refilled meanwhile: that
      // waits for P V of this tile.)
      if (n0 + BN > L) {
        if (!bw.wait_warp(bar(C::kBarVFull + t % C::kSlots), (t / C::kSlots) & 1, 47)) {
          ok = false;
          break;
        }
      }
      if (n0 + r >= L) {
        const uint32_t vrow = v_addr(t % C::kSlots) + uint32_t(r) * 128;
#pragma unroll
        for (int x = 0; x < C::kBoxes; ++x)
#pragma unroll
          for (int k = 0; k < 8; ++k) st_shared_v4(vrow + x * C::kBoxBytes + k * 16, 0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarP));
    }
    // partial O (normalised) and log-sum-exp of this split for this row
    // (`ok` is warp-uniform; the tensor-memory loads below are warp-collective,
    // so every lane runs them and only the stores are limited to query rows)
    if (ok && n_kv > 0) ok = bw.wait_warp(bar(C::kBarOFinal), 0, 42);
    if (ok) {
      const size_t prow = ((size_t(b) * p.H + h) * p.Sq + i) * p.nsplit + split;
      float* dst = p.opart + prow * D;
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
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(dst + c0 + c) =
                make_float4(__uint_as_float(rr[c]) * inv_l, __uint_as_float(rr[c + 1]) * inv_l,
                            __uint_as_float(rr[c + 2]) * inv_l, __uint_as_float(rr[c + 3]) * inv_l);
        }
      }
      if (row_ok)
        p.lsepart[prow] = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994530942f
                                      : -INFINITY;
    }
    finish();
    return;
  }
  if (warp == kLoadKWarp) {
    // ------------------------------------------------------------ Q and K tiles
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      // the group's query heads for every new position: box (64 d, group heads, Sq rows)
      mbar_arrive_expect_tx(bar(C::kBarQ), rows * D * 2);
      for (int x = 0; x < C::kBoxes; ++x)
        tma_load_4d(sbase + C::kQOff + x * C::kBoxBytes, &tmQ, bar(C::kBarQ), x * 64,
                    g * p.group, 0, b);
      for (int t = 0; t < n_kv; ++t) {
        const int s = t % C::kSlots;
        const int u = t / C::kSlots;
        if (u > 0 && !bw.wait(bar(C::kBarKEmpty + s), (u - 1) & 1, 43)) break;
        const uint32_t fb = bar(C::kBarKFull + s);
        mbar_arrive_expect_tx(fb, C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_4d(k_addr(s) + x * C::kBoxBytes, &tmK, fb, x * 64, g, (j0 + t) * BN, b);
      }
    }
  } else if (warp == kLoadVWarp) {
    // ------------------------------------------------------------ V tiles
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmV);
      for (int t = 0; t < n_kv; ++t) {
        const int s = t % C::kSlots;
        const int u = t / C::kSlots;
        if (u > 0 && !bw.wait(bar(C::kBarVEmpty + s), (u - 1) & 1, 48)) break;
        const uint32_t fb = bar(C::kBarVFull + s);
        mbar_arrive_expect_tx(fb, C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_4d(v_addr(s) + x * C::kBoxBytes, &tmV, fb, x * 64, g, (j0 + t) * BN, b);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t idesc_qk = idesc_f32acc(BM, BN, false, false, E::kFmt);
      constexpr uint32_t idesc_pv = idesc_f32acc(BM, D, false, true, E::kFmt);
      const uint64_t q_desc = sdesc_sw128(sbase + C::kQOff, 16);
      bool ok = bw.wait(bar(C::kBarQ), 0, 44);
      // S(t) into buffer t % 2 as soon as K(t) has landed (its slot is handed
      // back when S(t) completes); S(t + 2) reuses the buffer once P V(t)
      // (which reads P(t) from it) is issued.
      auto issue_s = [&](int t) -> bool {
        const int s = t % C::kSlots;
        if (!bw.wait(bar(C::kBarKFull + s), (t / C::kSlots) & 1, 45)) return false;
        tc_fence_after();
        if constexpr (D == 128)
          mma_chain_kk8(tmem + C::col_s(t), q_desc, sdesc_sw128(k_addr(s), 16), idesc_qk, 0u);
        else
          mma_chain_kk4(tmem + C::col_s(t), q_desc, sdesc_sw128(k_addr(s), 16), idesc_qk, 0u);
        tc_commit(bar(C::kBarS + (t & 1)));
        tc_commit(bar(C::kBarKEmpty + s));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_kv > 1) ok = issue_s(1);
      for (int t = 0; ok && t < n_kv; ++t) {
        const int s = t % C::kSlots;
        if (!bw.wait(bar(C::kBarP), t & 1, 46)) break;
        if (!bw.wait(bar(C::kBarVFull + s), (t / C::kSlots) & 1, 49)) break;
        tc_fence_after();
        mma_chain_ts_mn8(tmem + C::kColO, tmem + C::col_s(t),
                         sdesc_sw128(v_addr(s), C::kBoxBytes), idesc_pv, t > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarO));
        tc_commit(bar(C::kBarVEmpty + s));
        if (t == n_kv - 1) tc_commit(bar(C::kBarOFinal));
        if (t + 2 < n_kv) ok = issue_s(t + 2);
      }
    }
  }
  finish();
}

// ---------------------------------------------------------------------------
// Transposed decode kernel: at most 16 query rows per K/V head, head_dim 128.
// ---------------------------------------------------------------------------
// With a handful of query rows (one new token and a few query heads per K/V
// head), putting the rows on the tensor-memory lanes leaves 124 of 128 lanes
// idle and makes every softmax thread exponentiate 128 scores of a padding
// row.  Here the keys are on the lanes instead:
//   S^T = K Q^T      (M = 128 keys, N = 16 rows; A = K tile, B = Q, both K-major)
//   O^T += V^T P^T   (M = 128 = head_dim, N = 16 rows; A = V tile read MN-major,
//                     B = P^T from shared memory, K-major over the keys)
// so each softmax thread owns one key and 16 scores.  At head_dim 64 the same
// kernel runs with M = 128 for O^T: the second 64-row block of its A operand
// (V^T) is a box cleared once per CTA, so rows 64..127 of O^T stay zero and are
// never written out; the smaller slots let two CTAs share an SM.  The row maximum is a
// reduction over the 128 threads (shuffles within a warp, then shared memory
// across the four warps); row sums stay per thread until the end.  P^T is
// written as 16-bit values into a double-buffered 4 KB shared tile.
namespace t16 {
constexpr int kRows = 16;       // N of both products
constexpr int kThreads = 224;   // warps 0-3 softmax, 4 MMA, 5 Q/K loads, 6 V loads
// D: head_dim.  At D = 64 the K and V slots hold one 64-column box, the
// rings have two slots, and one cleared box after the V ring stands in for
// rows 64..127 of the M = 128 product O^T (its descriptor's M stride points
// there): about 93 KB of shared memory, so two CTAs share an SM.
template <int D>
struct Cfg {
  static constexpr int kBoxBytes = BN * 128;         // K/V box: 128 rows x 64 columns
  static constexpr int kTileBytes = (D / 64) * kBoxBytes;  // K or V slot
  static constexpr int kSmallBox = kRows * 128;       // Q / P^T box: 16 rows x 64 columns
  static constexpr int kSlots = D == 128 ? 3 : 2;
  static constexpr int kQOff = 0;                                  // 2 small boxes
  static constexpr int kPOff = 2 * kSmallBox;                      // 2 buffers x 2 small boxes
  static constexpr int kKOff = kPOff + 4 * kSmallBox;              // K ring (1024-aligned)
  static constexpr int kVOff = kKOff + kSlots * kTileBytes;        // V ring
  static constexpr int kZeroOff = kVOff + kSlots * kTileBytes;     // D = 64: one cleared box
  static constexpr int kRedOff = kZeroOff + (D == 64 ? kBoxBytes : 0);  // [2][4 warps][16] floats
  static constexpr int kBarOff = kRedOff + 2 * 4 * kRows * 4;
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kSlots;
  static constexpr int kBarVFull = kBarKEmpty + kSlots;
  static constexpr int kBarVEmpty = kBarVFull + kSlots;
  static constexpr int kBarS = kBarVEmpty + kSlots;   // [2]
  static constexpr int kBarP = kBarS + 2;
  static constexpr int kBarPFree = kBarP + 1;         // [2]: P V of the buffer's last use done
  static constexpr int kBarO = kBarPFree + 2;
  static constexpr int kBarOFinal = kBarO + 1;        // once, after the last P V (see above)
  static constexpr int kBarDone = kBarOFinal + 1;
  static constexpr int kNumBars = kBarDone + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr int kCtasPerSm = D == 128 ? 1 : 2;
  static constexpr uint32_t kColO = 2 * kRows;        // S^T buffers at 0 and 16, O^T at 32
  static constexpr int kTmemCols = 64;
  static_assert(kKOff % 1024 == 0 && kVOff % 1024 == 0 && kZeroOff % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory exceeds the 227 KB per block of sm_100");
  static_assert(kCtasPerSm == 1 || kSmemBytes + 1024 <= 233472 / 2,
                "two CTAs per SM must fit the SM's shared memory");
};

// Butterfly reduction of 16 per-lane values over the 32 lanes of a warp: 16
// shuffles; afterwards lane l holds the result for row l >> 1 in v[0].
template <class Op>
__device__ __forceinline__ float warp_reduce16(float (&v)[kRows], Op op) {
#pragma unroll
  for (int half = 8, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
    const bool upper = (threadIdx.x & bit) != 0;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float send = upper ? v[k] : v[k + half];
      const float mine = upper ? v[k + half] : v[k];
      v[k] = op(mine, __shfl_xor_sync(0xffffffffu, send, bit));
    }
  }
  return op(v[0], __shfl_xor_sync(0xffffffffu, v[0], 1));
}

// D: head_dim, 64 or 128.
template <int D, class E>
__global__ void __launch_bounds__(kThreads, Cfg<D>::kCtasPerSm)
    attn_decode_t16_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const Params p) {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  using C = Cfg<D>;
  constexpr int kBoxes = D / 64;                 // 64-column boxes loaded per K/V tile
  constexpr int kLoadBytes = BN * D * 2;         // bytes landing per K/V tile
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
  // the combine grid may be scheduled now; it waits for this grid to finish
  griddep_launch_dependents();

  const int split = blockIdx.x;
  const int g = blockIdx.y;  // K/V head
  const int b = blockIdx.z;
  const int L = min(max(p.seqlens[b], 0), p.Smax);
  const int rows = p.group * p.Sq;  // <= 16
  const int n_tiles = (L + BN - 1) / BN;
  const int j0 = split * p.tiles_per_split;
  const int j1 = min(j0 + p.tiles_per_split, n_tiles);
  const int n_kv = j1 > j0 ? j1 - j0 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) mbar_init(bar(i), i == C::kBarP ? 128u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Q rows past `rows` are never loaded: zero the two small boxes once.
  for (int e = threadIdx.x; e < 2 * C::kSmallBox / 16; e += kThreads)
    reinterpret_cast<uint4*>(smem + C::kQOff)[e] = make_uint4(0u, 0u, 0u, 0u);
  if constexpr (D == 64) {
    // the cleared box: rows 64..127 of the M = 128 product O^T
    for (int e = threadIdx.x; e < C::kBoxBytes / 16; e += kThreads)
      reinterpret_cast<uint4*>(smem + C::kZeroOff)[e] = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Bounded bw{abort_flag, p.err, p.timeout_ns};
  auto k_addr = [&](int s) { return sbase + C::kKOff + s * C::kTileBytes; };
  auto v_addr = [&](int s) { return sbase + C::kVOff + s * C::kTileBytes; };
  auto p_addr = [&](int buf) { return sbase + C::kPOff + buf * 2 * C::kSmallBox; };

  auto finish = [&]() {
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
      const uint64_t drain_ns = 2000000000ull;
      if (warp == kMmaWarp && lane == 0) {
        tc_commit(bar(C::kBarDone));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bar(C::kBarDone), 0))
          if (globaltimer_ns() - t0 > drain_ns) break;
      }
      if ((warp == 5 || warp == 6) && lane == 0 && n_kv > 0) {
        // every issued load lands within microseconds; give them time before
        // the shared memory goes away
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000ull) {
        }
      }
      tc_fence_before();
      __syncthreads();
    }
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, C::kTmemCols);
    }
  };

  if (warp < 4) {
    // ------------------------------------------------------------ softmax (one key per thread)
    const int j = warp * 32 + lane;  // key within the tile = tensor-memory lane
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    float* red = reinterpret_cast<float*>(smem + C::kRedOff);  // [2][4][16]
    float m_run[kRows], lsum[kRows];
    int hi[kRows];  // last visible key of each row (inclusive); -1 for padding rows
#pragma unroll
    for (int c = 0; c < kRows; ++c) {
      m_run[c] = -INFINITY;
      lsum[c] = 0.f;
      const int i = c / p.group;
      hi[c] = c < rows ? (p.causal ? min(L - 1, L - p.Sq + i) : L - 1) : -1;
    }
    // Every warp meets the others at one barrier per tile; a failed wait is
    // carried to that barrier, so that all four warps stop at the same tile.
    bool carry = true;
    bool ok = true;
    for (int t = 0; t < n_kv; ++t) {
      const int n0 = (j0 + t) * BN;
      const int key = n0 + j;
      const int buf = t & 1;
      bool wok = carry && bw.wait_warp(bar(C::kBarS + buf), (t >> 1) & 1, 60);
      float s[kRows];
      if (wok) {
        tc_fence_after();
        uint32_t rr[kRows];
        tmem_ld16(tmem + lane_off + uint32_t(buf * kRows), rr);
#pragma unroll
        for (int c = 0; c < kRows; ++c) s[c] = key <= hi[c] ? __uint_as_float(rr[c]) : -INFINITY;
      } else {
#pragma unroll
        for (int c = 0; c < kRows; ++c) s[c] = -INFINITY;
      }
      {
        float v[kRows];
#pragma unroll
        for (int c = 0; c < kRows; ++c) v[c] = s[c];
        const float wm = warp_reduce16(v, [](float a, float b2) { return fmaxf(a, b2); });
        if ((lane & 1) == 0) red[(buf * 4 + warp) * kRows + (lane >> 1)] = wm;
      }
      if (!named_bar_and(1, 128, wok)) { ok = false; break; }
      carry = true;
      float mx[kRows];
      {
        const float4* r4 = reinterpret_cast<const float4*>(red + buf * 4 * kRows);
#pragma unroll
        for (int q4 = 0; q4 < kRows / 4; ++q4) {
          float4 a = r4[q4];
#pragma unroll
          for (int w = 1; w < 4; ++w) {
            const float4 o4 = r4[w * (kRows / 4) + q4];
            a.x = fmaxf(a.x, o4.x);
            a.y = fmaxf(a.y, o4.y);
            a.z = fmaxf(a.z, o4.z);
            a.w = fmaxf(a.w, o4.w);
          }
          mx[4 * q4] = a.x;
          mx[4 * q4 + 1] = a.y;
          mx[4 * q4 + 2] = a.z;
          mx[4 * q4 + 3] = a.w;
        }
      }
      // online update with the lazy rescale (identical in every thread)
      float alpha[kRows], pv[kRows];
      bool any_bump = false;
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        const float m_cand = mx[c] * sl2;
        const bool bump = m_cand > m_run[c] + kRescaleThreshold;
        const float m_new = bump ? m_cand : m_run[c];
        alpha[c] = bump ? ex2_approx(m_run[c] - m_new) : 1.0f;
        any_bump |= bump;
        m_run[c] = m_new;
        const float m_eff = (m_new == -INFINITY) ? 0.0f : m_new;
        pv[c] = ex2_approx(fmaf(s[c], sl2, -m_eff));
        lsum[c] = fmaf(lsum[c], alpha[c], pv[c]);
      }
      // this P^T buffer was last read by P V(t - 2)
      if (t >= 2 && !bw.wait_warp(bar(C::kBarPFree + buf), ((t >> 1) + 1) & 1, 61)) {
        carry = false;
        continue;
      }
      {
        const uint32_t pb = p_addr(buf) + uint32_t(j >> 6) * C::kSmallBox;
        const uint32_t jj = uint32_t(j & 63);
        uint8_t* pbase = smem + (pb - sbase) + (jj & 7) * 2;
#pragma unroll
        for (int c = 0; c < kRows; ++c) {
          const uint32_t off = uint32_t(c) * 128 + (((jj >> 3) ^ uint32_t(c & 7)) << 4);
          *reinterpret_cast<uint16_t*>(pbase + off) = uint16_t(E::pack2(pv[c], 0.f) & 0xFFFFu);
        }
      }
      if (t > 0 && any_bump) {
        if (!bw.wait_warp(bar(C::kBarO), (t - 1) & 1, 62)) {
          carry = false;
          continue;
        }
        tc_fence_after();
        uint32_t rr[kRows];
        tmem_ld16(tmem + lane_off + C::kColO, rr);
#pragma unroll
        for (int c = 0; c < kRows; ++c) rr[c] = __float_as_uint(__uint_as_float(rr[c]) * alpha[c]);
        tmem_st16(tmem + lane_off + C::kColO, rr);
      }
      // V rows past the sequence hold no value of this sequence: zero this
      // thread's row of the slot, once the tile has landed, before P V reads it.
      if (n0 + BN > L) {
        if (!bw.wait_warp(bar(C::kBarVFull + t % C::kSlots), (t / C::kSlots) & 1, 63)) {
          carry = false;
          continue;
        }
        if (key >= L) {
          const uint32_t vrow = v_addr(t % C::kSlots) + uint32_t(j) * 128;
#pragma unroll
          for (int x = 0; x < kBoxes; ++x)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              st_shared_v4(vrow + x * C::kBoxBytes + k * 16, 0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(C::kBarP));
    }
    // ------------------------------------------------------------ partial output
    bool eok = ok && carry;
    if (eok && n_kv > 0) eok = bw.wait_warp(bar(C::kBarOFinal), 0, 64);
    {
      float v[kRows];
#pragma unroll
      for (int c = 0; c < kRows; ++c) v[c] = lsum[c];
      const float ws = warp_reduce16(v, [](float a, float b2) { return a + b2; });
      if ((lane & 1) == 0) red[((n_kv & 1) * 4 + warp) * kRows + (lane >> 1)] = ws;
    }
    // all four warps reach this barrier (a warp that left the loop early left
    // it at the same tile as the others)
    if (named_bar_and(1, 128, eok)) {
      const float* rl = red + (n_kv & 1) * 4 * kRows;
      if (n_kv > 0) tc_fence_after();
      uint32_t rr[kRows];
      if (n_kv > 0) {
        tmem_ld16(tmem + lane_off + C::kColO, rr);
      } else {
#pragma unroll
        for (int c = 0; c < kRows; ++c) rr[c] = 0u;
      }
      const int d = j;  // O^T lane = head-dim index (lanes D..127 hold zeros at D = 64)
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        if (c >= rows || d >= D) break;
        const float l = rl[c] + rl[kRows + c] + rl[2 * kRows + c] + rl[3 * kRows + c];
        const int i = c / p.group;
        const int h = g * p.group + c % p.group;
        const size_t prow = ((size_t(b) * p.H + h) * p.Sq + i) * p.nsplit + split;
        p.opart[prow * D + d] = l > 0.f ? __uint_as_float(rr[c]) / l : 0.f;
        if (d == 0)
          p.lsepart[prow] =
              l > 0.f ? (m_run[c] + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      }
    }
    finish();
    return;
  }
  if (warp == 5) {
    // ------------------------------------------------------------ Q and K tiles
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_arrive_expect_tx(bar(C::kBarQ), rows * D * 2);
      for (int x = 0; x < kBoxes; ++x)
        tma_load_4d(sbase + C::kQOff + x * C::kSmallBox, &tmQ, bar(C::kBarQ), x * 64,
                    g * p.group, 0, b);
      for (int t = 0; t < n_kv; ++t) {
        const int s = t % C::kSlots;
        const int u = t / C::kSlots;
        if (u > 0 && !bw.wait(bar(C::kBarKEmpty + s), (u - 1) & 1, 65)) break;
        const uint32_t fb = bar(C::kBarKFull + s);
        mbar_arrive_expect_tx(fb, kLoadBytes);
        for (int x = 0; x < kBoxes; ++x)
          tma_load_4d(k_addr(s) + x * C::kBoxBytes, &tmK, fb, x * 64, g, (j0 + t) * BN, b);
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ V tiles
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmV);
      for (int t = 0; t < n_kv; ++t) {
        const int s = t % C::kSlots;
        const int u = t / C::kSlots;
        if (u > 0 && !bw.wait(bar(C::kBarVEmpty + s), (u - 1) & 1, 66)) break;
        const uint32_t fb = bar(C::kBarVFull + s);
        mbar_arrive_expect_tx(fb, kLoadBytes);
        for (int x = 0; x < kBoxes; ++x)
          tma_load_4d(v_addr(s) + x * C::kBoxBytes, &tmV, fb, x * 64, g, (j0 + t) * BN, b);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t idesc_s = idesc_f32acc(BN, kRows, false, false, E::kFmt);
      constexpr uint32_t idesc_o = idesc_f32acc(128, kRows, true, false, E::kFmt);  // M = 128 rows of O^T
      const uint64_t q_desc = sdesc_sw128(sbase + C::kQOff, 16);
      bool ok = bw.wait(bar(C::kBarQ), 0, 67);
      // S^T(t) into buffer t % 2 once K(t) has landed (the K slot is handed
      // back when it completes); S^T(t + 2) reuses the buffer after P(t) has
      // been read out of it (the softmax arrived P(t)).
      auto issue_s = [&](int t) -> bool {
        const int s = t % C::kSlots;
        if (!bw.wait(bar(C::kBarKFull + s), (t / C::kSlots) & 1, 68)) return false;
        tc_fence_after();
        if constexpr (D == 128)
          mma_chain_kk8_b16(tmem + uint32_t((t & 1) * kRows), sdesc_sw128(k_addr(s), 16), q_desc,
                            idesc_s, 0u);
        else
          mma_chain_kk4(tmem + uint32_t((t & 1) * kRows), sdesc_sw128(k_addr(s), 16), q_desc,
                        idesc_s, 0u);
        tc_commit(bar(C::kBarS + (t & 1)));
        tc_commit(bar(C::kBarKEmpty + s));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_kv > 1) ok = issue_s(1);
      for (int t = 0; ok && t < n_kv; ++t) {
        const int s = t % C::kSlots;
        if (!bw.wait(bar(C::kBarP), t & 1, 69)) break;
        if (!bw.wait(bar(C::kBarVFull + s), (t / C::kSlots) & 1, 70)) break;
        tc_fence_after();
        // A = V^T: at D = 64 its second 64-row block is the cleared box
        const uint32_t m_stride = D == 128 ? uint32_t(C::kBoxBytes)
                                           : sbase + C::kZeroOff - v_addr(s);
        mma_chain_mnk8_b16(tmem + C::kColO, sdesc_sw128(v_addr(s), m_stride),
                           sdesc_sw128(p_addr(t & 1), 16), idesc_o, t > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarO));
        tc_commit(bar(C::kBarVEmpty + s));
        tc_commit(bar(C::kBarPFree + (t & 1)));
        if (t == n_kv - 1) tc_commit(bar(C::kBarOFinal));
        if (t + 2 < n_kv) ok = issue_s(t + 2);
      }
    }
  }
  finish();
}
}  // namespace t16

// Merge the splits of one (batch, query head, new position) row per warp:
// LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s, rounded to E.
template <int D, class E>
__global__ void __launch_bounds__(256) attn_decode_combine_kernel(
    const float* __restrict__ opart, const float* __restrict__ lsepart,
    uint16_t* __restrict__ o, float* __restrict__ lse, int B, int Sq, int H, int nsplit) {
  // launched as a programmatic dependent of the split kernel: wait for it to
  // complete before reading its partial results
  griddep_wait();
  const long long row = (long long)blockIdx.x * 8 + threadIdx.x / 32;  // (b, h, i)
  const int lane = threadIdx.x % 32;
  if (row >= (long long)B * H * Sq) return;
  const int i = int(row % Sq);
  const int h = int((row / Sq) % H);
  const int b = int(row / ((long long)Sq * H));
  const float* lp = lsepart + row * nsplit;
  float mx = -INFINITY;
  for (int s = lane; s < nsplit; s += 32) mx = fmaxf(mx, lp[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float den = 0.f;
  if (mx != -INFINITY)
    for (int s = lane; s < nsplit; s += 32) den += __expf(lp[s] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  const float total = mx == -INFINITY ? -INFINITY : mx + __logf(den);
  constexpr int kPer = D / 32;  // elements of the row per lane (2 or 4)
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  if (total != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const float ls = lp[s];
      if (ls == -INFINITY) continue;
      const float w = __expf(ls - total);
      const float* src = opart + (row * nsplit + s) * D + lane * kPer;
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, src[e], acc[e]);
    }
  }
  uint16_t* dst = o + ((size_t(b) * Sq + i) * H + h) * D + lane * kPer;
#pragma unroll
  for (int e = 0; e < kPer; e += 2)
    *reinterpret_cast<uint32_t*>(dst + e) = E::pack2(acc[e], acc[e + 1]);
  if (lane == 0) lse[(size_t(b) * H + h) * Sq + i] = total;
}

}  // namespace dec
}  // namespace attn156
