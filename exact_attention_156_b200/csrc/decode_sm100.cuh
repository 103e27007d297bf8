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
//  * the split's 128-key K/V tiles stream through a shared-memory ring (TMA,
//    mbarrier full/empty pairs); tcgen05 computes S = Q K^T and O += P V in
//    tensor memory (the tensor core is mostly idle: the rows that are not
//    query rows are padding);
//  * warps 0-3: online softmax (one thread = one row), warp 4: MMA issue,
//    warp 5: TMA; S is double-buffered in tensor memory, so the products of
//    one tile (S of the next, P V of the previous) run under the softmax of
//    the other;
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
constexpr int kThreads = 192;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct Cfg {
  static constexpr int kBoxBytes = BN * 128;  // 128 rows x 64 columns
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = BN * D * 2;
  static constexpr int kStages = (D == 128) ? 3 : 6;  // K+V tile pairs in flight
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kTileBytes;  // stage s: [K tile | V tile]
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kStageBytes;
  static constexpr int kBarQ = 0;
  static constexpr int kBarFull = 1;
  static constexpr int kBarEmpty = kBarFull + kStages;
  static constexpr int kBarS = kBarEmpty + kStages;  // [2]: per S buffer
  static constexpr int kBarP = kBarS + 2;
  static constexpr int kBarO = kBarP + 1;
  static constexpr int kBarDone = kBarO + 1;
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
  auto kv_addr = [&](int s) { return sbase + C::kKVOff + s * C::kStageBytes; };

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
      if (warp == kLoadWarp && lane == 0 && n_kv > 0) {
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
      // V rows past the sequence (this thread's row r of the stage's V tile)
      // hold no value of this sequence: zero them before P V reads them.
      if (n0 + r >= L) {
        const uint32_t vrow = kv_addr(t % C::kStages) + C::kTileBytes + uint32_t(r) * 128;
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
    if (ok && n_kv > 0) ok = bw.wait_warp(bar(C::kBarO), (n_kv - 1) & 1, 42);
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
  if (warp == kLoadWarp) {
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // the group's query heads for every new position: box (64 d, group heads, Sq rows)
      mbar_arrive_expect_tx(bar(C::kBarQ), rows * D * 2);
      for (int x = 0; x < C::kBoxes; ++x)
        tma_load_4d(sbase + C::kQOff + x * C::kBoxBytes, &tmQ, bar(C::kBarQ), x * 64,
                    g * p.group, 0, b);
      for (int t = 0; t < n_kv; ++t) {
        const int s = t % C::kStages;
        const int u = t / C::kStages;
        if (u > 0 && !bw.wait(bar(C::kBarEmpty + s), (u - 1) & 1, 43)) break;
        const int n0 = (j0 + t) * BN;
        const uint32_t fb = bar(C::kBarFull + s);
        mbar_arrive_expect_tx(fb, 2 * C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x) {
          tma_load_4d(kv_addr(s) + x * C::kBoxBytes, &tmK, fb, x * 64, g, n0, b);
          tma_load_4d(kv_addr(s) + C::kTileBytes + x * C::kBoxBytes, &tmV, fb, x * 64, g, n0, b);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t idesc_qk = idesc_f32acc(BM, BN, false, false, E::kFmt);
      constexpr uint32_t idesc_pv = idesc_f32acc(BM, D, false, true, E::kFmt);
      const uint64_t q_desc = sdesc_sw128(sbase + C::kQOff, 16);
      bool ok = bw.wait(bar(C::kBarQ), 0, 44);
      // S(t) into buffer t % 2 as soon as its K/V tile has landed; S(t + 2)
      // reuses the buffer once P V(t) (which reads P(t) from it) is issued.
      auto issue_s = [&](int t) -> bool {
        const int s = t % C::kStages;
        if (!bw.wait(bar(C::kBarFull + s), (t / C::kStages) & 1, 45)) return false;
        tc_fence_after();
        if constexpr (D == 128)
          mma_chain_kk8(tmem + C::col_s(t), q_desc, sdesc_sw128(kv_addr(s), 16), idesc_qk, 0u);
        else
          mma_chain_kk4(tmem + C::col_s(t), q_desc, sdesc_sw128(kv_addr(s), 16), idesc_qk, 0u);
        tc_commit(bar(C::kBarS + (t & 1)));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_kv > 1) ok = issue_s(1);
      for (int t = 0; ok && t < n_kv; ++t) {
        const int s = t % C::kStages;
        if (!bw.wait(bar(C::kBarP), t & 1, 46)) break;
        tc_fence_after();
        mma_chain_ts_mn8(tmem + C::kColO, tmem + C::col_s(t),
                         sdesc_sw128(kv_addr(s) + C::kTileBytes, C::kBoxBytes), idesc_pv,
                         t > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarO));
        tc_commit(bar(C::kBarEmpty + s));
        if (t + 2 < n_kv) ok = issue_s(t + 2);
      }
    }
  }
  finish();
}

// Merge the splits of one (batch, query head, new position) row per warp:
// LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s, rounded to E.
template <int D, class E>
__global__ void __launch_bounds__(256) attn_decode_combine_kernel(
    const float* __restrict__ opart, const float* __restrict__ lsepart,
    uint16_t* __restrict__ o, float* __restrict__ lse, int B, int Sq, int H, int nsplit) {
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
