// common.cuh - mask geometry and packed-sequence spans shared by the kernels.
#pragma once

#include <stdint.h>

namespace attn156 {

// "Unbounded" window side.  Sequence lengths are below 2^25 (every tensor holds
// fewer than 2^31 elements and head_dim >= 64), so i + delta +/- kUnbounded
// never overflows a 32-bit int.
constexpr int kUnbounded = 1 << 30;

// Key j is visible to query i iff lo(i) <= j <= hi(i), with delta = Sk - Sq:
//   lo(i) = max(0, i + delta - left),  hi(i) = min(Sk - 1, i + delta + right)
// where left = win_left (or unbounded) and right = min(0 if causal,
// win_right if >= 0) (or unbounded).  Both bounds grow with i.
struct MaskGeom {
  int delta;
  int left;
  int right;
  int Sq;
  int Sk;

  __host__ __device__ static MaskGeom make(int Sq, int Sk, int causal, int win_left,
                                           int win_right) {
    MaskGeom g;
    g.delta = Sk - Sq;
    g.left = win_left >= 0 ? win_left : kUnbounded;
    int r = kUnbounded;
    if (causal) r = 0;
    if (win_right >= 0 && win_right < r) r = win_right;
    g.right = r;
    g.Sq = Sq;
    g.Sk = Sk;
    return g;
  }
  __host__ __device__ int lo(int i) const {
    int v = i + delta - left;
    return v < 0 ? 0 : v;
  }
  __host__ __device__ int hi(int i) const {
    int v = i + delta + right;
    return v > Sk - 1 ? Sk - 1 : v;
  }
  // Smallest / largest query index that sees key j (before clipping to [0, Sq)).
  __host__ __device__ int qmin(int j) const { return j - delta - right; }
  __host__ __device__ int qmax(int j) const { return j - delta + left; }
};

// Block order of a (tile, head-batch) grid.  The linear block index walks the
// head-batch combinations in chunks of `chunk`; inside a chunk it takes tile 0
// of every combination, then tile 1, and so on (tile 0 is the heaviest under a
// causal mask).  chunk = 1 is head-major order (one head's tiles side by side,
// sharing its operands in L2); chunk = n_hb is tile-major over the whole grid.
// A chunk whose operands fit in L2 together keeps that sharing while the
// heaviest tiles of every head start early, instead of the heaviest tiles of
// the last heads trailing after everything else.
struct ChunkedOrder {
  int tile, hb;
};
__host__ __device__ __forceinline__ ChunkedOrder chunked_order(int lin, int n_tiles, int n_hb, int chunk) {
  const int per = n_tiles * chunk;  // blocks of one full chunk
  const int full = n_hb / chunk;
  int c, rem, csz;
  if (lin < full * per) {
    c = lin / per;
    rem = lin - c * per;
    csz = chunk;
  } else {
    c = full;
    rem = lin - full * per;
    csz = n_hb - full * chunk;
  }
  ChunkedOrder o;
  o.tile = rem / csz;
  o.hb = c * chunk + rem % csz;
  return o;
}

// Device error word code for malformed packed-sequence boundaries.
constexpr uint32_t kErrSeqlens = 13u;

// One sequence of a packed variable-length batch: its first query and key
// rows and its lengths.  `ok` is false (and the lengths 0, so that nothing is
// read or written) unless 0 <= cu_q[b] <= cu_q[b+1] <= total_q with length at
// most max_q, and the same for the keys.
struct SeqSpan {
  int q0, k0, Lq, Lk;
  bool ok;
};
__device__ __forceinline__ SeqSpan seq_span(const int* cu_q, const int* cu_k, int b, int total_q,
                                            int total_k, int max_q, int max_k) {
  const int a0 = cu_q[b], a1 = cu_q[b + 1], c0 = cu_k[b], c1 = cu_k[b + 1];
  SeqSpan s{0, 0, 0, 0, false};
  if (a0 < 0 || a1 < a0 || a1 > total_q || a1 - a0 > max_q || c0 < 0 || c1 < c0 ||
      c1 > total_k || c1 - c0 > max_k)
    return s;
  s.q0 = a0;
  s.k0 = c0;
  s.Lq = a1 - a0;
  s.Lk = c1 - c0;
  s.ok = true;
  return s;
}

// Packed batches of at most kCompactMaxB sequences run on a compact grid: one
// CTA per (tile, sequence) that has work, instead of the longest sequence's tile
// count for every sequence (CTAs that only find their sequence too short to
// reach them still cost a launch and a shared-memory allocation each).
// Tiles are numbered level by level: level l holds tile l of every sequence
// that has more than l tiles, in sequence order, so the first level (each
// sequence's heaviest tile) starts first and the light tiles form the tail.
// A malformed sequence has no tiles.
constexpr int kCompactMaxB = 256;

// Tile `idx` of that numbering: returns the sequence (and its tile, 0 = the
// first level) or -1 past the last tile.  Every thread of a warp calls it
// (warp shuffles); lane i holds the tile counts of sequences i, i + 32, ....
// `rows`: rows per tile of the query axis (by_keys = 0) or the key axis.
__device__ __forceinline__ int compact_tile(const int* cu_q, const int* cu_k, int B, int total_q,
                                           int total_k, int max_q, int max_k, bool by_keys,
                                           int rows, int idx, int& tile) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = kCompactMaxB / 32;
  int cnt[kPer];
  int tmax = 0;
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int b = r * 32 + lane;
    cnt[r] = 0;
    if (b < B) {
      const SeqSpan sp = seq_span(cu_q, cu_k, b, total_q, total_k, max_q, max_k);
      cnt[r] = ((by_keys ? sp.Lk : sp.Lq) + rows - 1) / rows;
    }
    tmax = max(tmax, cnt[r]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) tmax = max(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
  for (int l = 0; l < tmax; ++l) {
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      if (r * 32 >= B) break;
      const unsigned has = __ballot_sync(0xffffffffu, cnt[r] > l);
      const int n = __popc(has);
      if (idx < n) {
        // the idx-th set bit of `has`
        unsigned m = has;
        for (int j = 0; j < idx; ++j) m &= m - 1;
        tile = l;
        return r * 32 + __ffs(m) - 1;
      }
      idx -= n;
    }
  }
  tile = 0;
  return -1;
}

// Run by one full warp of one CTA of a compact grid: a malformed sequence has
// no tiles, so no CTA of its own reports it; and with malformed (overlapping)
// boundaries the valid sequences' tiles could outnumber the grid.  Either sets
// the device error word.
__device__ __forceinline__ void compact_check(const int* cu_q, const int* cu_k, int B,
                                              int total_q, int total_k, int max_q, int max_k,
                                              bool by_keys, int rows, long long grid,
                                              uint32_t* err) {
  const int lane = threadIdx.x & 31;
  long long tiles = 0;
  bool bad = false;
  for (int b = lane; b < B; b += 32) {
    const SeqSpan sp = seq_span(cu_q, cu_k, b, total_q, total_k, max_q, max_k);
    bad = bad || !sp.ok;
    tiles += ((by_keys ? sp.Lk : sp.Lq) + rows - 1) / rows;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, off);
  bad = __any_sync(0xffffffffu, bad) != 0;
  if (lane == 0 && (bad || tiles > grid)) atomicCAS(err, 0u, kErrSeqlens);
}

}  // namespace attn156
