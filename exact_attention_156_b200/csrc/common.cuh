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

}  // namespace attn156
