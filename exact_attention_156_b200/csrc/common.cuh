// common.cuh - mask geometry shared by the forward and backward kernels.
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

}  // namespace attn156
