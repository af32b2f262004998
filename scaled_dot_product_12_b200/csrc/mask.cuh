// Generalized Sliding Window: per-sequence window, per-row key interval and
// the tile plan (which 128x128 tiles hold any allowed pair, and which need no
// element test).  Compiled for host and device so the host exports
// attn_tile_plan / attn_allowed_pairs run exactly the code the kernels run.
//
// Rule (AOTriton 0.10b release notes, "Major Changes from Release 0.9 Beta";
// AOTriton 0.15b release notes, "Bottom-Right Aligned Sliding Windows"):
// with d = seqlen_k - seqlen_q, a numeric window (wl, wr) is (L, R) = (wl, wr)
// under TOP_LEFT and (wl - d, wr + d) under BOTTOM_RIGHT; the causal
// sentinels mean (INF, 0) and (INF, d) whatever the diagonal bit says; row i
// sees keys j with i - L <= j <= i + R.
#pragma once

#include <stdint.h>

#ifndef ATTN_HD
#ifdef __CUDACC__
#define ATTN_HD __host__ __device__ __forceinline__
#else
#define ATTN_HD inline
#endif
#endif

namespace attn {

constexpr int32_t kWindowInf = 2147483647;
constexpr int32_t kCausalTopLeft = -2147483647 - 1;
constexpr int32_t kCausalBottomRight = -2147483647;
// |L|, |R| are clamped to this; sequence lengths are below it, so int32
// arithmetic on i - L and i + R cannot overflow and a clamped side still
// covers (or excludes) every key.
constexpr int32_t kBig = 1 << 30;
constexpr int kTileM = 128;
constexpr int kTileN = 128;

struct SeqWindow {
  int32_t L, R;  // key j allowed for row i iff i - L <= j <= i + R
};

ATTN_HD int64_t clamp_big(int64_t x) { return x < -kBig ? -kBig : (x > kBig ? kBig : x); }

ATTN_HD SeqWindow seq_window(int32_t wl, int32_t wr, bool bottom_right, int32_t sq, int32_t sk) {
  const int64_t d = (int64_t)sk - (int64_t)sq;
  int64_t L, R;
  if (wl == kCausalTopLeft) {
    L = kBig;
    R = 0;
  } else if (wl == kCausalBottomRight) {
    L = kBig;
    R = d;
  } else {
    L = (wl == kWindowInf) ? (int64_t)kBig : (bottom_right ? (int64_t)wl - d : (int64_t)wl);
    R = (wr == kWindowInf) ? (int64_t)kBig : (bottom_right ? (int64_t)wr + d : (int64_t)wr);
  }
  SeqWindow w;
  w.L = (int32_t)clamp_big(L);
  w.R = (int32_t)clamp_big(R);
  return w;
}

// First and last allowed key of row i (first > last when the row is empty).
ATTN_HD int32_t row_lo(const SeqWindow& w, int32_t i) {
  int32_t lo = i - w.L;
  return lo < 0 ? 0 : lo;
}
ATTN_HD int32_t row_hi(const SeqWindow& w, int32_t i, int32_t sk) {
  int32_t hi = i + w.R;
  return hi > sk - 1 ? sk - 1 : hi;
}

// Key tiles [*nb, *ne) that the query rows [m0, m0 + rows) may attend.
// lo(i) and hi(i) never decrease with i, so the union of the rows' intervals
// lies in [lo(m0), hi(m_last)].
ATTN_HD void fwd_tile_range(const SeqWindow& w, int32_t sq, int32_t sk, int32_t m0, int32_t rows,
                            int32_t* nb, int32_t* ne) {
  *nb = 0;
  *ne = 0;
  if (m0 >= sq || sk <= 0) return;
  int32_t m_last = m0 + rows - 1;
  if (m_last > sq - 1) m_last = sq - 1;
  const int32_t first = row_lo(w, m0);
  const int32_t last = row_hi(w, m_last, sk);
  if (first > last) return;
  *nb = first / kTileN;
  *ne = last / kTileN + 1;
}

// True if every pair of query tile [m0, m0 + kTileM) x key tile [n0, n0 +
// kTileN) is allowed and in range, so the kernels may skip the element test.
ATTN_HD bool tile_is_full(const SeqWindow& w, int32_t sq, int32_t sk, int32_t m0, int32_t n0) {
  if (m0 + kTileM > sq || n0 + kTileN > sk) return false;
  const int32_t m_last = m0 + kTileM - 1;
  const int32_t n_last = n0 + kTileN - 1;
  return row_lo(w, m_last) <= n0 && row_hi(w, m0, sk) >= n_last;
}

// Query tiles [*mb, *me) whose rows see any key of [n0, n0 + kTileN): row i
// sees key j iff j - R <= i <= j + L (for 0 <= j < sk).
ATTN_HD void bwd_tile_range(const SeqWindow& w, int32_t sq, int32_t sk, int32_t n0, int32_t* mb,
                            int32_t* me) {
  *mb = 0;
  *me = 0;
  if (n0 >= sk || sq <= 0) return;
  int32_t n_last = n0 + kTileN - 1;
  if (n_last > sk - 1) n_last = sk - 1;
  int32_t first = n0 - w.R;
  if (first < 0) first = 0;
  int32_t last = n_last + w.L;
  if (last > sq - 1) last = sq - 1;
  if (first > last) return;
  *mb = first / kTileM;
  *me = last / kTileM + 1;
}

}  // namespace attn
