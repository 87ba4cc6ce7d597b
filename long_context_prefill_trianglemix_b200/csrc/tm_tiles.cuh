// Static tile list of the TriangleMix patterns, shared by host and device.
//
// The kernels never branch over skipped tiles: every q-block derives, from a
// closed form, the ascending list of k-blocks that hold at least one kept
// pair and visits exactly those (the "jump by index instead of testing every
// block" idea that the FlashPrefill summary, section 2.3, contrasts with
// logical skipping). For the triangle pattern (TriangleMix blog post,
// section 介绍; 36kr interview, lead) the kept keys of row i are
//   [0, i]                                      if i >= N - L,
//   [0, min(S, i+1)) U [max(0, i-W+1), i]        otherwise,
// so a q-block with rows [r0, r1] needs
//   every k-block 0 .. r1/BN                    if r1 >= N - L,
//   sinks 0 .. ceil(min(S, r1+1)/BN) - 1 and the band
//   floor(max(0, r0-W+1)/BN) .. r1/BN           otherwise (merged if they touch).
// Every listed tile holds a kept pair: row r1 keeps each sink column and, for a
// band column c, row max(c, r0) keeps it.
#pragma once

#if defined(__CUDACC__)
#define TM_HD __host__ __device__ __forceinline__
#else
#define TM_HD inline
#endif

namespace trimix {

struct Pattern {
  int N, S, W, L;  // S, L clamped to [0, N]; W clamped to [1, N]
  int causal;
};

TM_HD int imin(int a, int b) { return a < b ? a : b; }
TM_HD int imax(int a, int b) { return a > b ? a : b; }

TM_HD Pattern make_pattern(int N, int causal, int S, int W, int L) {
  Pattern p;
  p.N = N;
  p.causal = causal ? 1 : 0;
  p.S = imin(imax(S, 0), N);
  p.W = imin(imax(W, 1), N);
  p.L = imin(imax(L, 0), N);
  return p;
}

// Kept k-blocks of one q-block: [0, n_a) followed by [b_lo, b_lo + n_b).
struct BlockTiles {
  int n_a;
  int b_lo;
  int n_b;
  TM_HD int count() const { return n_a + n_b; }
  TM_HD int kb(int t) const { return t < n_a ? t : b_lo + (t - n_a); }
};

// Kept k-blocks of the query rows [r0, r1] (r1 < N): the union of their kept
// keys, which is the closed form at the block's first and last rows.
TM_HD BlockTiles block_tiles_rows(const Pattern& p, int r0, int r1, int BN) {
  const int last = r1 / BN;
  BlockTiles t;
  if (p.causal || r1 >= p.N - p.L) {
    t.n_a = last + 1; t.b_lo = 0; t.n_b = 0;
    return t;
  }
  const int sink_end = imin(p.S, r1 + 1);          // exclusive column bound of the sinks
  const int n_sink = (sink_end + BN - 1) / BN;
  const int b_lo = imax(0, r0 - p.W + 1) / BN;
  if (b_lo <= n_sink) {                            // sinks and band touch: one run
    t.n_a = last + 1; t.b_lo = 0; t.n_b = 0;
  } else {
    t.n_a = n_sink; t.b_lo = b_lo; t.n_b = last - b_lo + 1;
  }
  return t;
}

TM_HD BlockTiles block_tiles(const Pattern& p, int qb, int BM, int BN) {
  return block_tiles_rows(p, qb * BM, imin(p.N, qb * BM + BM) - 1, BN);
}

// 1 iff every pair of the tile's existing rows [r0, r1] and columns [c0, c1] is
// kept. Rows below N-L exclude exactly the columns [S, i-W]; that gap only
// grows with i, so the largest such row decides.
TM_HD int tile_full(const Pattern& p, int qb, int kb, int BM, int BN) {
  const int r0 = qb * BM, r1 = imin(p.N, r0 + BM) - 1;
  const int c0 = kb * BN, c1 = imin(p.N, c0 + BN) - 1;
  if (c1 > r0) return 0;                           // some pair lies above the diagonal
  if (p.causal) return 1;
  const int i_max = imin(r1, p.N - p.L - 1);        // largest row outside the last-L rows
  if (i_max < r0) return 1;
  const int lo = imax(p.S, c0), hi = imin(i_max - p.W, c1);
  return lo > hi ? 1 : 0;
}

// The kernel also masks tiles whose columns run past N (TMA zero-fills them).
TM_HD int tile_needs_mask(const Pattern& p, int qb, int kb, int BM, int BN) {
  return (!tile_full(p, qb, kb, BM, BN)) || (kb * BN + BN > p.N);
}

// Kept (i, j) test for one element, used inside masked tiles only.
TM_HD bool keep(const Pattern& p, int i, int j) {
  if (j > i || j >= p.N) return false;
  if (p.causal || i >= p.N - p.L) return true;
  return j < p.S || i - j < p.W;
}

}  // namespace trimix
