// mask_rules.cuh -- the mask_mod keep rules of the forward kernel, in the two forms it
// uses: per tile (which key tiles a query tile must visit, and whether a visited tile
// needs per-element masking) and per row (the contiguous interval of kept key columns
// inside one key tile).
//
// Keep rules (FlyDSL PR 931 "Add flex_attention (score_mod / mask_mod) on the generic
// flash-attention kernel", Summary: built-in causal / sliding_window mask_mods, plus an
// offset rule for cross-attention), indices absolute (top-left aligned):
//   NONE:            keep
//   CAUSAL:          j <= i
//   SLIDING_WINDOW:  j <= i  &&  i - j < W
//   KV_LE_Q_PLUS_OFF j <= i + off
//   DOCUMENT         i and j in the same document (captured per-batch boundaries
//                    off_q / off_kv: position p is in document d iff off[d] <= p < off[d+1])
//   DOCUMENT_CAUSAL  DOCUMENT && j <= i
// and every rule also requires j < Skv (the pad rule for a ragged last key tile).
// The document rules are tensor-capturing mask_mods (FlyDSL PR 931, Out of scope: a
// later phase); with non-decreasing boundaries the keys of row i's document form one
// interval, so they ride on the same interval machinery.
//
// For each rule the kept keys of row i form one interval [a(i), b(i)] with a and b
// non-decreasing in i, so the kept keys of a query tile (rows q0..q1-1) form the
// interval [a(q0), b(q1-1)], and a key tile [k0, k1) is FULL exactly when
// a(q1-1) <= k0 and k1 - 1 <= b(q0) and k1 <= Skv.
#pragma once

#include <cstdint>

namespace flexattn {

enum MaskKind : int {
  kMaskNone = 0,
  kMaskCausal = 1,
  kMaskSliding = 2,
  kMaskOffset = 3,
  kMaskDocument = 5,
  kMaskDocumentCausal = 6
};
enum ScoreKind : int { kScoreNone = 0, kScoreAlibi = 1 };
enum TileClass : int { kTileEmpty = 0, kTileFull = 1, kTilePartial = 2 };

struct MaskArgs {
  int Skv;
  int window;
  int offset;
  // document rules: this batch's boundaries, n_docs + 1 entries each (device memory)
  const int32_t* off_q = nullptr;
  const int32_t* off_kv = nullptr;
  int n_docs = 0;
};

// Largest d in [0, n] with off[d] <= i, or -1 when i < off[0] (binary search over
// non-decreasing boundaries; reads only off[0..n]).
__device__ __forceinline__ int doc_floor(const int32_t* off, int n, int64_t i) {
  if (static_cast<int64_t>(__ldg(off)) > i) return -1;
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<int64_t>(__ldg(off + mid)) <= i) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Kept key interval [lo, hi] of row i under the document rules, given d = its
// doc_floor.  Rows outside every document keep nothing; their empty interval sits at the
// boundary of the neighbouring documents so that both ends stay non-decreasing in i.
__device__ __forceinline__ void doc_interval(const MaskArgs& m, int d, int64_t i, bool causal, int64_t& lo,
                                             int64_t& hi) {
  const int dk = d < 0 ? 0 : d;
  const int64_t a = __ldg(m.off_kv + dk);
  const int64_t e = (d < 0 || d >= m.n_docs) ? a : static_cast<int64_t>(__ldg(m.off_kv + d + 1));
  lo = a > 0 ? a : 0;
  hi = static_cast<int64_t>(m.Skv) - 1;
  hi = e - 1 < hi ? e - 1 : hi;
  if (causal) hi = i < hi ? i : hi;
}

// Kept key interval [lo, hi] (inclusive, may be empty: lo > hi) of query row i.
template <int MASK>
__host__ __device__ __forceinline__ void row_interval(int64_t i, const MaskArgs& m, int64_t& lo,
                                                      int64_t& hi) {
  lo = 0;
  hi = static_cast<int64_t>(m.Skv) - 1;
  if (MASK == kMaskCausal) {
    hi = i < hi ? i : hi;
  } else if (MASK == kMaskSliding) {
    hi = i < hi ? i : hi;
    const int64_t a = i - m.window + 1;
    lo = a > 0 ? a : 0;
  } else if (MASK == kMaskOffset) {
    const int64_t b = i + m.offset;
    hi = b < hi ? b : hi;
  } else if (MASK == kMaskDocument || MASK == kMaskDocumentCausal) {
#ifdef __CUDA_ARCH__
    doc_interval(m, doc_floor(m.off_q, m.n_docs, i), i, MASK == kMaskDocumentCausal, lo, hi);
#else
    lo = 0;
    hi = -1;
#endif
  }
}

// Kept query interval [lo, hi] (inclusive, may be empty) of key j, for kernels whose
// rows are keys (the backward's dK/dV): keep(i, j) holds for i < Sq exactly when
// lo <= i <= hi.  Keys at or beyond Skv keep nothing.
template <int MASK>
__device__ __forceinline__ void key_interval(int64_t j, const MaskArgs& m, int Sq, int64_t& lo, int64_t& hi) {
  lo = 0;
  hi = static_cast<int64_t>(Sq) - 1;
  if (j >= m.Skv) {
    lo = 1;
    hi = 0;
    return;
  }
  if (MASK == kMaskCausal) {
    lo = j;
  } else if (MASK == kMaskSliding) {
    lo = j;
    const int64_t b = j + m.window - 1;
    hi = b < hi ? b : hi;
  } else if (MASK == kMaskOffset) {
    const int64_t a = j - m.offset;
    lo = a > 0 ? a : 0;
  } else if (MASK == kMaskDocument || MASK == kMaskDocumentCausal) {
    const int d = doc_floor(m.off_kv, m.n_docs, j);
    if (d < 0 || d >= m.n_docs) {
      lo = 1;
      hi = 0;
      return;
    }
    const int64_t a = __ldg(m.off_q + d), e = static_cast<int64_t>(__ldg(m.off_q + d + 1)) - 1;
    lo = a > 0 ? a : 0;
    hi = e < hi ? e : hi;
    if (MASK == kMaskDocumentCausal) lo = j > lo ? j : lo;
  }
}

// Key-tile range [t_lo, t_hi) that rows [q0, q1) (q1 exclusive, already clipped to Sq)
// must visit; empty (t_lo == t_hi == 0) when no key of these rows is kept.
template <int MASK>
__host__ __device__ __forceinline__ void tile_range(int q0, int q1, int BN, const MaskArgs& m,
                                                    int& t_lo, int& t_hi) {
  int64_t lo_first, hi_first, lo_last, hi_last;
  row_interval<MASK>(q0, m, lo_first, hi_first);
  row_interval<MASK>(q1 - 1, m, lo_last, hi_last);
  const int64_t jlo = lo_first;  // a() is non-decreasing
  const int64_t jhi = hi_last;   // b() is non-decreasing
  if (q1 <= q0 || jhi < jlo || jhi < 0) {
    t_lo = t_hi = 0;
    return;
  }
  t_lo = static_cast<int>(jlo / BN);
  t_hi = static_cast<int>(jhi / BN) + 1;
}

// FULL or PARTIAL for a key tile [k0, k0 + BN) inside the visited range.
template <int MASK>
__host__ __device__ __forceinline__ int tile_class(int q0, int q1, int k0, int BN, const MaskArgs& m) {
  const int64_t k1 = static_cast<int64_t>(k0) + BN;
  if (k1 > m.Skv) return kTilePartial;
  if (MASK == kMaskNone) return kTileFull;
  int64_t lo_first, hi_first, lo_last, hi_last;
  row_interval<MASK>(q0, m, lo_first, hi_first);
  row_interval<MASK>(q1 - 1, m, lo_last, hi_last);
  return (lo_last <= k0 && k1 - 1 <= hi_first) ? kTileFull : kTilePartial;
}

// Column interval [c_lo, c_hi] (relative to k0) of the kept keys [lo, hi] of one row.
__host__ __device__ __forceinline__ void col_interval_of(int64_t lo, int64_t hi, int k0, int& c_lo, int& c_hi) {
  lo -= k0;
  hi -= k0;
  // clamp to a range that fits in int and keeps "lo > hi" meaning empty
  c_lo = static_cast<int>(lo < -1 ? -1 : (lo > 1 << 20 ? 1 << 20 : lo));
  c_hi = static_cast<int>(hi < -1 ? -1 : (hi > 1 << 20 ? 1 << 20 : hi));
  if (lo > hi) {
    c_lo = 1;
    c_hi = 0;
  }
}

// Column interval [c_lo, c_hi] (relative to k0) kept in row i of a key tile at k0.
template <int MASK>
__host__ __device__ __forceinline__ void col_interval(int64_t i, int k0, const MaskArgs& m, int& c_lo,
                                                      int& c_hi) {
  int64_t lo, hi;
  row_interval<MASK>(i, m, lo, hi);
  col_interval_of(lo, hi, k0, c_lo, c_hi);
}

// FULL or PARTIAL for a key tile [k0, k0 + BN) from the kept intervals of the tile's
// first row (hi_first) and last row (lo_last), as tile_class computes them.
__host__ __device__ __forceinline__ int tile_class_of(int64_t lo_last, int64_t hi_first, int k0, int BN, int Skv) {
  const int64_t k1 = static_cast<int64_t>(k0) + BN;
  if (k1 > Skv) return kTilePartial;
  return (lo_last <= k0 && k1 - 1 <= hi_first) ? kTileFull : kTilePartial;
}

}  // namespace flexattn
