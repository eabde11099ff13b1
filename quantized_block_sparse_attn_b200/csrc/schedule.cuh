// K-tile schedule of one 128-row query tile under the band / causal masks.
//
// Mask semantics (npu_fusion_attention guide, "昇腾 NPU 融合注意力算子详解与迁移指南",
// §4.3): sparse_mode 0 keeps key j for query i when i - pre_tokens <= j <= i +
// next_tokens; mode 2 (causal, top-left vertex) keeps j <= i; mode 3 (causal,
// bottom-right vertex) keeps j <= i + (S_kv - S_q).  Indices are 0-based inside one
// sequence (per sequence for TND).  The same function runs on the host (schedule
// export, launch sizing) and on the device (each CTA's K loop), so the two agree
// bit for bit.
#pragma once

#include <cstdint>

namespace qbsa {

constexpr int kTile = 128;

struct TileRange {
  int kt_begin;    // first K tile to visit
  int kt_end;      // one past the last K tile to visit (== kt_begin: visit nothing)
  int full_begin;  // K tiles in [full_begin, full_end) need no element mask
  int full_end;
};

struct Band {
  int64_t lo_off;  // row i keeps j >= i - lo_off
  int64_t hi_off;  // row i keeps j <= i + hi_off
};

__host__ __device__ inline Band band_of(int sparse_mode, int64_t pre_tokens, int64_t next_tokens, int64_t sq,
                                        int64_t skv) {
  Band b;
  if (sparse_mode == 2) {
    b.lo_off = (int64_t)1 << 40;
    b.hi_off = 0;
  } else if (sparse_mode == 3) {
    b.lo_off = (int64_t)1 << 40;
    b.hi_off = skv - sq;
  } else {
    b.lo_off = pre_tokens;
    b.hi_off = next_tokens;
  }
  return b;
}

__host__ __device__ inline int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }
__host__ __device__ inline int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// Tiles of query tile qt (rows [128 qt, min(sq, 128 qt + 128))) over keys [0, skv).
__host__ __device__ inline TileRange tile_range(int qt, int64_t sq, int64_t skv, Band band) {
  TileRange r{0, 0, 0, 0};
  const int64_t q0 = (int64_t)qt * kTile;
  const int64_t q1 = min64(sq, q0 + kTile);  // exclusive
  if (q1 <= q0 || skv <= 0) return r;
  // rows with a non-empty clamped interval [max(0, i - lo), min(skv - 1, i + hi)]
  if (band.lo_off + band.hi_off < 0) return r;
  const int64_t i_first = max64(q0, -band.hi_off);
  const int64_t i_last = min64(q1 - 1, skv - 1 + band.lo_off);
  if (i_first > i_last) return r;
  const int64_t j_lo = max64(0, i_first - band.lo_off);
  const int64_t j_hi = min64(skv - 1, i_last + band.hi_off);
  r.kt_begin = (int)(j_lo / kTile);
  r.kt_end = (int)(j_hi / kTile) + 1;
  // full tiles: every row of the tile keeps every column of the tile, and the
  // tile lies inside [0, skv).  Needs all rows non-empty: rows q0 and q1-1 bound it.
  const int64_t lo_last = (q1 - 1) - band.lo_off;   // lower bound of the last row
  const int64_t hi_first = q0 + band.hi_off;        // upper bound of the first row
  int64_t f_lo = max64(0, lo_last);                 // first column kept by all rows
  int64_t f_hi = min64(skv - 1, hi_first);          // last column kept by all rows
  if (f_lo > f_hi || q0 < -band.hi_off || (q1 - 1) > skv - 1 + band.lo_off) {
    r.full_begin = r.full_end = r.kt_begin;
  } else {
    int fb = (int)((f_lo + kTile - 1) / kTile);
    int fe = (int)((f_hi + 1) / kTile);  // tiles whose last column <= f_hi
    if (fb < r.kt_begin) fb = r.kt_begin;
    if (fe > r.kt_end) fe = r.kt_end;
    if (fe < fb) fe = fb;
    r.full_begin = fb;
    r.full_end = fe;
  }
  return r;
}

}  // namespace qbsa
