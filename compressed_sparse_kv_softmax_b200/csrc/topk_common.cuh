// Shared constants of the score histogram the indexer builds for the top-k.
#pragma once

#include <stdint.h>

namespace cskv {

// Histogram over the top 12 bits of the order-preserving score key (sign,
// exponent and 3 mantissa bits): 4096 buckets, each 1/8 of an octave wide.
constexpr int kTopkBins = 4096;
constexpr int kTopkShift = 20;
// Candidates (entries inside the threshold bucket) kept per row; rows with
// more fall back to the single-CTA selection of the whole row.
constexpr int kCandCap = 8192;
// Most CTAs that share one row in the multi-CTA selection.
constexpr int kMaxSplits = 256;

// Score-key bins that hold +inf or positive NaN (keys 0xff800000 and up), and
// -inf or negative NaN (keys up to 0x007fffff).  A scoring CTA that gave up
// counts its unscored entries (stored as NaN) in kTopkNanBin; the selection
// sends a row whose histogram has anything in these bins through the path
// that checks every score.
constexpr int kTopkNanBin = kTopkBins - 1;
__host__ __device__ constexpr bool topk_extreme_bin(int bin) { return bin < 8 || bin >= kTopkBins - 8; }

// Indexer workspace layout, one section after another, each 256-byte aligned:
//   scores   rows x ld fp32
//   hist     rows x kTopkBins u32  score histogram: built by the scoring kernel,
//                                  cleared by the selection once read (it only
//                                  guides the selection: a stale one costs time,
//                                  not correctness)
//   ctr      rows x 4 u32          candidate count, meeting-point arrivals
//                                  (cleared by the scoring kernel)
//   wins     rows x kMaxSplits u32 entries above the threshold bucket per CTA
//   cand     rows x kCandCap u64   entries inside the threshold bucket, (index << 32) | key
struct IndexerWs {
  float *scores;
  uint32_t *hist;
  uint32_t *ctr;
  uint32_t *wins;
  uint64_t *cand;
  long long ld;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline IndexerWs indexer_ws_layout(void *base, long long rows, long long max_entries, int k,
                                   size_t *total) {
  (void)k;
  IndexerWs w{};
  w.ld = (max_entries + 3) & ~3LL;
  if (w.ld < 4) w.ld = 4;
  uint8_t *p = static_cast<uint8_t *>(base);
  size_t off = 0;
  w.scores = reinterpret_cast<float *>(p + off);      off = align256(off + rows * w.ld * 4);
  w.hist = reinterpret_cast<uint32_t *>(p + off);     off = align256(off + rows * kTopkBins * 4);
  w.ctr = reinterpret_cast<uint32_t *>(p + off);      off = align256(off + rows * 16);
  w.wins = reinterpret_cast<uint32_t *>(p + off);     off = align256(off + rows * (size_t)kMaxSplits * 4);
  w.cand = reinterpret_cast<uint64_t *>(p + off);     off = align256(off + rows * (size_t)kCandCap * 8);
  if (total) *total = off;
  return w;
}

}  // namespace cskv
