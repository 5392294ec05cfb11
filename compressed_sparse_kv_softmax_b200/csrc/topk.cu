// Exact top-k selection over lightning-indexer scores.
//
// The lightning indexer forwards the k most relevant CSA entries (512 for
// V4-Flash, 1,024 for V4-Pro; «Chinas KI-Unabhaengigkeit?: Bei Deepseek V4
// haben kleine Aenderungen grosse Wirkung», "Komprimierte Erinnerung fuer
// laengere Kontexte").  Selection here is exact: the k largest scores of the
// row's visible entries, ties to the lower entry index, written in ascending
// entry order, -1 / -inf padding when fewer than k are visible.  Scores are
// compared through an order-preserving uint32 key.
//
// Two kernels:
//  * topk_rows_kernel - one CTA per row: a 4-pass 8-bit radix select finds
//    the k-th largest key and how many equal keys to take, then an ordered
//    compaction in index order writes the result.  Used after the generic
//    scoring kernel and as the fall-back for pathological rows.
//  * topk_select_kernel - several CTAs per row, each owning a contiguous
//    slice of the row, after the tensor-core scoring kernel has built a
//    histogram of the top 12 key bits:
//      1. every CTA finds the bucket b* holding the k-th largest key, counts
//         its slice's entries above b* and appends the entries inside b*
//         (candidates) to the row's list;
//      2. the row's CTAs meet once at a bounded barrier;
//      3. every CTA reads the whole candidate list (a few thousand entries)
//         and resolves the exact k-th key and the ties to take, so all of
//         them hold the same decision; per-slice counts give each CTA the
//         offset of its slice in the output;
//      4. every CTA writes its slice's selected entries in index order, so
//         the output comes out ascending without a sort.
#include <climits>

#include "cskv_internal.cuh"
#include "topk_common.cuh"

namespace cskv {

namespace {

// exclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024);
// returns the block total in *total
__device__ __forceinline__ int block_exclusive_scan(int x, int *scratch, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? scratch[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < nw) scratch[lane] = wi - w;     // exclusive warp offsets
    if (lane == 31) scratch[32] = wi;          // total
  }
  __syncthreads();
  const int res = scratch[warp] + incl - x;
  *total = scratch[32];
  __syncthreads();
  return res;
}

// Exclusive prefix sum over the block with one block barrier: a warp scan,
// then each thread adds the totals of the warps before its own (read from
// `wsum`).  A following call must be separated from this one by a barrier.
__device__ __forceinline__ int block_exclusive_scan1(int x, int *wsum, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int before = incl - x, tot = 0;
  for (int w = 0; w < nw; ++w) {
    const int t = wsum[w];
    before += w < warp ? t : 0;
    tot += t;
  }
  *total = tot;
  return before;
}

// Bins are counts of keys sharing a digit; this finds the bin holding the
// `target`-th largest key: scanning bins from the top (bin nbins-1 down), the
// first bin at which the running count reaches `target`.  Thread t owns
// `per` consecutive bins from the top; a block-wide prefix sum of the owners'
// totals locates the owner, which walks its own bins.  Results land in
// *out_bin and *out_above (count of keys in higher bins); every thread must
// call it, and it ends with a block barrier.
template <typename Bins>
__device__ void find_threshold_bin(const Bins &bins, int nbins, int target, int *scan_scratch,
                                   int *out_bin, int *out_above) {
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  const int top = nbins - 1 - (int)threadIdx.x * per;
  int lsum = 0;
  for (int i = 0; i < per; ++i)
    if (top - i >= 0) lsum += (int)bins(top - i);
  int total;
  const int before = block_exclusive_scan(lsum, scan_scratch, &total);
  if (before < target && before + lsum >= target) {
    int cum = before;
    for (int i = 0; i < per && top - i >= 0; ++i) {
      const int c = (int)bins(top - i);
      if (cum + c >= target) {
        *out_bin = top - i;
        *out_above = cum;
        break;
      }
      cum += c;
    }
  }
  __syncthreads();
}

// Same search with two block barriers: thread t owns `per` consecutive bins
// from the top (nbins = blockDim.x * per), a warp scan gives the counts
// inside a warp, shared memory the counts of the warps above.
template <typename Bins>
__device__ void find_threshold_bin2(const Bins &bins, int nbins, int target, int *wsum,
                                    int *out_bin, int *out_above) {
  const int per = nbins / blockDim.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int top = nbins - 1 - (int)threadIdx.x * per;
  int lsum = 0;
  for (int i = 0; i < per; ++i) lsum += (int)bins(top - i);
  int incl = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int before = incl - lsum;
  for (int w = 0; w < warp; ++w) before += wsum[w];
  if (before < target && before + lsum >= target) {
    int cum = before;
    for (int i = 0; i < per; ++i) {
      const int c = (int)bins(top - i);
      if (cum + c >= target) {
        *out_bin = top - i;
        *out_above = cum;
        break;
      }
      cum += c;
    }
  }
  __syncthreads();
}

// A row with a NaN score (a scoring CTA that gave up marks its entries so,
// and NaN inputs give NaN scores) has no ranking: every slot of the row
// reads -1 / NaN and the event is recorded.
__device__ void write_failed_row(int k, int32_t *__restrict__ oi, float *__restrict__ os,
                                 unsigned int *status) {
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    oi[i] = -1;
    if (os) os[i] = __int_as_float(0x7fffffff);
  }
  if (threadIdx.x == 0) record_event(status, CSKV_DEV_ROW_FAILED);
}

// Whole-row exact top-k by one CTA (any blockDim multiple of 32).
// (not inlined: inside the multi-CTA selection it is the rarely taken
// fall-back, kept out of the hot code's instruction stream)
__device__ __noinline__ void topk_row_single_cta(const float *__restrict__ s, long long n, int k,
                                    int32_t *__restrict__ oi, float *__restrict__ os,
                                    unsigned int *status) {
  __shared__ int hist[256];
  __shared__ int scan_scratch[33];
  const int tid = threadIdx.x;
  uint32_t thr = 0;
  int take_eq = 0;
  const bool all = n <= k;
  if (all) {
    bool nan = false;
    for (long long j = tid; j < n; j += blockDim.x) nan |= isnan(s[j]);
    if (__syncthreads_or(nan)) {
      write_failed_row(k, oi, os, status);
      return;
    }
  } else {
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      bool nan = false;
      for (long long j = tid; j < n; j += blockDim.x) {
        const float sv = s[j];
        nan |= isnan(sv);
        const uint32_t key = score_key(sv);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
      }
      if (__syncthreads_or(nan)) {      // (only the first pass can see one)
        write_failed_row(k, oi, os, status);
        return;
      }
      __shared__ int s_bin, s_above;
      if (tid == 0) { s_bin = 0; s_above = 0; }
      find_threshold_bin([&](int i) { return hist[i]; }, 256, remaining, scan_scratch, &s_bin,
                         &s_above);
      prefix = prefix | ((uint32_t)s_bin << shift);
      remaining = remaining - s_above;
      mask |= 255u << shift;
      __syncthreads();
    }
    thr = prefix;
    take_eq = remaining;
  }
  int base_gt = 0, base_eq = 0;
  for (long long j0 = 0; j0 < n; j0 += blockDim.x) {
    const long long j = j0 + tid;
    int gt = 0, eq = 0;
    float sv = 0.f;
    if (j < n) {
      sv = s[j];
      const uint32_t key = score_key(sv);
      gt = all || key > thr;
      eq = !all && key == thr;
    }
    int tot_gt, tot_eq;
    const int pre_gt = block_exclusive_scan(gt, scan_scratch, &tot_gt);
    const int pre_eq = block_exclusive_scan(eq, scan_scratch, &tot_eq);
    const int eq_rank = base_eq + pre_eq;
    const bool take = gt || (eq && eq_rank < take_eq);
    const int slot = base_gt + pre_gt + min(eq_rank, take_eq);
    if (take && slot < k) {
      oi[slot] = (int32_t)j;
      if (os) os[slot] = sv;
    }
    base_gt += tot_gt;
    base_eq += tot_eq;
  }
  const int taken = all ? (int)n : k;
  for (int i = taken + tid; i < k; i += blockDim.x) {
    oi[i] = -1;
    if (os) os[i] = -__int_as_float(0x7f800000);
  }
}

__device__ __forceinline__ long long visible(const int64_t *q_pos, int row, int stride,
                                             long long max_entries) {
  long long n = (q_pos[row] + 1) / stride;
  if (n > max_entries) n = max_entries;
  return n < 0 ? 0 : n;
}

// Checked build: a row's visible entries (q_pos + 1) / stride within the
// host bound max_entries, which the scoring and the selection both stop at
// (one thread of the row's first CTA; nothing in the regular build)
__device__ __forceinline__ void check_visible(const int64_t *q_pos, int row, int stride,
                                              long long max_entries, unsigned int *status) {
  if constexpr (kChecked) {
    if (threadIdx.x == 0 && (q_pos[row] + 1) / stride > max_entries)
      record_event(status, CSKV_DEV_BOUNDS);
  }
}

// Ascending bitonic sort of v[0..m) in shared memory, m a power of two.
template <typename T>
__device__ void bitonic_sort_smem(T *v, int m) {
  for (int size = 2; size <= m; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (m >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const T a = v[lo], b = v[hi];
        if ((a > b) == up) { v[lo] = b; v[hi] = a; }
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ uint64_t pack_entry(long long j, uint32_t key) {
  return ((uint64_t)(uint32_t)j << 32) | key;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

constexpr int kSelThreads = 512;
constexpr int kSelPer = 8;                        // consecutive entries per thread and pass
constexpr int kSelChunk = kSelThreads * kSelPer;  // entries per CTA and pass
constexpr int kMaxK = 4096;
constexpr int kTieCap = kTopkBins;                // exact ties held in the histogram's space

struct SelSmem {
  uint32_t hist[kTopkBins];   // row histogram, then refine bins, then the tie list
  uint64_t cand[kCandCap];    // (index << 32) | key of every candidate of the row
  int cnt[kMaxSplits];        // selected entries per slice of the row
  int scan[33];
  int bstar, above, thr_bin, take, n_eq, state, n_cand, base, total, wins;
  unsigned solo_cand;         // candidate count when one CTA owns the row
  uint32_t tie_cut, thr_full;
};

// scores j0 .. j0+7 of a row (entries at or beyond j_hi read as -inf)
__device__ __forceinline__ void load8(const float *__restrict__ s, long long j0, long long j_hi,
                                      float (&v)[kSelPer]) {
  if (j0 + kSelPer <= j_hi) {
    const float4 a = __ldcg(reinterpret_cast<const float4 *>(s + j0));
    const float4 b = __ldcg(reinterpret_cast<const float4 *>(s + j0) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < kSelPer; ++e)
      v[e] = j0 + e < j_hi ? __ldcg(s + j0 + e) : -__int_as_float(0x7f800000);
  }
}

}  // namespace

__global__ void __launch_bounds__(1024)
topk_rows_kernel(const float *__restrict__ scores, long long ld, const int64_t *__restrict__ q_pos,
                 int stride, long long max_entries, int k, int32_t *__restrict__ out_idx,
                 float *__restrict__ out_score, unsigned int *status) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  const long long n = visible(q_pos, row, stride, max_entries);
  check_visible(q_pos, row, stride, max_entries, status);
  topk_row_single_cta(scores + (long long)row * ld, n, k, out_idx + (long long)row * k,
                      out_score ? out_score + (long long)row * k : nullptr, status);
}

// kDeep: slices longer than one pass (a CTA per row of a long chunk); the
// next two passes' scores are then requested while one is counted
template <bool kDeep>
__global__ void __launch_bounds__(kSelThreads, 1)
topk_select_kernel(const IndexerWs w, const int64_t *__restrict__ q_pos, int stride,
                   long long max_entries, int k, int32_t *__restrict__ out_idx,
                   float *__restrict__ out_score, unsigned int *status, uint32_t spin_limit) {
  extern __shared__ __align__(16) uint8_t sel_smem_raw[];
  SelSmem &sm = *reinterpret_cast<SelSmem *>(sel_smem_raw);
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nsplit = gridDim.x, me = blockIdx.x;
  const float *s = w.scores + (long long)row * w.ld;
  int32_t *oi = out_idx + (long long)row * k;
  float *os = out_score ? out_score + (long long)row * k : nullptr;
  // slices follow the host bound, so this CTA's first scores, the histogram
  // and the row's position are all requested before any of them is used
  const long long per = ((max_entries + nsplit - 1) / nsplit + kSelPer - 1) / kSelPer * kSelPer;
  const long long j_lo = (long long)me * per;
  const long long j_cap = j_lo + per < max_entries ? j_lo + per : max_entries;
  const long long pos = q_pos[row];
  constexpr int kHPer = kTopkBins / kSelThreads;
  uint32_t hv[kHPer];
  {
    const uint32_t *hrow = w.hist + (size_t)row * kTopkBins;
#pragma unroll
    for (int e = 0; e < kHPer; ++e) hv[e] = __ldcg(hrow + tid + e * kSelThreads);
  }
  float keep[kSelPer];                 // the first pass's scores
  load8(s, j_lo + (long long)tid * kSelPer, j_cap, keep);
  long long n = (pos + 1) / stride;
  if (n > max_entries) n = max_entries;
  if (n < 0) n = 0;
  if (me == 0) check_visible(q_pos, row, stride, max_entries, status);

  // the row's histogram is cleared for the next scoring call once every CTA
  // of the row has read it (here, or past the row barrier below)
  uint4 *hclear = reinterpret_cast<uint4 *>(w.hist + (size_t)row * kTopkBins);
  if (n <= k) {            // every visible entry is selected, already in order
    if (me == 0) {
      bool nan = false;
      for (long long i = tid; i < n; i += blockDim.x) nan |= isnan(s[i]);
      if (__syncthreads_or(nan)) {
        write_failed_row(k, oi, os, status);
      } else {
        for (int i = tid; i < k; i += blockDim.x) {
          oi[i] = i < n ? i : -1;
          if (os) os[i] = i < n ? s[i] : -__int_as_float(0x7f800000);
        }
      }
      // (the histogram is not read on this path)
      for (int i = tid; i < kTopkBins / 4; i += blockDim.x) hclear[i] = make_uint4(0, 0, 0, 0);
    }
    return;
  }

  // ---- 0. a histogram with counts in the NaN / infinity bins (a scoring CTA
  // gave up, or the inputs hold NaN): the row's first CTA checks every score
  // in the whole-row path; the last CTA to pass here clears the histogram
  {
    bool extreme = false;
#pragma unroll
    for (int e = 0; e < kHPer; ++e) extreme |= hv[e] != 0u && topk_extreme_bin(tid + e * kSelThreads);
    if (__syncthreads_or(extreme)) {
      if (tid == 0) sm.state = atomicAdd(&w.ctr[(size_t)row * 4 + 1], 1u) == (uint32_t)nsplit - 1;
      __syncthreads();
      if (sm.state)
        for (int i = tid; i < kTopkBins / 4; i += blockDim.x) hclear[i] = make_uint4(0, 0, 0, 0);
      if (me == 0) topk_row_single_cta(s, n, k, oi, os, status);
      return;
    }
  }

  // ---- 1. threshold bucket b*, this slice's winners and candidates
  if (tid == 0) { sm.bstar = 0; sm.above = -1; sm.wins = 0; sm.solo_cand = 0u; }
#pragma unroll
  for (int e = 0; e < kHPer; ++e) sm.hist[tid + e * kSelThreads] = hv[e];
  __syncthreads();
  find_threshold_bin2([&](int i) { return sm.hist[i]; }, kTopkBins, k, sm.scan, &sm.bstar,
                      &sm.above);
  const uint32_t bstar = (uint32_t)sm.bstar;
  const int above = sm.above;

  const long long j_hi = j_lo + per < n ? j_lo + per : n;
  uint32_t *ctr = w.ctr + (size_t)row * 4;
  uint64_t *candrow = w.cand + (size_t)row * kCandCap;
  int wins = 0;
  float v[kSelPer], p1[kSelPer], p2[kSelPer];
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) v[e] = keep[e];
  if (kDeep) {
    if (j_lo + kSelChunk < j_hi) load8(s, j_lo + kSelChunk + (long long)tid * kSelPer, j_hi, p1);
    if (j_lo + 2 * kSelChunk < j_hi)
      load8(s, j_lo + 2 * kSelChunk + (long long)tid * kSelPer, j_hi, p2);
  }
  for (long long c0 = j_lo; c0 < j_hi; c0 += kSelChunk) {
    const long long j0 = c0 + (long long)tid * kSelPer;
    if (c0 != j_lo) {
      if (kDeep) {
#pragma unroll
        for (int e = 0; e < kSelPer; ++e) { v[e] = p1[e]; p1[e] = p2[e]; }
        if (c0 + 2 * kSelChunk < j_hi) load8(s, j0 + 2 * kSelChunk, j_hi, p2);
      } else {
        load8(s, j0, j_hi, v);
      }
    }
    int nc = 0;
    uint32_t cmask = 0;
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) {
      if (j0 + e < j_hi) {
        const uint32_t bkt = score_key(v[e]) >> kTopkShift;
        wins += bkt > bstar;
        if (bkt == bstar) { cmask |= 1u << e; ++nc; }
      }
    }
    // warp-aggregated append of the candidates
    int incl = nc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    uint32_t base = 0;
    // (a CTA that owns the whole row counts in shared memory: no L2 round
    // trip per pass)
    if (lane == 31 && incl)
      base = nsplit == 1 ? atomicAdd(&sm.solo_cand, (uint32_t)incl)
                         : atomicAdd(&ctr[0], (uint32_t)incl);
    base = __shfl_sync(0xffffffffu, base, 31);
    uint32_t p = base + (uint32_t)(incl - nc);
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) {
      if (cmask >> e & 1u) {
        if (p < (uint32_t)kCandCap) candrow[p] = pack_entry(j0 + e, score_key(v[e]));
        ++p;
      }
    }
  }
  wins = __reduce_add_sync(0xffffffffu, wins);
  if (lane == 0 && wins) atomicAdd(&sm.wins, wins);

  // ---- 2. row barrier: every slice's candidates and winner count are visible
  // (the block barrier orders the CTA's writes before thread 0's fence and
  // release; the acquiring load and the next block barrier order the reads)
  __syncthreads();
  if (tid == 0) {
    w.wins[(size_t)row * kMaxSplits + me] = (uint32_t)sm.wins;
    __threadfence();
    atomicAdd(&ctr[1], 1u);
    int state = 0;
    uint32_t spins = 0;
    while (ld_acquire_u32(&ctr[1]) < (uint32_t)nsplit) {
      if (++spins > spin_limit) {
        state = 1;
        record_event(status, CSKV_DEV_TOPK_BARRIER);
        break;
      }
      __nanosleep(64);
    }
    sm.state = state;
    sm.n_cand = nsplit == 1 ? (int)sm.solo_cand : (int)ld_acquire_u32(&ctr[0]);
  }
  __syncthreads();
  // every CTA of the row has read the histogram before arriving (a CTA that
  // gave up waiting selects from the scores alone and leaves the histogram:
  // a stale one costs the next call time, not correctness)
  if (me == 0 && sm.state == 0)
    for (int i = tid; i < kTopkBins / 4; i += blockDim.x) hclear[i] = make_uint4(0, 0, 0, 0);
  const int n_cand = sm.n_cand;
  const int r = k - above;             // candidates still to take
  bool fallback = sm.state != 0 || above < 0 || above >= k || r < 1 || r > n_cand ||
                  n_cand > kCandCap;

  // ---- 3. the exact k-th key among the candidates (same result in every CTA)
  uint32_t thr = 0, tie_cut = 0xffffffffu;
  // per-slice winner counts, requested now and used after the refinement
  const int wins_c = tid < nsplit ? (int)__ldcg(w.wins + (size_t)row * kMaxSplits + tid) : 0;
  if (!fallback) {
    {
      constexpr int kC = kCandCap / kSelThreads;
      uint64_t v[kC];
#pragma unroll
      for (int e = 0; e < kC; ++e) {
        const int i = tid + e * kSelThreads;
        v[e] = i < n_cand ? __ldcg(candrow + i) : 0ull;
      }
      // the next histogram's bins and the per-slice counts start meanwhile
      for (int i = tid; i < kTopkBins; i += blockDim.x) sm.hist[i] = 0;
      if (tid < nsplit) sm.cnt[tid] = wins_c;
      if (tid == 0) { sm.thr_bin = 0; sm.take = 0; sm.n_eq = 0; }
#pragma unroll
      for (int e = 0; e < kC; ++e) {
        const int i = tid + e * kSelThreads;
        if (i < n_cand) sm.cand[i] = v[e];
      }
    }
    __syncthreads();
    // radix select of the r-th largest candidate key (all candidates share
    // the bucket bits): bits 19..8 in one 4096-bin pass, then the few
    // candidates left in the chosen bin by one warp (up to 32 of them, ties
    // included) or by a 256-bin pass over bits 7..0
    uint32_t prefix = bstar << kTopkShift;
    int remaining = r;
    for (int i = tid; i < n_cand; i += blockDim.x)
      atomicAdd(&sm.hist[((uint32_t)sm.cand[i] >> 8) & 4095u], 1u);
    __syncthreads();
    find_threshold_bin2([&](int i) { return sm.hist[i]; }, kTopkBins, remaining, sm.scan,
                        &sm.thr_bin, &sm.take);
    prefix |= (uint32_t)sm.thr_bin << 8;
    remaining -= sm.take;
    const int in_bin = (int)sm.hist[sm.thr_bin];
    __syncthreads();
    if (in_bin <= 32) {
      uint64_t *lst = reinterpret_cast<uint64_t *>(sm.hist);   // the bin's candidates
      for (int i = tid; i < n_cand; i += blockDim.x) {
        const uint64_t c = sm.cand[i];
        if (((uint32_t)c >> 8) == (prefix >> 8)) lst[atomicAdd(&sm.n_eq, 1)] = c;
      }
      __syncthreads();
      if (warp == 0) {
        const int cnt = sm.n_eq;
        const uint64_t c = lane < cnt ? lst[lane] : 0ull;
        const uint32_t key = (uint32_t)c, idx = (uint32_t)(c >> 32);
        int gt = 0, ge = 0;
        for (int m = 0; m < cnt; ++m) {
          const uint32_t o = __shfl_sync(0xffffffffu, key, m);
          gt += o > key;
          ge += o >= key;
        }
        // the key whose rank range covers `remaining` (equal keys agree)
        const unsigned hit = __ballot_sync(0xffffffffu, lane < cnt && gt < remaining && remaining <= ge);
        const int src = hit ? __ffs(hit) - 1 : 0;
        const uint32_t tkey = __shfl_sync(0xffffffffu, key, src);
        const int take = remaining - __shfl_sync(0xffffffffu, gt, src);
        // exact ties: the take-th smallest index among the keys equal to tkey
        const bool eq = lane < cnt && key == tkey;
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        int rank = 0;
        for (int m = 0; m < cnt; ++m) {
          const uint32_t oi = __shfl_sync(0xffffffffu, idx, m);
          rank += (eqm >> m & 1u) && oi < idx;
        }
        const unsigned cut = __ballot_sync(0xffffffffu, eq && rank == take - 1);
        const uint32_t cut_idx = __shfl_sync(0xffffffffu, idx, cut ? __ffs(cut) - 1 : 0);
        if (lane == 0) {
          sm.thr_full = tkey;
          sm.take = hit ? take : 0;       // 0: no rank matched -> fall-back
          // all equal keys taken: no cut; otherwise the take-th smallest index
          sm.tie_cut = (__popc(eqm) > take && cut) ? cut_idx : 0xffffffffu;
        }
      }
      __syncthreads();
      thr = sm.thr_full;
      tie_cut = sm.tie_cut;
      if (sm.take < 1) fallback = true;
    } else {
      for (int i = tid; i < 256; i += blockDim.x) sm.hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n_cand; i += blockDim.x) {
        const uint32_t key = (uint32_t)sm.cand[i];
        if ((key >> 8) == (prefix >> 8)) atomicAdd(&sm.hist[key & 255u], 1u);
      }
      __syncthreads();
      find_threshold_bin([&](int i) { return sm.hist[i]; }, 256, remaining, sm.scan, &sm.thr_bin,
                         &sm.take);
      prefix |= (uint32_t)sm.thr_bin;
      remaining -= sm.take;
      thr = prefix;
      const int take_eq = remaining;     // keys equal to thr to take, lowest indices first
      // exact ties: when more keys equal thr than are taken, the cut is the
      // take_eq-th smallest of their indices
      if (tid == 0) sm.n_eq = 0;
      __syncthreads();
      uint32_t *eqv = sm.hist;
      for (int i = tid; i < n_cand; i += blockDim.x) {
        const uint64_t c = sm.cand[i];
        if ((uint32_t)c == thr) {
          const int p = atomicAdd(&sm.n_eq, 1);
          if (p < kTieCap) eqv[p] = (uint32_t)(c >> 32);
        }
      }
      __syncthreads();
      const int n_eq = sm.n_eq;
      if (take_eq < 1 || n_eq < take_eq || n_eq > kTieCap) {
        fallback = true;
      } else if (n_eq > take_eq) {
        int m = 1;
        while (m < n_eq) m <<= 1;
        for (int i = n_eq + tid; i < m; i += blockDim.x) eqv[i] = 0xffffffffu;
        __syncthreads();
        bitonic_sort_smem(eqv, m);
        tie_cut = eqv[take_eq - 1];
      }
    }
  }

  // ---- per-slice counts of the selection, and this slice's output offset
  if (!fallback) {
    for (int i = tid; i < n_cand; i += blockDim.x) {
      const uint64_t c = sm.cand[i];
      const uint32_t key = (uint32_t)c, j = (uint32_t)(c >> 32);
      if (key > thr || (key == thr && j <= tie_cut)) atomicAdd(&sm.cnt[j / per], 1);
    }
    __syncthreads();
    if (warp == 0) {
      int tot = 0, before = 0;
      for (int c0 = 0; c0 < nsplit; c0 += 32) {
        const int c = c0 + lane;
        const int v = c < nsplit ? sm.cnt[c] : 0;
        tot += __reduce_add_sync(0xffffffffu, v);
        before += __reduce_add_sync(0xffffffffu, c < me ? v : 0);
      }
      if (lane == 0) { sm.total = tot; sm.base = before; }
    }
    __syncthreads();
    fallback = sm.total != k;
  }

  // ---- 4. this slice's selected entries, in index order, at its offset
  if (!fallback) {
    int base = sm.base;
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) v[e] = keep[e];
    if (kDeep) {
      if (j_lo + kSelChunk < j_hi) load8(s, j_lo + kSelChunk + (long long)tid * kSelPer, j_hi, p1);
      if (j_lo + 2 * kSelChunk < j_hi)
        load8(s, j_lo + 2 * kSelChunk + (long long)tid * kSelPer, j_hi, p2);
    }
    for (long long c0 = j_lo; c0 < j_hi; c0 += kSelChunk) {
      const long long j0 = c0 + (long long)tid * kSelPer;
      if (c0 != j_lo) {
        if (kDeep) {
#pragma unroll
          for (int e = 0; e < kSelPer; ++e) { v[e] = p1[e]; p1[e] = p2[e]; }
          if (c0 + 2 * kSelChunk < j_hi) load8(s, j0 + 2 * kSelChunk, j_hi, p2);
        } else {
          load8(s, j0, j_hi, v);
        }
      }
      uint32_t fl = 0;
#pragma unroll
      for (int e = 0; e < kSelPer; ++e) {
        const uint32_t key = score_key(v[e]);
        const bool take = j0 + e < j_hi &&
                          (key > thr || (key == thr && (uint32_t)(j0 + e) <= tie_cut));
        fl |= (uint32_t)take << e;
      }
      int tot;
      if (c0 != j_lo) __syncthreads();      // the previous pass has read sm.scan
      int p = base + block_exclusive_scan1(__popc(fl), sm.scan, &tot);
#pragma unroll
      for (int e = 0; e < kSelPer; ++e) {
        if ((fl >> e & 1u) && p < k) {
          oi[p] = (int32_t)(j0 + e);
          if (os) os[p] = v[e];
        }
        p += fl >> e & 1u;
      }
      base += tot;
    }
    return;
  }
  // inconsistent histogram or candidate overflow (never expected with the
  // scoring kernel's histogram): the row's first CTA selects the whole row.
  // A CTA that gave up at the meeting point cannot know whether the others
  // write their slices, so it selects the whole row too (every writer of a
  // slot writes the same exact value).
  if (me == 0 || sm.state != 0) topk_row_single_cta(s, n, k, oi, os, status);
}

void launch_topk_rows(const float *scores, long long ld, const int64_t *q_pos, int stride,
                      long long max_entries, int k, int rows, int32_t *out_idx,
                      float *out_score, unsigned int *status, cudaStream_t st) {
  launch_pdl(topk_rows_kernel, dim3(rows), dim3(1024), 0, st, scores, ld, q_pos, stride,
             max_entries, k, out_idx, out_score, status);
}

int launch_topk_select(const IndexerWs &w, const int64_t *q_pos, int stride,
                       long long max_entries, int k, int rows, int32_t *out_idx,
                       float *out_score, unsigned int *status, cudaStream_t st) {
  if (k > kMaxK) return CSKV_ERR_UNSUPPORTED;
  const size_t smem = sizeof(SelSmem);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // one pass of kSelChunk scores per CTA; the CTAs of a row wait for one
  // another once, so a row's CTAs must all be resident at the same time:
  // at most one CTA per SM over the whole grid, else one CTA per row
  long long splits = (max_entries + kSelChunk - 1) / kSelChunk;
  const long long cap = sms / rows;
  if (splits > cap) splits = cap;
  if (splits > kMaxSplits) splits = kMaxSplits;
  if (splits < 1) splits = 1;
  const long long per = ((max_entries + splits - 1) / splits + kSelPer - 1) / kSelPer * kSelPer;
  auto kernel = per > kSelChunk ? topk_select_kernel<true> : topk_select_kernel<false>;
  if (!ensure_dynamic_smem(kernel, smem)) return CSKV_ERR_UNSUPPORTED;
  launch_pdl(kernel, dim3((unsigned)splits, (unsigned)rows), dim3(kSelThreads), smem, st, w,
             q_pos, stride, max_entries, k, out_idx, out_score, status, topk_barrier_spins());
  return cudaGetLastError() == cudaSuccess ? CSKV_OK : CSKV_ERR_CUDA;
}

}  // namespace cskv
