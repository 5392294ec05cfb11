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
//  * topk_select_kernel - several CTAs per row, after the tensor-core scoring
//    kernel has built a histogram of the top 12 key bits:
//      1. every CTA finds the bucket b* holding the k-th largest key;
//      2. every CTA scans its slice of the row, appending entries above b*
//         (sure winners) and entries in b* (candidates);
//      3. the last CTA to finish (atomic ticket, nobody waits) selects the
//         missing candidates by the low 20 key bits, breaks exact ties by the
//         lower index, and sorts the k indices.
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

// Whole-row exact top-k by one CTA (any blockDim multiple of 32).
__device__ void topk_row_single_cta(const float *__restrict__ s, long long n, int k,
                                    int32_t *__restrict__ oi, float *__restrict__ os) {
  __shared__ int hist[256];
  __shared__ int scan_scratch[33];
  const int tid = threadIdx.x;
  uint32_t thr = 0;
  int take_eq = 0;
  const bool all = n <= k;
  if (!all) {
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      for (long long j = tid; j < n; j += blockDim.x) {
        const uint32_t key = score_key(s[j]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
      }
      __syncthreads();
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

// inverse of score_key
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

__device__ __forceinline__ uint64_t pack_entry(long long j, uint32_t key) {
  return ((uint64_t)(uint32_t)j << 32) | key;
}

constexpr int kSelThreads = 512;
constexpr int kCandSmem = kCandCap; // candidates the last CTA refines in shared memory
constexpr int kMaxK = 4096;
constexpr int kScanBatch = 8;       // scores a thread loads before processing any
// rows of up to this many entries are ordered through a bitmap plus word
// prefix counts, both held in the (by then unused) candidate buffer
constexpr int kBitmapWords = kCandSmem;                 // 8192 words x 2 arrays = 64 KB
constexpr long long kBitmapEntries = 32LL * kBitmapWords;

struct SelSmem {
  uint32_t hist[kTopkBins];         // row histogram, later refine histograms / tie list
  uint64_t cand[kCandSmem];         // (index << 32) | key
  uint64_t out[kMaxK];              // (index << 32) | key of the selection
  int scan[33];
  int bstar, above, is_last, thr2, take_eq, n_eq, n_gt, fallback, n_cand, n_sel;
};

}  // namespace

__global__ void __launch_bounds__(1024)
topk_rows_kernel(const float *__restrict__ scores, long long ld, const int64_t *__restrict__ q_pos,
                 int stride, long long max_entries, int k, int32_t *__restrict__ out_idx,
                 float *__restrict__ out_score) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  const long long n = visible(q_pos, row, stride, max_entries);
  topk_row_single_cta(scores + (long long)row * ld, n, k, out_idx + (long long)row * k,
                      out_score ? out_score + (long long)row * k : nullptr);
}

__global__ void __launch_bounds__(kSelThreads)
topk_select_kernel(const IndexerWs w, const int64_t *__restrict__ q_pos, int stride,
                   long long max_entries, int k, int32_t *__restrict__ out_idx,
                   float *__restrict__ out_score) {
  extern __shared__ __align__(16) uint8_t sel_smem_raw[];
  SelSmem &sm = *reinterpret_cast<SelSmem *>(sel_smem_raw);
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const long long n = visible(q_pos, row, stride, max_entries);
  const float *s = w.scores + (long long)row * w.ld;
  int32_t *oi = out_idx + (long long)row * k;
  float *os = out_score ? out_score + (long long)row * k : nullptr;

  if (n <= k) {            // every visible entry is selected, already in order
    if (blockIdx.x == 0) {
      for (int i = tid; i < k; i += blockDim.x) {
        oi[i] = i < n ? i : -1;
        if (os) os[i] = i < n ? s[i] : -__int_as_float(0x7f800000);
      }
    }
    return;
  }

  // 1. threshold bucket b*: the bucket holding the k-th largest key
  if (tid == 0) { sm.bstar = 0; sm.above = -1; }
  {
    const uint32_t *hrow = w.hist + (size_t)row * kTopkBins;
    constexpr int kPer = kTopkBins / kSelThreads;
    uint32_t v[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) v[e] = __ldcg(hrow + tid + e * kSelThreads);
#pragma unroll
    for (int e = 0; e < kPer; ++e) sm.hist[tid + e * kSelThreads] = v[e];
  }
  __syncthreads();
  find_threshold_bin([&](int i) { return sm.hist[i]; }, kTopkBins, k, sm.scan, &sm.bstar,
                     &sm.above);
  const uint32_t bstar = (uint32_t)sm.bstar;
  const int above = sm.above;

  // 2. this CTA's slice: sure winners (above b*) and candidates (in b*),
  //    appended as (index, key) pairs; one atomic per warp and batch
  uint32_t *ctr = w.ctr + (size_t)row * 4;
  uint64_t *selrow = w.sel + (size_t)row * k;
  uint64_t *candrow = w.cand + (size_t)row * kCandCap;
  const long long per = ((n + gridDim.x - 1) / gridDim.x + 31) & ~31LL;
  const long long j_lo = (long long)blockIdx.x * per;
  const long long j_hi = min(n, j_lo + per);
  const unsigned lt_mask = (1u << lane) - 1u;
  for (long long j0 = j_lo; j0 < j_hi; j0 += (long long)kScanBatch * kSelThreads) {
    uint32_t key[kScanBatch];
#pragma unroll
    for (int e = 0; e < kScanBatch; ++e) {
      const long long j = j0 + e * kSelThreads + tid;
      key[e] = j < j_hi ? score_key(__ldcg(s + j)) : 0u;
    }
    unsigned mg[kScanBatch], me[kScanBatch];
    int cg = 0, ce = 0;
#pragma unroll
    for (int e = 0; e < kScanBatch; ++e) {
      const long long j = j0 + e * kSelThreads + tid;
      const uint32_t bkt = key[e] >> kTopkShift;
      mg[e] = __ballot_sync(0xffffffffu, j < j_hi && bkt > bstar);
      me[e] = __ballot_sync(0xffffffffu, j < j_hi && bkt == bstar);
      cg += __popc(mg[e]);
      ce += __popc(me[e]);
    }
    uint32_t bg = 0, be = 0;
    if (lane == 0) {
      if (cg) bg = atomicAdd(&ctr[0], (uint32_t)cg);
      if (ce) be = atomicAdd(&ctr[1], (uint32_t)ce);
    }
    bg = __shfl_sync(0xffffffffu, bg, 0);
    be = __shfl_sync(0xffffffffu, be, 0);
#pragma unroll
    for (int e = 0; e < kScanBatch; ++e) {
      const long long j = j0 + e * kSelThreads + tid;
      if (mg[e] >> lane & 1u) {
        const uint32_t p = bg + __popc(mg[e] & lt_mask);
        if (p < (uint32_t)k) selrow[p] = pack_entry(j, key[e]);
      }
      if (me[e] >> lane & 1u) {
        const uint32_t p = be + __popc(me[e] & lt_mask);
        if (p < (uint32_t)kCandCap) candrow[p] = pack_entry(j, key[e]);
      }
      bg += __popc(mg[e]);
      be += __popc(me[e]);
    }
  }

  // 3. the last CTA of the row finishes the selection
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    sm.is_last = atomicAdd(&ctr[2], 1u) == gridDim.x - 1;
    if (sm.is_last) {
      __threadfence();
      sm.n_sel = (int)atomicAdd(&ctr[0], 0u);
      sm.n_cand = (int)atomicAdd(&ctr[1], 0u);
    }
  }
  __syncthreads();
  if (!sm.is_last) return;
  const int n_cand = sm.n_cand;
  const int r = k - above;                 // candidates still to take, 1 <= r <= n_cand
  // any inconsistency between the histogram and the scores (never expected)
  // sends the row to the single-CTA path instead of indexing out of range
  if (tid == 0)
    sm.fallback = above < 0 || above >= k || r < 1 || r > n_cand || n_cand > kCandSmem ||
                  sm.n_sel != above;
  __syncthreads();
  if (!sm.fallback) {
    {  // candidates and sure winners into shared memory, loads first
      constexpr int kC = kCandSmem / kSelThreads, kS = kMaxK / kSelThreads;
      uint64_t v[kC], u[kS];
#pragma unroll
      for (int e = 0; e < kC; ++e) {
        const int i = tid + e * kSelThreads;
        v[e] = i < n_cand ? __ldcg(candrow + i) : 0ull;
      }
#pragma unroll
      for (int e = 0; e < kS; ++e) {
        const int i = tid + e * kSelThreads;
        u[e] = i < above ? __ldcg(selrow + i) : 0ull;
      }
#pragma unroll
      for (int e = 0; e < kC; ++e) {
        const int i = tid + e * kSelThreads;
        if (i < n_cand) sm.cand[i] = v[e];
      }
#pragma unroll
      for (int e = 0; e < kS; ++e) {
        const int i = tid + e * kSelThreads;
        if (i < above) sm.out[i] = u[e];
      }
    }
    // radix select of the r-th largest candidate key on bits 19..10, then 9..0
    uint32_t prefix = bstar << kTopkShift, mask = 0xFFFu << kTopkShift;
    int remaining = r;
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = 10 - 10 * pass;
      for (int i = tid; i < 1024; i += blockDim.x) sm.hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n_cand; i += blockDim.x) {
        const uint32_t key = (uint32_t)sm.cand[i];
        if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 1023u], 1u);
      }
      __syncthreads();
      if (tid == 0) { sm.thr2 = 0; sm.take_eq = 0; }
      find_threshold_bin([&](int i) { return sm.hist[i]; }, 1024, remaining, sm.scan, &sm.thr2,
                         &sm.take_eq);
      prefix = prefix | ((uint32_t)sm.thr2 << shift);
      remaining = remaining - sm.take_eq;
      mask |= 1023u << shift;
      __syncthreads();
    }
    const uint32_t thr2 = prefix;
    const int take_eq = remaining;
    // candidates above thr2 follow the sure winners; the indices of candidates
    // equal to thr2 go to a tie list (the lowest take_eq of them are taken)
    if (tid == 0) { sm.n_gt = 0; sm.n_eq = 0; }
    __syncthreads();
    uint32_t *eqv = sm.hist;                 // up to kTopkBins entries
    for (int i = tid; i < n_cand; i += blockDim.x) {
      const uint64_t c = sm.cand[i];
      const uint32_t key = (uint32_t)c;
      if (key > thr2) {
        const int p = atomicAdd(&sm.n_gt, 1);
        if (above + p < k) sm.out[above + p] = c;
      } else if (key == thr2) {
        const int p = atomicAdd(&sm.n_eq, 1);
        if (p < kTopkBins) eqv[p] = (uint32_t)(c >> 32);
      }
    }
    __syncthreads();
    const int n_gt = sm.n_gt, n_eq = sm.n_eq;
    if (n_eq > kTopkBins || above + n_gt + take_eq != k || take_eq > n_eq) {
      if (tid == 0) sm.fallback = 1;
    } else {
      if (n_eq > take_eq) {
        int m = 1;
        while (m < n_eq) m <<= 1;
        for (int i = n_eq + tid; i < m; i += blockDim.x) eqv[i] = 0xffffffffu;
        __syncthreads();
        bitonic_sort_smem(eqv, m);
      }
      for (int i = tid; i < take_eq; i += blockDim.x)
        sm.out[above + n_gt + i] = ((uint64_t)eqv[i] << 32) | thr2;
    }
    __syncthreads();
    if (!sm.fallback) {
      if (n <= kBitmapEntries) {
        // ascending order by rank: the selected entries are distinct indices
        // below n; mark them in a bitmap, prefix-count the words, and each
        // entry's rank is the count of marked indices below it
        uint32_t *bits = reinterpret_cast<uint32_t *>(sm.cand);
        uint32_t *wpre = bits + kBitmapWords;
        const int nw = (int)((n + 31) >> 5);
        for (int i = tid; i < nw; i += blockDim.x) bits[i] = 0u;
        __syncthreads();
        for (int i = tid; i < k; i += blockDim.x) {
          const uint32_t j = (uint32_t)(sm.out[i] >> 32);
          atomicOr(&bits[j >> 5], 1u << (j & 31));
        }
        __syncthreads();
        // warp w owns words [w * span, (w + 1) * span), read lane-contiguous
        // (conflict-free); a warp scan inside, a block scan across warps
        const int nwarps = blockDim.x >> 5, warp = tid >> 5;
        const int span = (((nw + nwarps - 1) / nwarps) + 31) & ~31;
        const int wb = warp * span;
        int cnt = 0;
        for (int i = lane; i < span; i += 32)
          if (wb + i < nw) cnt += __popc(bits[wb + i]);
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        int tot;
        int run = block_exclusive_scan(lane == 0 ? cnt : 0, sm.scan, &tot);
        run = __shfl_sync(0xffffffffu, run, 0);
        for (int i0 = 0; i0 < span; i0 += 32) {
          const int wi = wb + i0 + lane;
          const int c = wi < nw ? __popc(bits[wi]) : 0;
          int incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          if (wi < nw) wpre[wi] = (uint32_t)(run + incl - c);
          run += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncthreads();
        for (int i = tid; i < k; i += blockDim.x) {
          const uint64_t e = sm.out[i];
          const uint32_t j = (uint32_t)(e >> 32);
          const int rank = (int)wpre[j >> 5] + __popc(bits[j >> 5] & ((1u << (j & 31)) - 1u));
          oi[rank] = (int32_t)j;
          if (os) os[rank] = key_score((uint32_t)e);
        }
      } else {
        int m = 1;
        while (m < k) m <<= 1;
        for (int i = k + tid; i < m; i += blockDim.x) sm.out[i] = ~0ull;
        __syncthreads();
        bitonic_sort_smem(sm.out, m);        // ascending entry index
        for (int i = tid; i < k; i += blockDim.x) {
          const uint64_t e = sm.out[i];
          oi[i] = (int32_t)(e >> 32);
          if (os) os[i] = key_score((uint32_t)e);
        }
      }
    }
  }
  __syncthreads();
  if (sm.fallback) topk_row_single_cta(s, n, k, oi, os);
}

void launch_topk_rows(const float *scores, long long ld, const int64_t *q_pos, int stride,
                      long long max_entries, int k, int rows, int32_t *out_idx,
                      float *out_score, cudaStream_t st) {
  launch_pdl(topk_rows_kernel, dim3(rows), dim3(1024), 0, st, scores, ld, q_pos, stride,
             max_entries, k, out_idx, out_score);
}

int launch_topk_select(const IndexerWs &w, const int64_t *q_pos, int stride,
                       long long max_entries, int k, int rows, int32_t *out_idx,
                       float *out_score, cudaStream_t st) {
  if (k > kMaxK) return CSKV_ERR_UNSUPPORTED;
  const size_t smem = sizeof(SelSmem);
  if (!ensure_dynamic_smem(topk_select_kernel, smem)) return CSKV_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // slices of at least 4096 scores; enough CTAs to cover the SMs at one row
  long long splits = (max_entries + 4095) / 4096;
  const long long cap = (sms + rows - 1) / rows;
  if (splits > cap) splits = cap;
  if (splits < 1) splits = 1;
  launch_pdl(topk_select_kernel, dim3((unsigned)splits, (unsigned)rows), dim3(kSelThreads), smem,
             st, w, q_pos, stride, max_entries, k, out_idx, out_score);
  return cudaGetLastError() == cudaSuccess ? CSKV_OK : CSKV_ERR_CUDA;
}

}  // namespace cskv
