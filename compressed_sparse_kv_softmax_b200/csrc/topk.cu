// Exact top-k selection over lightning-indexer scores.
//
// The lightning indexer forwards the k most relevant CSA entries (512 for
// V4-Flash, 1,024 for V4-Pro; «Chinas KI-Unabhaengigkeit?: Bei Deepseek V4
// haben kleine Aenderungen grosse Wirkung», "Komprimierte Erinnerung fuer
// laengere Kontexte").  Selection here is exact: the k largest scores of the
// row's visible entries, ties to the lower entry index, written in ascending
// entry order (deterministic), -1 / -inf padding when fewer than k are visible.
//
// Method: scores are mapped to order-preserving uint32 keys; a 4-pass 8-bit
// radix select finds the k-th largest key `thr` and how many entries equal
// to it are taken (`take_eq`); a final pass in index order keeps every key
// above thr and the first take_eq keys equal to it, placing each at its rank
// via a block-wide prefix sum.
#include "cskv_internal.cuh"

namespace cskv {

namespace {

constexpr int kTopkThreads = 1024;

// exclusive prefix sum over the block; returns the block total in *total
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

}  // namespace

// scores: [rows][ld] fp32, n_vis per row from q_pos; out_idx/out_score: [rows][k]
__global__ void __launch_bounds__(kTopkThreads)
topk_rows_kernel(const float *__restrict__ scores, long long ld, const int64_t *__restrict__ q_pos,
                 int stride, long long max_entries, int k, int32_t *__restrict__ out_idx,
                 float *__restrict__ out_score) {
  __shared__ int hist[256];
  __shared__ int scan_scratch[33];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  long long n = (q_pos[row] + 1) / stride;
  if (n > max_entries) n = max_entries;
  const float *s = scores + (long long)row * ld;
  int32_t *oi = out_idx + (long long)row * k;
  float *os = out_score ? out_score + (long long)row * k : nullptr;

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
      if (tid == 0) {
        int cum = 0, bkt = 255;
        for (; bkt > 0; --bkt) {
          if (cum + hist[bkt] >= remaining) break;
          cum += hist[bkt];
        }
        s_prefix = prefix | ((uint32_t)bkt << shift);
        s_remaining = remaining - cum;
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      mask |= 255u << shift;
      __syncthreads();
    }
    thr = prefix;
    take_eq = remaining;
  }

  // ordered compaction in index order
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

void launch_topk_rows(const float *scores, long long ld, const int64_t *q_pos, int stride,
                      long long max_entries, int k, int rows, int32_t *out_idx,
                      float *out_score, cudaStream_t st) {
  topk_rows_kernel<<<rows, kTopkThreads, 0, st>>>(scores, ld, q_pos, stride, max_entries, k,
                                                  out_idx, out_score);
}

}  // namespace cskv
