// Lightning-indexer scoring (generic CUDA-core path) and the indexer_topk driver.
//
// The indexer scores every compressed CSA entry per query at low precision
// («DeepSeek V4-Pro: Architektur, KV-Cache-Kompression und Hyper-Connections
// im Detail», "Kompression und Selektion"; «DeepSeek-V4: 1 Million Token
// Context endlich nutzbar», "Hybrid Attention: CSA und HCA").  Score of entry j
// for one query row:  s_j = sum_h w[h] * max(0, q[h] . k[j])  with q and k
// the dequantised FP8 (or fp32) vectors.
//
// This file holds the path for any (H_I, d_I) and both formats: one thread
// per entry, the query's heads dequantised once per CTA into shared memory.
// The 64-head x 128-dim FP8 layout at scale goes through the tensor-core
// kernel in indexer_tc.cu.
#include "cskv_internal.cuh"
#include "topk_common.cuh"

namespace cskv {

void launch_topk_rows(const float *scores, long long ld, const int64_t *q_pos, int stride,
                      long long max_entries, int k, int rows, int32_t *out_idx,
                      float *out_score, unsigned int *status, cudaStream_t st);
int launch_topk_select(const IndexerWs &w, const int64_t *q_pos, int stride,
                       long long max_entries, int k, int rows, int32_t *out_idx,
                       float *out_score, unsigned int *status, cudaStream_t st);
bool indexer_tc_supported(const IndexerArgs &a);
bool indexer_mxf4_supported(const IndexerArgs &a);
int launch_indexer_mxf4(const IndexerArgs &a, float *scores, long long ld, uint32_t *hist,
                        uint32_t *ctr, cudaStream_t st);
int launch_indexer_tc(const IndexerArgs &a, float *scores, long long ld, uint32_t *hist,
                      uint32_t *ctr, cudaStream_t st);
int launch_indexer_rows(const IndexerArgs &a, float *scores, long long ld, uint32_t *hist,
                        uint32_t *ctr, cudaStream_t st);

namespace {

constexpr int kKeys = 128;   // entries per CTA (one per thread)

__global__ void __launch_bounds__(kKeys)
indexer_score_kernel(IndexerArgs a, float *__restrict__ scores, long long ld) {
  extern __shared__ float sm[];
  pdl_wait();
  pdl_trigger();
  const int H = a.H_I, dI = a.d_I;
  float *q = sm;                       // [H][dI]
  float *w = q + H * dI;               // [H]
  float *kt = w + H;                   // [kKeys][dI + 1]
  const int row = blockIdx.y;
  const int b = row / a.Tq;
  long long n = (a.q_pos[row] + 1) / a.stride;
  if (n > a.max_entries) n = a.max_entries;
  const long long j0 = (long long)blockIdx.x * kKeys;
  if (j0 >= n) return;
  const int tid = threadIdx.x;
  const long long qoff = (long long)row * H * dI;
  for (int i = tid; i < H * dI; i += blockDim.x) {
    if (a.ik.fmt == CSKV_FMT_F32) {
      q[i] = reinterpret_cast<const float *>(a.q_ik)[qoff + i];
    } else if (a.ik.fmt == CSKV_FMT_MXFP4) {
      // packed codes of head i / dI, dim i % dI; one E8M0 byte per 32 dims
      const uint8_t code = reinterpret_cast<const uint8_t *>(a.q_ik)[(qoff + i) >> 1];
      const uint8_t *ex = reinterpret_cast<const uint8_t *>(a.q_ik_scale);
      q[i] = mxfp4_value(code >> (((qoff + i) & 1) << 2), ex[(qoff + i) >> 5]);
    } else {
      const int h = i / dI, d = i % dI;
      // query scales follow the keys' layout: per 64 dims, or one per head
      const float sc = a.ik.fmt == CSKV_FMT_E4M3_VEC
                           ? a.q_ik_scale[(long long)row * H + h]
                           : a.q_ik_scale[((long long)row * H + h) * (dI >> 6) + (d >> 6)];
      q[i] = e4m3_decode(reinterpret_cast<const uint8_t *>(a.q_ik)[qoff + i]) * sc;
    }
  }
  for (int h = tid; h < H; h += blockDim.x) w[h] = a.head_w[(long long)row * H + h];
  // dequantise this CTA's keys (coalesced over dims)
  for (int i = tid; i < kKeys * dI; i += blockDim.x) {
    const int r = i / dI, d = i % dI;
    const long long j = j0 + r;
    kt[r * (dI + 1) + d] = j < n ? a.ik.value(b, j, d) : 0.f;
  }
  __syncthreads();
  const long long j = j0 + tid;
  if (j >= n) return;
  const float *kr = kt + tid * (dI + 1);
  float s = 0.f;
  for (int h = 0; h < H; ++h) {
    const float *qh = q + h * dI;
    float dot = 0.f;
    for (int d = 0; d < dI; ++d) dot = fmaf(qh[d], kr[d], dot);
    s = fmaf(w[h], fmaxf(dot, 0.f), s);
  }
  scores[(long long)row * ld + j] = s;
}

}  // namespace

size_t indexer_ws_bytes(int B, int Tq, long long max_entries, int k) {
  size_t total = 0;
  indexer_ws_layout(nullptr, (long long)B * Tq, max_entries, k, &total);
  return total;
}

int launch_indexer_topk(const IndexerArgs &a, int phases, cudaStream_t st) {
  const int rows = a.B * a.Tq;
  if (rows == 0) return CSKV_OK;
  const IndexerWs w = indexer_ws_layout(a.ws, rows, a.max_entries, a.k, nullptr);
  const bool score = phases & kIndexerScore, select = phases & kIndexerSelect;
  const bool mxf4 = a.max_entries > 0 && indexer_mxf4_supported(a);
  if (a.max_entries > 0 && (mxf4 || indexer_tc_supported(a))) {
    // tensor-core scoring builds the score histogram the multi-CTA selection
    // uses.  The histogram only guides the selection (every count it implies
    // is checked against the scores, and a row whose counts disagree is
    // selected from its scores alone), so it is not cleared before the call:
    // the selection clears each row's histogram once it has read it, and a
    // fresh workspace's first call at worst takes the slower path.  The
    // scoring kernel clears the selection's counters.
    if (score) {
      // several query rows per sequence share each key tile; one row streams alone
      // (FP4 keys: one query row per CTA group, block-scaled MMAs)
      int rc = mxf4 ? launch_indexer_mxf4(a, w.scores, w.ld, w.hist, w.ctr, st)
                    : launch_indexer_rows(a, w.scores, w.ld, w.hist, w.ctr, st);
      if (!mxf4 && rc == CSKV_ERR_UNSUPPORTED)
        rc = launch_indexer_tc(a, w.scores, w.ld, w.hist, w.ctr, st);
      if (rc != CSKV_OK) return rc;
    }
    if (!select) return CSKV_OK;
    return launch_topk_select(w, a.q_pos, a.stride, a.max_entries, a.k, rows, a.out_idx,
                              a.out_score, a.status, st);
  }
  if (score && a.max_entries > 0) {
    const size_t smem = sizeof(float) * ((size_t)a.H_I * a.d_I + a.H_I +
                                         (size_t)kKeys * (a.d_I + 1));
    if (!ensure_dynamic_smem(indexer_score_kernel, smem)) return CSKV_ERR_UNSUPPORTED;
    dim3 grid((unsigned)((a.max_entries + kKeys - 1) / kKeys), (unsigned)rows);
    if (launch_pdl(indexer_score_kernel, grid, dim3(kKeys), smem, st, a, w.scores, w.ld) !=
        cudaSuccess)
      return CSKV_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return CSKV_ERR_CUDA;
  }
  if (select)
    launch_topk_rows(w.scores, w.ld, a.q_pos, a.stride, a.max_entries, a.k, rows, a.out_idx,
                     a.out_score, a.status, st);
  return cudaGetLastError() == cudaSuccess ? CSKV_OK : CSKV_ERR_CUDA;
}

}  // namespace cskv
