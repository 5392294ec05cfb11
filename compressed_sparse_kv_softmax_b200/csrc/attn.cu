// Hybrid attention: compressed entries (sparse CSA selection or dense HCA) plus
// the raw sliding window under one softmax, split over key chunks and merged
// through log-sum-exp.
//
// CSA attends the lightning indexer's top-k entries, HCA attends densely over
// all compressed blocks («DeepSeek-V4: 1 Million Token Context endlich
// nutzbar», "Hybrid Attention: CSA und HCA"); both additionally attend the raw
// last 128 tokens («Chinas KI-Unabhaengigkeit?: Bei Deepseek V4 haben kleine
// Aenderungen grosse Wirkung», "Komprimierte Erinnerung fuer laengere
// Kontexte").  For one query row with key set K (compressed part then window)
//   l_h = sm_scale * q_h . K,  out_h = softmax(l_h) V,  lse_h = log sum exp l_h.
// Each CTA computes a partial (o, lse) over one chunk of the key list; the
// merge kernel combines the partials: L = log sum_i e^{lse_i},
// out = sum_i e^{lse_i - L} o_i.
//
// This file holds the CUDA-core path for any head count / head dim / format
// and the merge kernel; the 64-head x 512-dim FP8+BF16 layout goes through the
// tensor-core kernel in attn_tc.cu.
#include <math_constants.h>

#include "cskv_internal.cuh"

namespace cskv {

bool attn_tc_supported(const AttnArgs &a);
int launch_attn_tc(const AttnArgs &a, float *part_o, float *part_lse, int n_chunks,
                   cudaStream_t st);
int attn_tc_chunk_keys();

namespace {

constexpr int kChunk = 32;        // keys per CTA in the CUDA-core path
constexpr int kThreads = 256;

struct RowInfo {
  long long pos;          // query position
  long long n_comp;       // compressed keys in the row's list (incl. -1 holes for sel)
  long long w_lo;         // first window position
  int n_win;              // window keys
};

__device__ __forceinline__ RowInfo row_info(const AttnArgs &a, int row) {
  RowInfo r;
  const int b = row / a.Tq;
  r.pos = a.pos_is_ctx_len ? a.pos[b] - 1 : a.pos[row];
  if (!a.has_comp) {
    r.n_comp = 0;
  } else if (a.sel) {
    r.n_comp = a.k;
  } else {
    long long n = (r.pos + 1) / a.comp_stride;
    r.n_comp = n < a.max_entries ? n : a.max_entries;
  }
  r.w_lo = r.pos - a.window + 1;
  if (r.w_lo < 0) r.w_lo = 0;
  r.n_win = (int)(r.pos - r.w_lo + 1);
  return r;
}

__global__ void __launch_bounds__(kThreads)
attn_chunk_kernel(AttnArgs a, int n_comp_chunks, int n_chunks, float *__restrict__ part_o,
                  float *__restrict__ part_lse) {
  extern __shared__ float sm[];
  const int Hq = a.Hq, D = a.D, Dv = a.Dv;
  const bool sep_v = a.win_v.data != nullptr;
  float *q = sm;                          // [Hq][D]
  float *kt = q + Hq * D;                 // [kChunk][D+1]
  float *vt = sep_v ? kt + kChunk * (D + 1) : kt;   // [kChunk][Dv+1]
  float *p = (sep_v ? vt + kChunk * (Dv + 1) : kt + kChunk * (D + 1));  // [Hq][kChunk]
  __shared__ long long key_slot[kChunk];
  __shared__ int key_src[kChunk];         // 0 none, 1 compressed, 2 window

  const int row = blockIdx.y, chunk = blockIdx.x;
  const int b = row / a.Tq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const RowInfo ri = row_info(a, row);

  if (tid < kChunk) {
    int src = 0;
    long long slot = 0;
    if (chunk < n_comp_chunks) {
      const long long i = (long long)chunk * kChunk + tid;
      if (i < ri.n_comp) {
        long long j = a.sel ? (long long)a.sel[(long long)row * a.k + i] : i;
        if (j >= 0 && j < a.comp_k.cap && j < a.comp_v.cap) { src = 1; slot = j; }
      }
    } else {
      const long long i = (long long)(chunk - n_comp_chunks) * kChunk + tid;
      if (i < ri.n_win) { src = 2; slot = a.win_k.slot_of(ri.w_lo + i); }
    }
    key_src[tid] = src;
    key_slot[tid] = slot;
  }
  // query row -> fp32
  const long long qoff = (long long)row * Hq * D;
  for (int i = tid; i < Hq * D; i += kThreads) {
    q[i] = a.win_k.fmt == CSKV_FMT_F32
               ? reinterpret_cast<const float *>(a.q)[qoff + i]
               : __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(a.q)[qoff + i]);
  }
  __syncthreads();
  for (int i = tid; i < kChunk * D; i += kThreads) {
    const int r = i / D, d = i % D;
    const int src = key_src[r];
    float v = 0.f;
    if (src == 1) v = a.comp_k.value(b, key_slot[r], d);
    else if (src == 2) v = a.win_k.value(b, key_slot[r], d);
    kt[r * (D + 1) + d] = v;
  }
  if (sep_v) {
    for (int i = tid; i < kChunk * Dv; i += kThreads) {
      const int r = i / Dv, d = i % Dv;
      const int src = key_src[r];
      float v = 0.f;
      if (src == 1) v = a.comp_v.value(b, key_slot[r], d);
      else if (src == 2) v = a.win_v.value(b, key_slot[r], d);
      vt[r * (Dv + 1) + d] = v;
    }
  }
  __syncthreads();
  // logits: warp <-> head, lane <-> key
  for (int h = warp; h < Hq; h += kThreads / 32) {
    float l = -CUDART_INF_F;
    if (key_src[lane]) {
      const float *qh = q + h * D;
      const float *kr = kt + lane * (D + 1);
      float dot = 0.f;
      for (int d = 0; d < D; ++d) dot = fmaf(qh[d], kr[d], dot);
      l = a.sm_scale * dot;
    }
    const float m = warp_max(l);
    const float e = (m == -CUDART_INF_F || l == -CUDART_INF_F) ? 0.f : expf(l - m);
    const float s = warp_sum(e);
    p[h * kChunk + lane] = s > 0.f ? e / s : 0.f;
    if (lane == 0)
      part_lse[((long long)row * n_chunks + chunk) * Hq + h] =
          s > 0.f ? m + logf(s) : -CUDART_INF_F;
  }
  __syncthreads();
  // partial output o_h = sum_c p[h][c] V[c]
  const int vstride = sep_v ? Dv + 1 : D + 1;
  float *po = part_o + ((long long)row * n_chunks + chunk) * Hq * Dv;
  for (int i = tid; i < Hq * Dv; i += kThreads) {
    const int h = i / Dv, d = i % Dv;
    const float *ph = p + h * kChunk;
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < kChunk; ++c) acc = fmaf(ph[c], vt[c * vstride + d], acc);
    po[i] = acc;
  }
}

// out[row][h][:] = sum_i e^{lse_i - L} o_i,  lse[row][h] = L = log sum_i e^{lse_i}
// CTA (row * Hq + head, d-block of 128); 4 groups of 128 threads split the chunks,
// each thread one output dim; a shared-memory sum joins the groups.
constexpr int kMergeD = 128, kMergeGroups = 4;

__global__ void __launch_bounds__(kMergeD * kMergeGroups)
attn_merge_kernel(int Hq, int Dv, int n_chunks, const float *__restrict__ part_o,
                  const float *__restrict__ part_lse, float *__restrict__ out,
                  float *__restrict__ lse) {
  extern __shared__ float wts[];          // [n_chunks]
  __shared__ float red[kMergeGroups][kMergeD];
  __shared__ float s_L;
  const int row = blockIdx.x / Hq, h = blockIdx.x % Hq;
  const int tid = threadIdx.x, grp = tid / kMergeD, dl = tid % kMergeD;
  const int d = blockIdx.y * kMergeD + dl;
  const float *pl = part_lse + (long long)row * n_chunks * Hq + h;
  for (int i = tid; i < n_chunks; i += blockDim.x) wts[i] = __ldg(pl + (long long)i * Hq);
  __syncthreads();
  if (tid < 32) {
    float m = -CUDART_INF_F;
    for (int i = tid; i < n_chunks; i += 32) m = fmaxf(m, wts[i]);
    m = warp_max(m);
    float s = 0.f;
    for (int i = tid; i < n_chunks; i += 32) s += wts[i] == -CUDART_INF_F ? 0.f : expf(wts[i] - m);
    s = warp_sum(s);
    const float L = m + logf(s);
    __syncwarp();
    for (int i = tid; i < n_chunks; i += 32)
      wts[i] = wts[i] == -CUDART_INF_F ? 0.f : expf(wts[i] - L);
    if (tid == 0) s_L = L;
  }
  __syncthreads();
  float acc = 0.f;
  if (d < Dv) {
    const float *po = part_o + (long long)row * n_chunks * Hq * Dv + (long long)h * Dv + d;
    const long long cstride = (long long)Hq * Dv;
#pragma unroll 8
    for (int i = grp; i < n_chunks; i += kMergeGroups) {
      const float w = wts[i];
      if (w != 0.f) acc = fmaf(w, __ldg(po + i * cstride), acc);
    }
  }
  red[grp][dl] = acc;
  __syncthreads();
  if (grp == 0 && d < Dv) {
    float t = red[0][dl];
#pragma unroll
    for (int g = 1; g < kMergeGroups; ++g) t += red[g][dl];
    out[((long long)row * Hq + h) * Dv + d] = t;
  }
  if (blockIdx.y == 0 && tid == 0) lse[(long long)row * Hq + h] = s_L;
}

int chunk_keys(const AttnArgs &a) { return attn_tc_supported(a) ? attn_tc_chunk_keys() : kChunk; }

}  // namespace

static void plan_chunks(long long max_comp, int window, int chunk, int *n_comp_chunks,
                        int *n_chunks) {
  *n_comp_chunks = (int)((max_comp + chunk - 1) / chunk);
  *n_chunks = *n_comp_chunks + (window + chunk - 1) / chunk;
}

size_t attn_ws_bytes(int B, int Tq, int Hq, int Dv, long long max_entries, int window) {
  // sized for the smaller chunk of the two paths (more partials)
  int ncc, nc;
  plan_chunks(max_entries, window, kChunk, &ncc, &nc);
  const size_t rows = (size_t)B * Tq;
  return rows * nc * Hq * ((size_t)Dv + 1) * sizeof(float) + 512;
}

int launch_attention(const AttnArgs &a, cudaStream_t st) {
  const int rows = a.B * a.Tq;
  if (rows == 0) return CSKV_OK;
  const int chunk = chunk_keys(a);
  int ncc, nc;
  plan_chunks(a.has_comp ? (a.sel ? a.k : a.max_entries) : 0, a.window, chunk, &ncc, &nc);
  float *part_o = reinterpret_cast<float *>(a.ws);
  float *part_lse = part_o + (size_t)rows * nc * a.Hq * a.Dv;
  part_lse = reinterpret_cast<float *>(((uintptr_t)part_lse + 255) & ~(uintptr_t)255);
  if (attn_tc_supported(a)) {
    const int rc = launch_attn_tc(a, part_o, part_lse, nc, st);
    if (rc != CSKV_OK) return rc;
  } else {
    const bool sep_v = a.win_v.data != nullptr;
    const size_t smem = sizeof(float) * ((size_t)a.Hq * a.D + (size_t)kChunk * (a.D + 1) +
                                         (sep_v ? (size_t)kChunk * (a.Dv + 1) : 0) +
                                         (size_t)a.Hq * kChunk);
    if (!ensure_dynamic_smem(attn_chunk_kernel, smem)) return CSKV_ERR_UNSUPPORTED;
    attn_chunk_kernel<<<dim3(nc, rows), kThreads, smem, st>>>(a, ncc, nc, part_o, part_lse);
    if (cudaGetLastError() != cudaSuccess) return CSKV_ERR_CUDA;
  }
  const size_t msmem = sizeof(float) * nc;
  if (!ensure_dynamic_smem(attn_merge_kernel, msmem)) return CSKV_ERR_UNSUPPORTED;
  attn_merge_kernel<<<dim3((unsigned)(rows * a.Hq), (a.Dv + kMergeD - 1) / kMergeD), kMergeD * kMergeGroups,
                      msmem, st>>>(a.Hq, a.Dv, nc, part_o, part_lse, a.out, a.lse);
  return cudaGetLastError() == cudaSuccess ? CSKV_OK : CSKV_ERR_CUDA;
}

}  // namespace cskv
