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

#include <cstdlib>

#include "cskv_internal.cuh"

namespace cskv {

bool attn_tc_supported(const AttnArgs &a);
int launch_attn_tc(const AttnArgs &a, const AttnPlan &p, float *part_o, float *part_lse,
                   cudaStream_t st);
int attn_tc_unit_keys(long long rows, long long keys);
size_t attn_tc_tile_bytes(int B, int Tq, long long max_entries);

namespace {

constexpr int kChunk = 32;        // keys per unit in the CUDA-core path (one per lane)
constexpr int kThreads = 256;
constexpr int kTargetCtas = 296;  // splits aim at two CTAs per SM of a 148-SM part

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
    // checked build: the row's visible entries within the host bound and the caches
    if (kChecked && threadIdx.x == 0)
      a.comp_k.check(n <= a.max_entries && n <= a.comp_k.cap && n <= a.comp_v.cap);
  }
  r.w_lo = r.pos - a.window + 1;
  if (r.w_lo < 0) r.w_lo = 0;
  r.n_win = (int)(r.pos - r.w_lo + 1);
  return r;
}

// CUDA-core path: a split runs its units (kChunk keys each) with an online
// softmax, the running output in shared memory.
__global__ void __launch_bounds__(kThreads)
attn_units_kernel(AttnArgs a, AttnPlan p, float *__restrict__ part_o,
                  float *__restrict__ part_lse) {
  extern __shared__ float sm[];
  pdl_wait();
  pdl_trigger();
  const int Hq = a.Hq, D = a.D, Dv = a.Dv;
  const bool sep_v = a.win_v.data != nullptr;
  float *q = sm;                                    // [Hq][D]
  float *kt = q + Hq * D;                           // [kChunk][D+1]
  float *vt = sep_v ? kt + kChunk * (D + 1) : kt;   // [kChunk][Dv+1]
  float *pt = (sep_v ? vt + kChunk * (Dv + 1) : kt + kChunk * (D + 1));  // [Hq][kChunk]
  float *o = pt + Hq * kChunk;                      // [Hq][Dv] running output
  float *mrun = o + Hq * Dv, *lrun = mrun + Hq, *alpha = lrun + Hq;
  __shared__ long long key_slot[kChunk];
  __shared__ int key_src[kChunk];                   // 0 none, 1 compressed, 2 window

  const int row = blockIdx.x, split = blockIdx.y;
  const int b = row / a.Tq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const RowInfo ri = row_info(a, row);
  const long long qoff = (long long)row * Hq * D;
  for (int i = tid; i < Hq * D; i += kThreads) {
    q[i] = a.win_k.fmt == CSKV_FMT_F32
               ? reinterpret_cast<const float *>(a.q)[qoff + i]
               : __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(a.q)[qoff + i]);
  }
  for (int i = tid; i < Hq * Dv; i += kThreads) o[i] = 0.f;
  for (int h = tid; h < Hq; h += kThreads) {
    mrun[h] = -CUDART_INF_F;
    lrun[h] = 0.f;
  }
  const int u_begin = split * p.per_cta;
  const int u_end = min(p.n_units, u_begin + p.per_cta);
  for (int unit = u_begin; unit < u_end; ++unit) {
    if (tid < kChunk) {
      int src = 0;
      long long slot = 0;
      if (unit < p.n_comp_units) {
        const long long i = (long long)unit * kChunk + tid;
        if (i < ri.n_comp) {
          const long long j = a.sel ? (long long)a.sel[(long long)row * a.k + i] : i;
          if (j >= 0 && j < a.comp_k.cap && j < a.comp_v.cap) { src = 1; slot = j; }
          // checked build: a selected entry is -1 or visible to the row
          if (kChecked && a.sel &&
              !a.comp_k.check(j == -1 || (src == 1 && j < (ri.pos + 1) / a.comp_stride)))
            src = 0;
        }
      } else {
        const long long i = (long long)(unit - p.n_comp_units) * kChunk + tid;
        if (i < ri.n_win) { src = 2; slot = a.win_k.slot_of(ri.w_lo + i); }
      }
      key_src[tid] = src;
      key_slot[tid] = slot;
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
    // logits and softmax update: warp <-> head, lane <-> key
    for (int h = warp; h < Hq; h += kThreads / 32) {
      float l = -CUDART_INF_F;
      if (key_src[lane]) {
        const float *qh = q + h * D;
        const float *kr = kt + lane * (D + 1);
        float dot = 0.f;
        for (int d = 0; d < D; ++d) dot = fmaf(qh[d], kr[d], dot);
        l = a.sm_scale * dot;
      }
      const float mold = mrun[h];
      const float mnew = fmaxf(mold, warp_max(l));
      const float e = l == -CUDART_INF_F ? 0.f : expf(l - mnew);
      const float s = warp_sum(e);
      pt[h * kChunk + lane] = e;
      if (lane == 0) {
        const float al = mold == -CUDART_INF_F ? 0.f : expf(mold - mnew);
        alpha[h] = al;
        lrun[h] = lrun[h] * al + s;
        mrun[h] = mnew;
      }
    }
    __syncthreads();
    const int vstride = sep_v ? Dv + 1 : D + 1;
    for (int i = tid; i < Hq * Dv; i += kThreads) {
      const int h = i / Dv, d = i % Dv;
      const float *ph = pt + h * kChunk;
      float acc = o[i] * alpha[h];
#pragma unroll 8
      for (int c = 0; c < kChunk; ++c) acc = fmaf(ph[c], vt[c * vstride + d], acc);
      o[i] = acc;
    }
    __syncthreads();
  }
  float *po = part_o + ((long long)row * p.splits + split) * Hq * Dv;
  for (int i = tid; i < Hq * Dv; i += kThreads) {
    const float l = lrun[i / Dv];
    po[i] = l > 0.f ? o[i] / l : 0.f;
  }
  for (int h = tid; h < Hq; h += kThreads)
    part_lse[((long long)row * p.splits + split) * Hq + h] =
        lrun[h] > 0.f ? mrun[h] + logf(lrun[h]) : -CUDART_INF_F;
}

// out[row][h][:] = sum_i e^{lse_i - L} o_i,  lse[row][h] = L = log sum_i e^{lse_i}
// CTA (row * Hq + head, half of the dims), 1024 threads: thread t takes 4
// consecutive dims (t % 64) and the partials i = t / 64, t / 64 + 16, ..;
// every partial a thread reads is requested before any is used, together
// with the LSEs, whose weights one warp computes; shared memory sums the 16
// groups.
constexpr int kMergeThreads = 1024, kMergeQuads = 64;            // 4-dim columns per CTA
constexpr int kMergeGroups = kMergeThreads / kMergeQuads;        // 16
constexpr int kMergeBatch = 9;      // partials per thread and batch (144 per CTA)
constexpr int kMergeLse = 2048;     // LSE weights held in shared memory

// four consecutive values p[0..3] of which the first n exist (16-byte load when
// vec and all four exist)
__device__ __forceinline__ float4 load4(const float *p, int n, bool vec) {
  if (vec && n >= 4) return __ldcg(reinterpret_cast<const float4 *>(p));
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  if (n > 0) r.x = __ldcg(p);
  if (n > 1) r.y = __ldcg(p + 1);
  if (n > 2) r.z = __ldcg(p + 2);
  if (n > 3) r.w = __ldcg(p + 3);
  return r;
}

__global__ void __launch_bounds__(kMergeThreads)
attn_merge_kernel(int Hq, int Dv, int n_chunks, const float *__restrict__ part_o,
                  const float *__restrict__ part_lse, float *__restrict__ out,
                  float *__restrict__ lse) {
  __shared__ float4 red[kMergeGroups][kMergeQuads];
  __shared__ float wts[kMergeLse];
  __shared__ float s_L;
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x / Hq, h = blockIdx.x % Hq;
  const int tid = threadIdx.x, q = tid % kMergeQuads, g = tid / kMergeQuads;
  const int d = (blockIdx.y * kMergeQuads + q) * 4;
  const bool dv = d < Dv;
  const int nd = Dv - d;                   // dims of this thread's four that exist
  const bool vec = (Dv & 3) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0;
  const float *pl = part_lse + (long long)row * n_chunks * Hq + h;
  const float *po = part_o + (long long)row * n_chunks * Hq * Dv + (long long)h * Dv + d;
  const long long cstride = (long long)Hq * Dv;
  // the LSEs (needed first) and the first batch of partials, all in flight at once
  const int nw = n_chunks < kMergeLse ? n_chunks : kMergeLse;
  float lv[kMergeLse / kMergeThreads];
#pragma unroll
  for (int e = 0; e < kMergeLse / kMergeThreads; ++e) {
    const int i = tid + e * kMergeThreads;
    lv[e] = i < nw ? __ldcg(pl + (long long)i * Hq) : 0.f;
  }
  float4 v[kMergeBatch];
#pragma unroll
  for (int k = 0; k < kMergeBatch; ++k) {
    const int i = g + k * kMergeGroups;
    v[k] = (i < n_chunks && dv) ? load4(po + i * cstride, nd, vec) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int e = 0; e < kMergeLse / kMergeThreads; ++e) {
    const int i = tid + e * kMergeThreads;
    if (i < nw) wts[i] = lv[e];
  }
  __syncthreads();
  if (tid < 32) {
    float m = -CUDART_INF_F;
    for (int i = tid; i < n_chunks; i += 32)
      m = fmaxf(m, i < kMergeLse ? wts[i] : __ldcg(pl + (long long)i * Hq));
    m = warp_max(m);
    float ssum = 0.f;
    if (m != -CUDART_INF_F)
      for (int i = tid; i < n_chunks; i += 32)
        ssum += expf((i < kMergeLse ? wts[i] : __ldcg(pl + (long long)i * Hq)) - m);
    ssum = warp_sum(ssum);
    const float L = m != -CUDART_INF_F ? m + logf(ssum) : -CUDART_INF_F;
    __syncwarp();
    for (int i = tid; i < nw; i += 32)
      wts[i] = wts[i] == -CUDART_INF_F ? 0.f : expf(wts[i] - L);
    if (tid == 0) s_L = L;
  }
  __syncthreads();
  const float L = s_L;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int b0 = 0; b0 < n_chunks; b0 += kMergeGroups * kMergeBatch) {
    if (b0 > 0) {
#pragma unroll
      for (int k = 0; k < kMergeBatch; ++k) {
        const int i = b0 + g + k * kMergeGroups;
        v[k] = (i < n_chunks && dv) ? load4(po + i * cstride, nd, vec)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) {
      const int i = b0 + g + k * kMergeGroups;
      if (i < n_chunks) {
        const float li = i < kMergeLse ? 0.f : __ldcg(pl + (long long)i * Hq);
        const float w = i < kMergeLse ? wts[i] : (li == -CUDART_INF_F ? 0.f : expf(li - L));
        acc.x = fmaf(w, v[k].x, acc.x);
        acc.y = fmaf(w, v[k].y, acc.y);
        acc.z = fmaf(w, v[k].z, acc.z);
        acc.w = fmaf(w, v[k].w, acc.w);
      }
    }
  }
  red[g][q] = acc;
  __syncthreads();
  // every partial has been read (the values were used before the barrier):
  // their 128-byte lines leave L2 without being written back to HBM
  if ((q & 7) == 0 && dv && (Dv & 31) == 0)
    for (int i = g; i < n_chunks; i += kMergeGroups) discard_l2_line(po + i * cstride);
  if (g == 0 && dv) {
    float4 t = red[0][q];
#pragma unroll
    for (int k = 1; k < kMergeGroups; ++k) {
      const float4 u = red[k][q];
      t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
    }
    float *o = out + ((long long)row * Hq + h) * Dv + d;
    if (vec) {
      *reinterpret_cast<float4 *>(o) = t;
    } else {
      o[0] = t.x;
      if (nd > 1) o[1] = t.y;
      if (nd > 2) o[2] = t.z;
      if (nd > 3) o[3] = t.w;
    }
  }
  if (blockIdx.y == 0 && tid == 0) lse[(long long)row * Hq + h] = L;
}

}  // namespace

// CSKV_SPLITS=<n> in the environment (read once per process): n splits per
// query row instead of the planned count, for tuning (clipped to the row's
// units; the workspace sizes follow it, so it has to be set before the first
// call that sizes a workspace).  0 when unset or not a positive number.
static long long splits_override() {
  static const long long v = [] {
    const char *e = std::getenv("CSKV_SPLITS");
    if (!e || !*e) return 0LL;
    char *end = nullptr;
    const long long n = std::strtoll(e, &end, 10);
    return (end && *end == '\0' && n > 0) ? n : 0LL;
  }();
  return v;
}

AttnPlan attn_plan(long long rows, long long max_comp, int window, int unit) {
  AttnPlan p;
  p.unit = unit;
  p.n_comp_units = (int)((max_comp + unit - 1) / unit);
  p.n_units = p.n_comp_units + (window + unit - 1) / unit;
  long long splits = (kTargetCtas + rows - 1) / rows;
  if (splits_override() > 0) splits = splits_override();
  if (splits > p.n_units) splits = p.n_units;
  if (splits < 1) splits = 1;
  p.per_cta = (int)((p.n_units + splits - 1) / splits);
  p.splits = (p.n_units + p.per_cta - 1) / p.per_cta;
  return p;
}

static size_t partial_bytes(const AttnPlan &p, long long rows, int Hq, int Dv) {
  if (p.splits <= 1) return 0;   // one split per row writes the output directly
  return (size_t)rows * p.splits * Hq * ((size_t)Dv + 1) * sizeof(float) + 512;
}

size_t attn_ws_bytes(int B, int Tq, int Hq, int Dv, long long max_entries, int window) {
  // either path may run: the larger of the two plans, or of the converted
  // key tiles of a dense prefill (used only when a row has one split)
  const long long rows = (long long)B * Tq;
  const size_t a = partial_bytes(attn_plan(rows, max_entries, window, kChunk), rows, Hq, Dv);
  const size_t b = partial_bytes(
      attn_plan(rows, max_entries, window, attn_tc_unit_keys(rows, max_entries + window)), rows,
      Hq, Dv);
  const size_t t = attn_tc_tile_bytes(B, Tq, max_entries);
  const size_t m = a > b ? a : b;
  return m > t ? m : t;
}

int launch_attention(const AttnArgs &a, cudaStream_t st) {
  const int rows = a.B * a.Tq;
  if (rows == 0) return CSKV_OK;
  const bool tc = attn_tc_supported(a);
  const long long max_comp = a.has_comp ? (a.sel ? a.k : a.max_entries) : 0;
  const AttnPlan p =
      attn_plan(rows, max_comp, a.window, tc ? attn_tc_unit_keys(rows, max_comp + a.window) : kChunk);
  const bool direct = p.splits == 1;
  float *part_o = direct ? a.out : reinterpret_cast<float *>(a.ws);
  float *part_lse = a.lse;
  if (!direct) {
    part_lse = part_o + (size_t)rows * p.splits * a.Hq * a.Dv;
    part_lse = reinterpret_cast<float *>(((uintptr_t)part_lse + 255) & ~(uintptr_t)255);
  }
  if (tc) {
    const int rc = launch_attn_tc(a, p, part_o, part_lse, st);
    if (rc != CSKV_OK) return rc;
  } else {
    const bool sep_v = a.win_v.data != nullptr;
    const size_t smem = sizeof(float) * ((size_t)a.Hq * a.D + (size_t)kChunk * (a.D + 1) +
                                         (sep_v ? (size_t)kChunk * (a.Dv + 1) : 0) +
                                         (size_t)a.Hq * kChunk + (size_t)a.Hq * a.Dv +
                                         3 * (size_t)a.Hq);
    if (!ensure_dynamic_smem(attn_units_kernel, smem)) return CSKV_ERR_UNSUPPORTED;
    if (launch_pdl(attn_units_kernel, dim3(rows, p.splits), dim3(kThreads), smem, st, a, p,
                   part_o, part_lse) != cudaSuccess)
      return CSKV_ERR_CUDA;
  }
  if (direct) return CSKV_OK;
  if (launch_pdl(attn_merge_kernel,
                 dim3((unsigned)(rows * a.Hq), (a.Dv + 4 * kMergeQuads - 1) / (4 * kMergeQuads)),
                 dim3(kMergeThreads), 0, st, a.Hq, a.Dv, p.splits, (const float *)part_o,
                 (const float *)part_lse, a.out, a.lse) != cudaSuccess)
    return CSKV_ERR_CUDA;
  return CSKV_OK;
}

}  // namespace cskv
