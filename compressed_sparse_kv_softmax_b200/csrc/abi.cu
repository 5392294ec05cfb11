// extern "C" entry points of libcskv.so: host-side argument checks, then the
// launchers.  Nothing is enqueued when a check fails.
#include <cstdint>

#include <nvtx3/nvToolsExt.h>

#include "cskv_internal.cuh"

using namespace cskv;

// most query rows (B x Tq) of one indexer call
constexpr int64_t kMaxIndexerRows = 65535;

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// An NVTX range named for the entry point around each call (host side: it
// brackets the checks and the launches, not the kernels' device time); with
// no profiler attached a push and a pop cost a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};
#define CSKV_RANGE() const NvtxRange nvtx_range_(__func__)

// ring: 1 / 0 required value, -1 either
int check_cache(const cskv_cache *c, int ring) {
  if (!c || !c->data) return CSKV_ERR_ARG;
  if (ring >= 0 && c->ring != ring) return CSKV_ERR_ARG;
  if (c->cap < 1 || c->d_nope < 0 || c->d_rope < 0 || c->d_nope + c->d_rope < 1)
    return CSKV_ERR_ARG;
  // (the device descriptor holds dims in 16 bits and strides in 32)
  if (c->d_nope > 16384 || c->d_rope > 16384 || c->data_stride < 0 || c->scale_stride < 0 ||
      c->rope_stride < 0 || c->data_stride >= (1LL << 31) || c->scale_stride >= (1LL << 31) ||
      c->rope_stride >= (1LL << 31))
    return CSKV_ERR_ARG;
  if (c->block_table) {
    // paged: compressed caches only, power-of-two blocks dividing cap
    if (c->ring || c->block_size < 1 || (c->block_size & (c->block_size - 1)) ||
        c->cap % c->block_size || c->num_blocks < 1 || c->num_blocks > (1LL << 31) - 1 ||
        ((uintptr_t)c->block_table & 3))
      return CSKV_ERR_ARG;
  }
  if (!aligned16(c->data) || c->data_stride % 16) return CSKV_ERR_ARG;
  if (c->fmt == CSKV_FMT_F32) {
    if (c->data_stride < 4LL * (c->d_nope + c->d_rope)) return CSKV_ERR_ARG;
    return CSKV_OK;
  }
  if (c->fmt == CSKV_FMT_MXFP4) {
    // packed E2M1 codes, one E8M0 byte per 32 dims (whole 4-byte groups)
    if (c->d_nope < 128 || c->d_nope % 128 || c->d_rope) return CSKV_ERR_UNSUPPORTED;
    if (c->data_stride < c->d_nope / 2) return CSKV_ERR_ARG;
    if (!c->scale || !aligned16(c->scale) || c->scale_stride % 4 ||
        c->scale_stride < c->d_nope / 32)
      return CSKV_ERR_ARG;
    return CSKV_OK;
  }
  if (c->fmt != CSKV_FMT_E4M3_BF16 && c->fmt != CSKV_FMT_E4M3_VEC) return CSKV_ERR_UNSUPPORTED;
  if (c->d_nope < 64 || c->d_nope % 64) return CSKV_ERR_UNSUPPORTED;
  if (c->fmt == CSKV_FMT_E4M3_VEC && c->d_rope) return CSKV_ERR_UNSUPPORTED;
  if (c->data_stride < c->d_nope) return CSKV_ERR_ARG;
  const long long n_scales = c->fmt == CSKV_FMT_E4M3_VEC ? 1 : c->d_nope / 64;
  if (!c->scale || !aligned16(c->scale) || c->scale_stride % 4 || c->scale_stride < 4LL * n_scales)
    return CSKV_ERR_ARG;
  if (c->d_rope) {
    if (c->d_rope % 8) return CSKV_ERR_UNSUPPORTED;
    if (!c->rope || !aligned16(c->rope) || c->rope_stride % 16 ||
        c->rope_stride < 2LL * c->d_rope)
      return CSKV_ERR_ARG;
  }
  return CSKV_OK;
}

bool same_layout(const cskv_cache *a, const cskv_cache *b) {
  return a->fmt == b->fmt && a->d_nope == b->d_nope && a->d_rope == b->d_rope;
}

int check_ws(const void *ws, size_t have, size_t need) {
  if (need == 0) return CSKV_OK;
  if (!ws || ((uintptr_t)ws & 255u) || have < need) return CSKV_ERR_WORKSPACE;
  return CSKV_OK;
}

#define CSKV_TRY(x)               \
  do {                            \
    const int _rc = (x);          \
    if (_rc != CSKV_OK) return _rc; \
  } while (0)

// channel = 0: one scalar gate per token (gate_b [pool]); channel = 1: one
// gate per channel (gate_b [pool][D], the indexer keys with gate_w_ik [d_I]
// and gate_b_ik [pool][d_I])
int compress_common(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                    const cskv_cache *raw_k, const cskv_cache *raw_v, const cskv_cache *raw_ik,
                    const float *gate_w, const float *gate_b, const float *gate_w_ik,
                    const float *gate_b_ik, int channel, int pool, int stride,
                    const cskv_cache *out_k, const cskv_cache *out_v, const cskv_cache *out_ik,
                    cskv_stream_t stream) {
  if (B < 0 || B > 65535 || max_new < 0 || max_new > 0x7fffffffLL) return CSKV_ERR_ARG;
  if (B == 0 || max_new == 0) return CSKV_OK;
  if (!t_begin || !t_end || !gate_w || !gate_b) return CSKV_ERR_ARG;
  if (stride < 1 || pool < stride || pool > 4096) return CSKV_ERR_ARG;
  CSKV_TRY(check_cache(raw_k, 1));
  CSKV_TRY(check_cache(out_k, 0));
  if (!same_layout(raw_k, out_k)) return CSKV_ERR_ARG;
  if ((raw_v == nullptr) != (out_v == nullptr)) return CSKV_ERR_ARG;
  if ((raw_ik == nullptr) != (out_ik == nullptr)) return CSKV_ERR_ARG;
  const cskv_cache *rings[3] = {raw_k, raw_v, raw_ik};
  const cskv_cache *outs[3] = {out_k, out_v, out_ik};
  for (int i = 1; i < 3; ++i) {
    if (!rings[i]) continue;
    CSKV_TRY(check_cache(rings[i], 1));
    CSKV_TRY(check_cache(outs[i], 0));
    if (!same_layout(rings[i], outs[i])) return CSKV_ERR_ARG;
    // V shares K's format; the indexer keys may take either E4M3 layout
    // beside an E4M3 KV cache, fp32 beside an fp32 one
    if (i == 1 ? rings[i]->fmt != raw_k->fmt
               : (rings[i]->fmt == CSKV_FMT_F32) != (raw_k->fmt == CSKV_FMT_F32))
      return CSKV_ERR_ARG;
  }
  for (int i = 0; i < 3; ++i) {
    if (!rings[i]) continue;
    if (rings[i]->cap < (max_new - 1) * (int64_t)stride + pool) return CSKV_ERR_ARG;
    if (outs[i]->cap < max_new) return CSKV_ERR_ARG;
  }
  if (channel) {
    // the value is pooled with the key's per-channel weights: same channels
    if (raw_v && raw_v->d_nope + raw_v->d_rope != raw_k->d_nope + raw_k->d_rope)
      return CSKV_ERR_ARG;
    if (raw_ik && (!gate_w_ik || !gate_b_ik)) return CSKV_ERR_ARG;
    return launch_compress_channel(B, t_begin, t_end, max_new, to_dev(raw_k), to_dev(raw_v),
                                   to_dev(raw_ik), gate_w, gate_b, gate_w_ik, gate_b_ik, pool,
                                   stride, to_dev(out_k), to_dev(out_v), to_dev(out_ik),
                                   (cudaStream_t)stream);
  }
  return launch_compress(B, t_begin, t_end, max_new, to_dev(raw_k), to_dev(raw_v),
                         to_dev(raw_ik), gate_w, gate_b, pool, stride, to_dev(out_k),
                         to_dev(out_v), to_dev(out_ik), (cudaStream_t)stream);
}

int attention_common(int B, int Tq, const int64_t *pos, int pos_is_ctx_len, const void *q,
                     int Hq, float sm_scale, const cskv_cache *comp_k, const cskv_cache *comp_v,
                     int comp_stride, const int32_t *sel, int k, int64_t max_entries,
                     const cskv_cache *win_k, const cskv_cache *win_v, int window, float *out,
                     float *lse, void *ws, size_t ws_bytes, cskv_stream_t stream) {
  if (B < 0 || Tq < 0 || (int64_t)B * Tq > 0x7fffffffLL) return CSKV_ERR_ARG;
  if (Hq < 1 || Hq > 65535 || window < 1) return CSKV_ERR_ARG;
  if ((int64_t)B * Tq * Hq > 0x7fffffffLL) return CSKV_ERR_ARG;
  if (B == 0 || Tq == 0) return CSKV_OK;
  if (!pos || !q || !out || !lse || !aligned16(q)) return CSKV_ERR_ARG;
  CSKV_TRY(check_cache(win_k, 1));
  if (win_k->cap < window) return CSKV_ERR_ARG;
  if (win_v) {
    CSKV_TRY(check_cache(win_v, 1));
    if (win_v->fmt != win_k->fmt || win_v->cap != win_k->cap) return CSKV_ERR_ARG;
  }
  int64_t max_comp = 0;
  if (comp_k) {
    CSKV_TRY(check_cache(comp_k, 0));
    if (!same_layout(comp_k, win_k) || comp_stride < 1) return CSKV_ERR_ARG;
    if ((comp_v == nullptr) != (win_v == nullptr)) return CSKV_ERR_ARG;
    if (comp_v) {
      CSKV_TRY(check_cache(comp_v, 0));
      if (!same_layout(comp_v, win_v)) return CSKV_ERR_ARG;
    }
    if (sel) {
      if (k < 1 || max_entries < k) return CSKV_ERR_ARG;
      max_comp = k;
    } else {
      if (max_entries < 0 || max_entries > comp_k->cap) return CSKV_ERR_ARG;
      if (comp_v && max_entries > comp_v->cap) return CSKV_ERR_ARG;
      max_comp = max_entries;
    }
  } else if (comp_v || sel) {
    return CSKV_ERR_ARG;
  }
  AttnArgs a{};
  a.B = B; a.Tq = Tq; a.Hq = Hq;
  a.D = win_k->d_nope + win_k->d_rope;
  a.Dv = win_v ? win_v->d_nope + win_v->d_rope : a.D;
  a.sm_scale = sm_scale;
  a.pos = pos; a.pos_is_ctx_len = pos_is_ctx_len;
  a.q = q;
  a.comp_k = to_dev(comp_k); a.comp_v = to_dev(comp_v ? comp_v : comp_k);
  a.has_comp = comp_k != nullptr; a.comp_stride = comp_stride;
  a.sel = sel; a.k = sel ? k : 0;
  a.max_entries = max_comp;
  a.win_k = to_dev(win_k);
  a.win_v = to_dev(win_v);
  a.window = window;
  a.out = out; a.lse = lse; a.ws = ws; a.ws_bytes = ws_bytes;
  CSKV_TRY(check_ws(ws, ws_bytes, attn_ws_bytes(B, Tq, Hq, a.Dv, max_comp, window)));
  a.status = device_status_word();
  if (!a.status) return CSKV_ERR_CUDA;
  return launch_attention(a, (cudaStream_t)stream);
}

int indexer_common(int phases, int B, int Tq, const int64_t *q_pos, const void *q_ik,
                   const float *q_ik_scale, const float *head_w, int H_I, int d_I,
                   const cskv_cache *ik, int stride, int k, int64_t max_entries,
                   int32_t *out_idx, float *out_score, void *ws, size_t ws_bytes,
                   cskv_stream_t stream) {
  if (B < 0 || Tq < 0 || (int64_t)B * Tq > 0x7fffffffLL) return CSKV_ERR_ARG;
  if (k < 1 || k > 4096 || stride < 1 || H_I < 1 || d_I < 1 || max_entries < 0)
    return CSKV_ERR_ARG;
  // query rows run along a grid's y dimension in the scoring and selection
  // kernels: at most 65,535 per call (larger batches are split by the caller)
  if ((int64_t)B * Tq > kMaxIndexerRows) return CSKV_ERR_UNSUPPORTED;
  if (B == 0 || Tq == 0) return CSKV_OK;
  if (!q_pos || !q_ik || !head_w || !out_idx || !aligned16(q_ik)) return CSKV_ERR_ARG;
  CSKV_TRY(check_cache(ik, 0));
  if (ik->d_rope != 0 || ik->d_nope != d_I || max_entries > ik->cap) return CSKV_ERR_ARG;
  if (ik->fmt == CSKV_FMT_E4M3_BF16 || ik->fmt == CSKV_FMT_E4M3_VEC ||
      ik->fmt == CSKV_FMT_MXFP4) {
    if (!q_ik_scale) return CSKV_ERR_ARG;
  } else if (q_ik_scale) {
    return CSKV_ERR_ARG;
  }
  if ((size_t)H_I * d_I * 4 + (size_t)H_I * 4 + 128ull * (d_I + 1) * 4 > 200 * 1024)
    return CSKV_ERR_UNSUPPORTED;
  CSKV_TRY(check_ws(ws, ws_bytes, indexer_ws_bytes(B, Tq, max_entries, k)));
  IndexerArgs a{};
  a.B = B; a.Tq = Tq; a.H_I = H_I; a.d_I = d_I; a.stride = stride; a.k = k;
  a.max_entries = max_entries;
  a.q_pos = q_pos; a.q_ik = q_ik; a.q_ik_scale = q_ik_scale; a.head_w = head_w;
  a.ik = to_dev(ik);
  a.out_idx = out_idx; a.out_score = out_score;
  a.ws = ws; a.ws_bytes = ws_bytes;
  a.status = device_status_word();
  if (!a.status) return CSKV_ERR_CUDA;
  a.stall_polls = indexer_stall_polls();
  return launch_indexer_topk(a, phases, (cudaStream_t)stream);
}

}  // namespace

extern "C" {

int csa_compress(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                 const cskv_cache *raw_k, const cskv_cache *raw_v, const cskv_cache *raw_ik,
                 const float *gate_w, const float *gate_b, int pool, int stride,
                 const cskv_cache *out_k, const cskv_cache *out_v, const cskv_cache *out_ik,
                 cskv_stream_t stream) {
  CSKV_RANGE();
  return compress_common(B, t_begin, t_end, max_new, raw_k, raw_v, raw_ik, gate_w, gate_b,
                         nullptr, nullptr, 0, pool, stride, out_k, out_v, out_ik, stream);
}

int csa_compress_channel_gate(int B, const int64_t *t_begin, const int64_t *t_end,
                              int64_t max_new, const cskv_cache *raw_k, const cskv_cache *raw_v,
                              const cskv_cache *raw_ik, const float *gate_w, const float *gate_b,
                              const float *gate_w_ik, const float *gate_b_ik, int pool,
                              int stride, const cskv_cache *out_k, const cskv_cache *out_v,
                              const cskv_cache *out_ik, cskv_stream_t stream) {
  CSKV_RANGE();
  return compress_common(B, t_begin, t_end, max_new, raw_k, raw_v, raw_ik, gate_w, gate_b,
                         gate_w_ik, gate_b_ik, 1, pool, stride, out_k, out_v, out_ik, stream);
}

int hca_compress(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                 const cskv_cache *raw_k, const cskv_cache *raw_v, const float *gate_w,
                 const float *gate_b, int pool, int stride, const cskv_cache *out_k,
                 const cskv_cache *out_v, cskv_stream_t stream) {
  CSKV_RANGE();
  return compress_common(B, t_begin, t_end, max_new, raw_k, raw_v, nullptr, gate_w, gate_b,
                         nullptr, nullptr, 0, pool, stride, out_k, out_v, nullptr, stream);
}

int hca_compress_channel_gate(int B, const int64_t *t_begin, const int64_t *t_end,
                              int64_t max_new, const cskv_cache *raw_k, const cskv_cache *raw_v,
                              const float *gate_w, const float *gate_b, int pool, int stride,
                              const cskv_cache *out_k, const cskv_cache *out_v,
                              cskv_stream_t stream) {
  CSKV_RANGE();
  return compress_common(B, t_begin, t_end, max_new, raw_k, raw_v, nullptr, gate_w, gate_b,
                         nullptr, nullptr, 1, pool, stride, out_k, out_v, nullptr, stream);
}

int cskv_ring_store(int B, const int64_t *pos, int n, const cskv_cache *const *src,
                    const cskv_cache *const *ring, cskv_stream_t stream) {
  CSKV_RANGE();
  if (B < 0 || B > 65535 || n < 1 || n > 8) return CSKV_ERR_ARG;
  if (B == 0) return CSKV_OK;
  if (!pos || !src || !ring) return CSKV_ERR_ARG;
  Cache s[8], r[8];
  for (int i = 0; i < n; ++i) {
    CSKV_TRY(check_cache(src[i], 0));
    CSKV_TRY(check_cache(ring[i], 1));
    if (!same_layout(src[i], ring[i])) return CSKV_ERR_ARG;
    s[i] = to_dev(src[i]);
    r[i] = to_dev(ring[i]);
  }
  return launch_ring_store(B, pos, n, s, r, (cudaStream_t)stream);
}

size_t cskv_indexer_workspace_size(int B, int Tq, int64_t max_entries, int k) {
  if (B <= 0 || Tq <= 0 || max_entries < 0) return 0;
  return indexer_ws_bytes(B, Tq, max_entries, k);
}

int indexer_topk(int B, int Tq, const int64_t *q_pos, const void *q_ik, const float *q_ik_scale,
                 const float *head_w, int H_I, int d_I, const cskv_cache *ik, int stride, int k,
                 int64_t max_entries, int32_t *out_idx, float *out_score, void *ws,
                 size_t ws_bytes, cskv_stream_t stream) {
  CSKV_RANGE();
  return indexer_common(kIndexerScore | kIndexerSelect, B, Tq, q_pos, q_ik, q_ik_scale, head_w,
                        H_I, d_I, ik, stride, k, max_entries, out_idx, out_score, ws, ws_bytes,
                        stream);
}

int indexer_score(int B, int Tq, const int64_t *q_pos, const void *q_ik, const float *q_ik_scale,
                  const float *head_w, int H_I, int d_I, const cskv_cache *ik, int stride, int k,
                  int64_t max_entries, int32_t *out_idx, float *out_score, void *ws,
                  size_t ws_bytes, cskv_stream_t stream) {
  CSKV_RANGE();
  return indexer_common(kIndexerScore, B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I, ik,
                        stride, k, max_entries, out_idx, out_score, ws, ws_bytes, stream);
}

int indexer_select(int B, int Tq, const int64_t *q_pos, const void *q_ik, const float *q_ik_scale,
                   const float *head_w, int H_I, int d_I, const cskv_cache *ik, int stride, int k,
                   int64_t max_entries, int32_t *out_idx, float *out_score, void *ws,
                   size_t ws_bytes, cskv_stream_t stream) {
  CSKV_RANGE();
  return indexer_common(kIndexerSelect, B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I, ik,
                        stride, k, max_entries, out_idx, out_score, ws, ws_bytes, stream);
}

size_t cskv_attn_workspace_size(int B, int Tq, int Hq, int Dv, int64_t max_entries, int window) {
  if (B <= 0 || Tq <= 0 || Hq <= 0 || Dv <= 0 || max_entries < 0 || window < 1) return 0;
  return attn_ws_bytes(B, Tq, Hq, Dv, max_entries, window);
}

int hybrid_attn_decode(int B, const int64_t *ctx_len, const void *q, int Hq, float sm_scale,
                       const cskv_cache *comp_k, const cskv_cache *comp_v, int comp_stride,
                       const int32_t *sel, int k, int64_t max_entries, const cskv_cache *win_k,
                       const cskv_cache *win_v, int window, float *out, float *lse, void *ws,
                       size_t ws_bytes, cskv_stream_t stream) {
  CSKV_RANGE();
  return attention_common(B, 1, ctx_len, 1, q, Hq, sm_scale, comp_k, comp_v, comp_stride, sel, k,
                          max_entries, win_k, win_v, window, out, lse, ws, ws_bytes, stream);
}

int hybrid_attn_prefill(int B, int Tq, const int64_t *q_pos, const void *q, int Hq,
                        float sm_scale, const cskv_cache *comp_k, const cskv_cache *comp_v,
                        int comp_stride, const int32_t *sel, int k, int64_t max_entries,
                        const cskv_cache *win_k, const cskv_cache *win_v, int window,
                        float *out, float *lse, void *ws, size_t ws_bytes,
                        cskv_stream_t stream) {
  CSKV_RANGE();
  return attention_common(B, Tq, q_pos, 0, q, Hq, sm_scale, comp_k, comp_v, comp_stride, sel, k,
                          max_entries, win_k, win_v, window, out, lse, ws, ws_bytes, stream);
}

const char *cskv_error_string(int status) {
  switch (status) {
    case CSKV_OK: return "ok";
    case CSKV_ERR_ARG: return "invalid argument (null pointer, shape, alignment or size bound)";
    case CSKV_ERR_UNSUPPORTED: return "unsupported format or dimension combination";
    case CSKV_ERR_CUDA: return "CUDA kernel launch failed";
    case CSKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case CSKV_ERR_SCRATCH_LIMIT:
      return "request needs more scratch than indexer_topk_noalloc's fixed array holds";
    case CSKV_ERR_DEVICE:
      return "a kernel recorded a device-side event (a bounded wait ran out or a row failed)";
    default: return "unknown status";
  }
}

int cskv_version(void) { return 100; }

int cskv_build_checked(void) { return kChecked ? 1 : 0; }

}  // extern "C"
