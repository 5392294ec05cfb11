/*
 * cskv.h - C ABI of the B200 (sm_100a) hybrid compressed sparse KV attention
 * library (libcskv.so).
 *
 * What it computes (DeepSeek-V4 hybrid attention as described on the pages):
 *  - CSA compresses the KV sequence 4x by softmax-gated pooling with a learned
 *    positional bias, over windows that overlap across group boundaries; a
 *    lightning indexer scores every CSA entry at low precision and the top-k
 *    (512 for V4-Flash, 1,024 for V4-Pro) are attended sparsely.
 *    («DeepSeek-V4: 1 Million Token Context endlich nutzbar», section "Hybrid
 *    Attention: CSA und HCA"; «DeepSeek V4-Pro: Architektur,
 *    KV-Cache-Kompression und Hyper-Connections im Detail», section
 *    "Kompression und Selektion"; «Chinas KI-Unabhaengigkeit?: Bei Deepseek V4
 *    haben kleine Aenderungen grosse Wirkung», section "Komprimierte
 *    Erinnerung fuer laengere Kontexte".)
 *  - HCA compresses 128x and attends densely over all compressed entries
 *    (same sections).
 *  - Both add the raw last-128-token sliding window, merged with the
 *    compressed part through log-sum-exp into one softmax over the union
 *    (golem.de section above; webconsulting.at "Das Wichtigste").
 *  - Cache entries store the non-RoPE dims as FP8 E4M3 and the last 64 (RoPE)
 *    dims as BF16 (chaosnode.de and golem.de sections above).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    allocates nothing, keeps no state between calls and never synchronises
 *    the stream; work is enqueued on `stream` (NULL = legacy default stream).
 *  - Per-step sizes that change from step to step (token counts, positions)
 *    are DEVICE int64 arrays, so a decode step can be captured in a CUDA graph.
 *    Host-side bounds (max_new, max_entries) size the launch grids.
 *  - Arguments are checked on the host before anything is enqueued; on an
 *    argument error nothing is launched and a negative status is returned.
 *  - Scratch memory comes from the caller's workspace `ws` of `ws_bytes`
 *    bytes (256-byte aligned), sized with the matching *_workspace_size().
 *  - Return value: CSKV_OK or a negative CSKV_ERR_* status; the text of a
 *    status is cskv_error_string(status).  CSKV_ERR_CUDA reports a launch
 *    error (the CUDA error is left pending for the caller to query).
 *  - Every call is thread-safe; concurrent calls must not share outputs or
 *    workspaces.
 */
#ifndef CSKV_H
#define CSKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared opaquely so the header needs no CUDA include. */
typedef struct CUstream_st *cskv_stream_t;

enum {
  CSKV_OK = 0,
  CSKV_ERR_ARG = -1,          /* null pointer, bad shape, misalignment, size bound */
  CSKV_ERR_UNSUPPORTED = -2,  /* valid but not implemented combination of formats/dims */
  CSKV_ERR_CUDA = -3,         /* a kernel launch failed */
  CSKV_ERR_WORKSPACE = -4,    /* ws is NULL, misaligned or smaller than required */
  CSKV_ERR_SCRATCH_LIMIT = -5, /* request larger than indexer_topk_noalloc's fixed scratch */
  CSKV_ERR_DEVICE = -6         /* cskv_check_device_errors: a kernel recorded an event below */
};

/*
 * Device-side events (bits of the sticky per-device status word that
 * cskv_check_device_errors reads).  Every wait inside a kernel is bounded
 * (seconds, far beyond any legitimate wait); when one runs out the kernel
 * records the event, leaves the affected results visibly invalid and
 * returns instead of hanging.
 */
enum {
  CSKV_DEV_INDEXER_WAIT = 1,  /* a scoring CTA gave up waiting on its copy / MMA pipeline;
                                 its scores read NaN and its rows are reported failed */
  CSKV_DEV_TOPK_BARRIER = 2,  /* the selection's per-row meeting point timed out; the row was
                                 selected from its scores by each CTA that gave up
                                 (result unchanged) */
  CSKV_DEV_ATTN_WAIT = 4,     /* an attention CTA gave up waiting on its copies / MMAs;
                                 the affected rows' lse is NaN */
  CSKV_DEV_ROW_FAILED = 8,    /* the selection met a row with a NaN score; that row's
                                 out_idx is all -1 and its out_score all NaN */
  CSKV_DEV_BOUNDS = 16        /* checked build only (cskv_build_checked() == 1): an index
                                 read from device memory failed its range test and the
                                 access was left out.  The tests: a selected entry is -1 or
                                 below both the row's visible count and the cache's
                                 cap; a slot that is read or written has a block in
                                 [0, num_blocks); a visible row needs no more than
                                 max_entries entries; a compressor call has no more than
                                 max_new entries per sequence, each below its caches' cap,
                                 and reads only positions its rings still hold
                                 (p > t_end - 1 - ring cap); a ring_store position is >= 0 */
};

enum {
  CSKV_FMT_F32 = 0,        /* fp32 values, d_nope + d_rope per slot (no scale/rope planes) */
  CSKV_FMT_E4M3_BF16 = 1,  /* d_nope E4M3 codes + d_nope/64 fp32 scales + d_rope BF16 */
  CSKV_FMT_E4M3_VEC = 2,   /* d_nope E4M3 codes + ONE fp32 scale per slot; d_rope = 0 */
  CSKV_FMT_MXFP4 = 3       /* d_nope FP4 E2M1 codes, two per byte + d_nope/32 E8M0 bytes; d_rope = 0 */
};

/*
 * A cache of `cap` slots per sequence, for B sequences stored back to back.
 * Slot s of sequence b starts at  plane + (b * cap + s) * plane_stride  in
 * each plane (strides in BYTES).
 *  - Compressed cache (ring = 0): entry j lives in slot j.
 *  - Raw-token ring   (ring = 1): token position p lives in slot p % cap.
 * E4M3_BF16 layout: value[d] = E4M3(data[d]) * scale[d / 64]  for d < d_nope,
 *                   value[d_nope + r] = BF16(rope[r])          for r < d_rope.
 * E4M3_VEC layout:  value[d] = E4M3(data[d]) * scale[0]        for d < d_nope
 *                   (one scale per vector, no RoPE plane).
 * MXFP4 layout (OCP Microscaling MXFP4, blocks of 32):
 *                   value[d] = E2M1(nibble d of data) * 2^(E[d / 32] - 127),
 *                   nibble d = bits 4*(d%2) .. 4*(d%2)+3 of byte d/2 (the even
 *                   element in the low nibble), E = the bytes of the scale
 *                   plane (the `scale` pointer then addresses uint8 E8M0
 *                   exponents, 255 = NaN); no RoPE plane.  The FP4 lightning
 *                   indexer («DeepSeek-V4: 1 Million Token Context endlich
 *                   nutzbar», "Hybrid Attention: CSA und HCA").
 * The lightning-indexer key cache uses any of the three E4M3 / MXFP4 layouts
 * with d_rope = 0; E4M3_VEC and MXFP4 are the ones the tensor-core scoring
 * path reads fastest (one accumulator per key and head), MXFP4 with half the
 * bytes.
 * Paged layout (block tables; no counterpart on the pages, a serving-side
 * storage choice): with block_table != NULL the planes hold num_blocks
 * blocks of block_size slots shared by all sequences, and slot s of sequence
 * b lives in physical row
 *     block_table[b * (cap / block_size) + s / block_size] * block_size
 *         + s % block_size
 * of every plane (row r starting at plane + r * plane_stride).  Only for
 * compressed caches (ring = 0); block_size a power of two dividing cap;
 * every table entry in [0, num_blocks).  A paged indexer-key cache keeps
 * the tensor-core scoring path when block_size is a multiple of 128 (each
 * 128-entry key tile then lies in one block), else the CUDA-core one; the
 * attention bulk-copies runs of consecutive entries when block_size >= 64.
 * Alignment: data and rope pointers and strides are multiples of 16 bytes;
 * scale pointer 16-byte aligned, scale stride a multiple of 4 bytes and at
 * least 4 * ceil(d_nope / 64) (E4M3_BF16), 4 (E4M3_VEC) or d_nope / 32
 * (MXFP4, d_nope a multiple of 128).  F32: data pointer and stride multiples of 16.
 */
typedef struct cskv_cache {
  int32_t fmt;            /* CSKV_FMT_* */
  int32_t d_nope;         /* E4M3 dims (multiple of 64) or leading fp32 dims */
  int32_t d_rope;         /* BF16 dims, or trailing fp32 dims */
  int32_t ring;           /* 0: slot = entry index; 1: slot = position % cap */
  int64_t cap;            /* slots per sequence */
  void *data;   int64_t data_stride;
  float *scale; int64_t scale_stride;
  void *rope;   int64_t rope_stride;
  /* Paged layout (compressed caches only; block_table NULL: contiguous) */
  const int32_t *block_table;  /* device [B][cap / block_size] physical block ids */
  int64_t block_size;          /* slots per block: a power of two */
  int64_t num_blocks;          /* blocks the planes hold */
} cskv_cache;

/*
 * csa_compress - CSA softmax-gated pooling (4x, overlapping windows).
 * Entry j pools the `pool` raw tokens at positions
 *     stride*(j+1) - pool + r,  r = 0 .. pool-1   (positions < 0 absent),
 * i.e. the previous group and group j for pool = 8, stride = 4.  Gate logits
 *     g_r = gate_w . k_{p_r} + gate_b[r]
 * (gate_w [D] fp32 over the dequantised key, gate_b [pool] fp32 per slot),
 * a = softmax(g) over present slots, entry = sum_r a_r x_{p_r} for the key,
 * the value (raw_v, separate-V layout only) and the raw indexer key (raw_ik)
 * alike.  E4M3 outputs are re-quantised per 64-element block (E4M3_BF16) or
 * per vector (E4M3_VEC) with scale = amax / 448 (1 for an all-zero block),
 * codes rounded to nearest even and saturated; BF16 dims rounded to nearest
 * even.  Each ring has its output's layout; raw_v has raw_k's format; raw_ik
 * is fp32 beside an fp32 raw_k and either E4M3 layout beside an E4M3 one.
 * Writes every entry j with n(t_begin[b]) <= j < n(t_end[b]), n(t) = t / stride,
 * at most max_new per sequence (the host bound that sizes the grid).
 *   t_begin, t_end : [B] device int64; tokens [t_begin, t_end) just arrived.
 *   raw_k, raw_v, raw_ik : rings (ring = 1) holding every position the new
 *       entries read; raw_v and raw_ik may be NULL (K = V; no indexer keys).
 *   out_k, out_v, out_ik : compressed caches (ring = 0) with cap >= n(t_end).
 * Requirements: pool >= stride; cap of each ring >= (max_new - 1) * stride + pool,
 * the span of positions that max_new consecutive entries read (checked on the
 * host).  The rings must still hold those positions when the call runs: a ring
 * that already holds tokens up to t_end - 1 keeps positions >= t_end - cap, so
 * with t_end not a multiple of stride it needs up to stride - 1 more slots
 * (cap >= max_new * stride + pool - 1 covers every t_end).  The kernels do not
 * see which positions a ring holds; the checked build records
 * CSKV_DEV_BOUNDS when an entry's first position is older than t_end - cap.
 */
int csa_compress(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                 const cskv_cache *raw_k, const cskv_cache *raw_v, const cskv_cache *raw_ik,
                 const float *gate_w, const float *gate_b, int pool, int stride,
                 const cskv_cache *out_k, const cskv_cache *out_v, const cskv_cache *out_ik,
                 cskv_stream_t stream);

/*
 * hca_compress - HCA pooling of 128 tokens into one entry by learned weights
 * (pool = stride = 128 on the pages).  Same definition and arguments as
 * csa_compress without the indexer keys.
 */
int hca_compress(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                 const cskv_cache *raw_k, const cskv_cache *raw_v,
                 const float *gate_w, const float *gate_b, int pool, int stride,
                 const cskv_cache *out_k, const cskv_cache *out_v, cskv_stream_t stream);

/*
 * csa_compress_channel_gate / hca_compress_channel_gate - the per-channel
 * gate variant of the same pooling (the pages name a softmax gate with a
 * learned positional bias, «DeepSeek-V4: 1 Million Token Context endlich
 * nutzbar», "Hybrid Attention: CSA und HCA", without its shape; this variant
 * gives every channel its own gate).  For entry j and channel c:
 *     g_{r,c} = gate_w[c] * k_{p_r}[c] + gate_b[r][c]      (present slots r)
 *     a_{.,c} = softmax_r(g_{.,c}),   entry[c] = sum_r a_{r,c} x_{p_r}[c]
 * over the dequantised key k; the value (raw_v, separate-V layout, same
 * channel count as the key) is pooled with the key's weights; the indexer
 * keys have gates of their own read from themselves (gate_w_ik [d_I],
 * gate_b_ik [pool][d_I], both required when raw_ik is given).
 *   gate_w : [D] fp32.   gate_b : [pool][D] fp32 (row r = slot r).
 * Everything else (positions, formats, re-quantisation, requirements) as
 * csa_compress / hca_compress.  The window of every plane is staged in shared
 * memory: CSKV_ERR_UNSUPPORTED when it does not fit (more than 200 KB).
 */
int csa_compress_channel_gate(int B, const int64_t *t_begin, const int64_t *t_end,
                              int64_t max_new, const cskv_cache *raw_k, const cskv_cache *raw_v,
                              const cskv_cache *raw_ik, const float *gate_w, const float *gate_b,
                              const float *gate_w_ik, const float *gate_b_ik, int pool,
                              int stride, const cskv_cache *out_k, const cskv_cache *out_v,
                              const cskv_cache *out_ik, cskv_stream_t stream);
int hca_compress_channel_gate(int B, const int64_t *t_begin, const int64_t *t_end,
                              int64_t max_new, const cskv_cache *raw_k, const cskv_cache *raw_v,
                              const float *gate_w, const float *gate_b, int pool, int stride,
                              const cskv_cache *out_k, const cskv_cache *out_v,
                              cskv_stream_t stream);

/*
 * cskv_ring_store - appends one new raw token per sequence to raw-token
 * rings: for each ring i and sequence b, the token held in slot 0 of
 * sequence b of src[i] (a cache of cap >= 1 slots per sequence, ring = 0)
 * is copied into slot pos[b] % cap of ring[i] (ring = 1), every plane
 * (codes, scales, RoPE) byte for byte.  This is the cache append that
 * precedes csa_compress / hca_compress and the window's attention; the pages
 * keep the last 128 raw tokens for the sliding window («Chinas
 * KI-Unabhaengigkeit?: Bei Deepseek V4 haben kleine Aenderungen grosse
 * Wirkung», "Komprimierte Erinnerung fuer laengere Kontexte").
 *   pos       : [B] device int64, position of each sequence's new token.
 *   n         : number of (src, ring) pairs, 1 <= n <= 8; each pair has one
 *               layout (fmt, d_nope, d_rope) and its planes' alignments.
 * No ring may also be another pair's ring or source.
 */
int cskv_ring_store(int B, const int64_t *pos, int n, const cskv_cache *const *src,
                    const cskv_cache *const *ring, cskv_stream_t stream);

/*
 * indexer_topk - lightning-indexer scores of every visible CSA entry and the
 * top-k selection per query row.
 *   s_j = sum_h head_w[h] * max(0, q_ik[h] . k_ik[j])       (per query row)
 * over visible entries j < n(q_pos + 1) = (q_pos + 1) / stride, then the k
 * highest scores, ties to the lower index; fewer than k visible -> all of
 * them, remaining slots -1.  The indices of one row are written in ascending
 * entry order.
 *   q_pos    : [B][Tq] device int64, position of each query token.
 *   q_ik     : [B][Tq][H_I][d_I]; E4M3 codes when ik->fmt is E4M3_BF16 (with
 *              q_ik_scale [B][Tq][H_I][d_I/64] fp32) or E4M3_VEC (with
 *              q_ik_scale [B][Tq][H_I], one fp32 scale per head), fp32 when
 *              ik->fmt is F32 (q_ik_scale NULL); MXFP4: [B][Tq][H_I][d_I/2]
 *              packed E2M1 codes with q_ik_scale pointing to [B][Tq][H_I][d_I/32]
 *              E8M0 bytes.  16-byte aligned.
 *   head_w   : [B][Tq][H_I] fp32.
 *   ik       : indexer-key cache (ring = 0, d_nope = d_I, d_rope = 0).
 *   k        : selections per row, 1 <= k <= 4096.
 *   max_entries : host bound on visible entries per row (<= ik->cap).
 *   out_idx  : [B][Tq][k] int32.   out_score : [B][Tq][k] fp32 or NULL.
 *   B * Tq   : at most 65,535 query rows per call (CSKV_ERR_UNSUPPORTED
 *              otherwise, before anything is launched); split larger batches.
 *   ws       : cskv_indexer_workspace_size(B, Tq, max_entries, k) bytes.
 *              The scoring leaves a per-row score histogram in it that only
 *              guides the selection (every count is checked against the
 *              scores); the selection clears it for the next call.  A
 *              workspace holding anything else (never zero-filled, or last
 *              used with other shapes) costs its first call time, not
 *              correctness.
 */
int indexer_topk(int B, int Tq, const int64_t *q_pos,
                 const void *q_ik, const float *q_ik_scale, const float *head_w,
                 int H_I, int d_I, const cskv_cache *ik, int stride, int k,
                 int64_t max_entries, int32_t *out_idx, float *out_score,
                 void *ws, size_t ws_bytes, cskv_stream_t stream);

/*
 * indexer_score / indexer_select - the two halves of indexer_topk, for callers
 * that time or schedule the scoring (the HBM stream over every indexer key)
 * apart from the selection (an L2-resident pass over the scores).  Both take
 * exactly indexer_topk's arguments; indexer_score followed by indexer_select
 * on the same stream with the same arguments and workspace is indexer_topk.
 *  - indexer_score writes the scores of every visible entry, and the
 *    histogram the selection starts from, into the workspace; out_idx and
 *    out_score are not written.
 *  - indexer_select reads them and writes out_idx / out_score.  The
 *    workspace must not be used by another call in between.
 * (The pages describe the indexer and the top-k as one step; the split is an
 * interface convenience with no counterpart there.)
 */
int indexer_score(int B, int Tq, const int64_t *q_pos,
                  const void *q_ik, const float *q_ik_scale, const float *head_w,
                  int H_I, int d_I, const cskv_cache *ik, int stride, int k,
                  int64_t max_entries, int32_t *out_idx, float *out_score,
                  void *ws, size_t ws_bytes, cskv_stream_t stream);
int indexer_select(int B, int Tq, const int64_t *q_pos,
                   const void *q_ik, const float *q_ik_scale, const float *head_w,
                   int H_I, int d_I, const cskv_cache *ik, int stride, int k,
                   int64_t max_entries, int32_t *out_idx, float *out_score,
                   void *ws, size_t ws_bytes, cskv_stream_t stream);

size_t cskv_indexer_workspace_size(int B, int Tq, int64_t max_entries, int k);

/*
 * indexer_topk_noalloc - indexer_topk for callers that cannot provide a
 * workspace (no counterpart on the pages: it is a deployment convenience).
 * Callers that may not allocate device memory themselves - a host framework
 * that owns every device allocation through its own pool and passes plug-ins
 * no scratch, a real-time loop that forbids allocation after start-up, an
 * op interface without a workspace argument - use this variant.  Same
 * arguments and results as indexer_topk minus ws/ws_bytes; the scratch is a
 * fixed array of cskv_noalloc_scratch_bytes() (8 MiB) in the library's device
 * memory, held on every GPU that loads the library until the process exits.
 *  - The first call on a device looks the array's address up (once per
 *    device, with that device current); make that first call before any
 *    stream capture.
 *  - A request fits when cskv_indexer_workspace_size(B, Tq, max_entries, k)
 *    <= cskv_noalloc_scratch_bytes(): e.g. up to 7 query rows at a
 *    1,048,576-token context (k = 1,024), or 56 rows at 65,536 tokens
 *    (k = 512).  Larger requests return CSKV_ERR_SCRATCH_LIMIT before
 *    anything is enqueued.
 *  - All calls share the array: calls that may overlap on the GPU (other
 *    streams or host threads on the same device) race and must be serialised
 *    by the caller.  Nothing in the array needs to start at zero, and calls
 *    of different shapes may follow one another.
 *  - It allocates nothing (no cudaMalloc / cudaFree or allocating library call).
 */
int indexer_topk_noalloc(int B, int Tq, const int64_t *q_pos,
                         const void *q_ik, const float *q_ik_scale, const float *head_w,
                         int H_I, int d_I, const cskv_cache *ik, int stride, int k,
                         int64_t max_entries, int32_t *out_idx, float *out_score,
                         cskv_stream_t stream);

/* Size in bytes of indexer_topk_noalloc's fixed scratch array. */
size_t cskv_noalloc_scratch_bytes(void);

/*
 * hybrid_attn_decode - one query token per sequence at position ctx_len-1.
 * Keys: the compressed entries (sel != NULL: the k listed CSA entries, -1
 * skipped; sel == NULL: every visible entry j < ctx_len / comp_stride, HCA)
 * plus the raw window positions max(0, pos-window+1) .. pos, all under one
 * softmax per head:
 *   l = sm_scale * q_h . K,  out_h = sum softmax(l) V,  lse_h = log sum e^l.
 * MQA: all Hq heads share one KV head; K = V = the whole entry unless comp_v /
 * win_v are given (separate-V layout).  comp_k == NULL: window only.
 *   ctx_len : [B] device int64, tokens including the query token.
 *   q       : [B][Hq][D] BF16 for E4M3_BF16 caches, fp32 for F32 caches.
 *   sel     : [B][k] int32 or NULL.   max_entries: host bound on compressed
 *             keys per row (k when sel != NULL; visible entries otherwise).
 *   win_k   : raw ring (ring = 1), cap >= window.
 *   out     : [B][Hq][Dv] fp32.   lse : [B][Hq] fp32 (natural log).
 *   ws      : cskv_attn_workspace_size(B, 1, Hq, Dv, max_entries, window) bytes.
 */
int hybrid_attn_decode(int B, const int64_t *ctx_len, const void *q, int Hq, float sm_scale,
                       const cskv_cache *comp_k, const cskv_cache *comp_v, int comp_stride,
                       const int32_t *sel, int k, int64_t max_entries,
                       const cskv_cache *win_k, const cskv_cache *win_v, int window,
                       float *out, float *lse, void *ws, size_t ws_bytes, cskv_stream_t stream);

/*
 * hybrid_attn_prefill - Tq query tokens per sequence at positions q_pos
 * (chunked prefill); every row uses its own visibility: compressed entries
 * j < (q_pos + 1) / comp_stride (dense) or its own sel row (sparse), and the
 * window max(0, q_pos-window+1) .. q_pos, which makes attention causal inside
 * the chunk.  Same definition and layouts as hybrid_attn_decode with a Tq
 * axis: q [B][Tq][Hq][D], sel [B][Tq][k], out [B][Tq][Hq][Dv], lse [B][Tq][Hq].
 * The ring must hold every position the chunk's windows reach.
 * With comp_k dense (sel == NULL) and several rows per sequence, the call
 * first converts the visible compressed entries once into the workspace
 * (cskv_attn_workspace_size with Tq > 1 includes that space).
 */
int hybrid_attn_prefill(int B, int Tq, const int64_t *q_pos, const void *q, int Hq,
                        float sm_scale, const cskv_cache *comp_k, const cskv_cache *comp_v,
                        int comp_stride, const int32_t *sel, int k, int64_t max_entries,
                        const cskv_cache *win_k, const cskv_cache *win_v, int window,
                        float *out, float *lse, void *ws, size_t ws_bytes, cskv_stream_t stream);

size_t cskv_attn_workspace_size(int B, int Tq, int Hq, int Dv, int64_t max_entries, int window);

/*
 * cskv_check_device_errors - waits for `stream` to finish, then reads and
 * clears the current device's sticky status word: the CSKV_DEV_* events that
 * kernels of this library recorded on the device since the last read (from
 * any stream).  Writes the bits to *events (may be NULL) and returns CSKV_OK
 * when none was recorded, CSKV_ERR_DEVICE when some were, CSKV_ERR_CUDA when
 * the synchronisation or the read failed.  Not for use inside stream capture.
 */
int cskv_check_device_errors(cskv_stream_t stream, uint32_t *events);

/*
 * cskv_debug_topk_barrier_spins - sets how many times a CTA of the multi-CTA
 * top-k selection polls its row's meeting point before it gives up (default
 * 4,194,304, i.e. seconds), and returns the previous setting.  Test hook of
 * the failure path: with 0 a CTA that arrives before the others gives up at
 * once and selects the whole row from its scores (the result is the same)
 * and CSKV_DEV_TOPK_BARRIER is recorded.  Affects later calls in this
 * process, on every device.
 */
uint32_t cskv_debug_topk_barrier_spins(uint32_t spins);

/*
 * cskv_debug_indexer_stall - test hook of the failure path.  With polls > 0,
 * every later tensor-core scoring launch in this process leaves out the copy
 * of the first key tile of its first CTA and bounds
 * every wait of its kernel to `polls` mbarrier polls instead of seconds: that
 * CTA's waits for the missing tile run out, nothing it issued is left in
 * flight, it writes NaN into its score slots, and the selection reports its
 * query rows as failed (row 0; with several query rows per sequence, the
 * group of up to 8 rows of sequence 0 that the CTA scores), recording
 * CSKV_DEV_INDEXER_WAIT and CSKV_DEV_ROW_FAILED.
 * polls = 0 switches it off (the default).  Returns the previous setting.
 */
uint32_t cskv_debug_indexer_stall(uint32_t polls);

/*
 * cskv_build_checked - 1 for the checked build of the library
 * (libcskv_check.so, compiled with -DCSKV_CHECK), whose kernels test every
 * index they read from device memory and record CSKV_DEV_BOUNDS in the status
 * word when one is out of range; 0 for the regular build, whose kernels leave
 * such an access out (or keep it inside the planes) without recording it.
 * Results of valid inputs are the same bits in both builds.
 */
int cskv_build_checked(void);

/* Static text for a status code. */
const char *cskv_error_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int cskv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CSKV_H */
