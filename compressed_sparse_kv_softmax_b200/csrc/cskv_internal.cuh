// Internal device/host helpers shared by the kernels of libcskv.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "cskv.h"

namespace cskv {

// FP4 E2M1 (low 4 bits of `code`) times the E8M0 scale 2^(e - 127); e = 255
// (the E8M0 NaN) gives NaN.  E2M1: sign, 2 exponent bits (bias 1), 1 mantissa
// bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__host__ __device__ __forceinline__ float e2m1_decode(uint32_t code) {
  const uint32_t m = code & 7u;
  const float mag = m < 2 ? 0.5f * (float)m : (float)(2u + (m & 1u)) * (float)(1u << ((m >> 1) - 1)) * 0.5f;
  return (code & 8u) ? -mag : mag;
}
__device__ __forceinline__ float mxfp4_value(uint32_t code, uint8_t e) {
  return e == 255 ? __int_as_float(0x7fffffff) : ldexpf(e2m1_decode(code), (int)e - 127);
}

// Checked build (compiled with -DCSKV_CHECK, libcskv_check.so): every index
// a kernel takes from device memory (a selected entry, a block-table entry, a
// position that names a ring slot or a cache entry) is tested against its
// range before the access; a failed test records CSKV_DEV_BOUNDS in the
// device status word and the access is left out, as the regular build leaves
// it out (or keeps it inside the planes) without saying so.
#ifdef CSKV_CHECK
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

// Sticky per-device status word (status.cu): kernels OR CSKV_DEV_* bits into
// it when a bounded wait runs out (and, in the checked build, when an index
// fails its test).  device_status_word() is its device address on the
// current device (nullptr if the lookup failed).
unsigned int *device_status_word();
__device__ __forceinline__ void record_event(unsigned int *status, unsigned int bit) {
  if (status) atomicOr(status, bit);
}

// Device-side view of a cskv_cache (passed to kernels by value).
// Tiles of a paged key cache whose first rows a scoring CTA resolves up front
// (the producer warp's lanes together, into shared memory), so that no tile
// waits on its block-table load; later tiles read the table when they come.
constexpr int kPagedTiles = 64;

// How a kernel maps a slot to its plane row: kRowAuto looks at the cache
// (block table or not), kRowFlat is the contiguous layout only (rings, and
// the instantiations of the latency-bound kernels that leave paging out so
// that their code stays as small as before).
constexpr int kRowAuto = 0, kRowFlat = 1;

// (kept at 72 bytes: kernels that hand a descriptor to an out-of-line
// helper copy it per thread, and the cold-cache compressor felt every byte)
struct Cache {
  int16_t fmt, d_nope, d_rope, ring;
  int32_t bs_log2, nblk;      // paged layout: 2^bs_log2 slots per block, nblk blocks
  long long cap;
  uint8_t *data, *scale, *rope;
  int32_t data_stride, scale_stride, rope_stride;   // bytes
  // paged layout: bt [B][cap >> bs_log2] physical block ids (nullptr: rows
  // b * cap + slot)
  const int32_t *bt;
#ifdef CSKV_CHECK
  unsigned int *status;       // checked build: where a failed index test is recorded
#endif

  // checked build: records CSKV_DEV_BOUNDS when `ok` is false; returns `ok`
  __device__ __forceinline__ bool check(bool ok) const {
#ifdef CSKV_CHECK
    if (!ok) record_event(status, CSKV_DEV_BOUNDS);
#endif
    return ok;
  }

  __host__ __device__ int dims() const { return d_nope + d_rope; }
  // scales per slot, the dims each covers, and the bytes they take
  // (fp32 scales; one E8M0 byte per 32 dims for MXFP4)
  __host__ __device__ int n_scales() const {
    return fmt == CSKV_FMT_E4M3_VEC ? 1 : (fmt == CSKV_FMT_MXFP4 ? d_nope >> 5 : d_nope >> 6);
  }
  __host__ __device__ int scale_block() const {
    return fmt == CSKV_FMT_E4M3_VEC ? d_nope : (fmt == CSKV_FMT_MXFP4 ? 32 : 64);
  }
  __host__ __device__ int scale_bytes() const {
    return fmt == CSKV_FMT_MXFP4 ? n_scales() : 4 * n_scales();
  }
  // bytes of the data plane that a slot's values take
  __host__ __device__ int data_bytes() const {
    return fmt == CSKV_FMT_F32 ? 4 * dims() : (fmt == CSKV_FMT_MXFP4 ? d_nope >> 1 : d_nope);
  }
  // plane row of a slot (device: the block table lives in device memory)
  template <int M = kRowAuto>
  __device__ long long row(int b, long long slot) const {
    if (M == kRowFlat || !bt) return (long long)b * cap + slot;
    long long blk = bt[(long long)b * (cap >> bs_log2) + (slot >> bs_log2)];
    // (a slot that is read or written has a block; a bad table stays in bounds)
    if (!check(blk >= 0 && blk < nblk)) blk = blk < 0 ? 0 : nblk - 1;
    return (blk << bs_log2) + (slot & ((1LL << bs_log2) - 1));
  }
  // whether slot s of sequence b has a block (always, unpaged)
  __device__ bool mapped(int b, long long slot) const {
    if (!bt) return true;
    const long long blk = bt[(long long)b * (cap >> bs_log2) + (slot >> bs_log2)];
    return blk >= 0 && blk < nblk;
  }
  // plane row of slot j0 of sequence b, the first of a run of slots that
  // stays inside one block (paged: j0's block names a block of the planes);
  // `invalid` when the block table names none (a slot past the sequence's
  // allocation)
  __device__ long long run_row0(int b, long long j0, long long invalid) const {
    if (!bt) return (long long)b * cap + j0;
    const long long blk = bt[(long long)b * (cap >> bs_log2) + (j0 >> bs_log2)];
    if (blk < 0 || blk >= nblk) return invalid;
    return (blk << bs_log2) + (j0 & ((1LL << bs_log2) - 1));
  }
  // rows the planes hold (B sequences of cap slots, or the block pool)
  __host__ __device__ long long plane_rows(int B) const {
    return bt ? ((long long)nblk << bs_log2) : (long long)B * cap;
  }
  // slot holding token position p (ring) or entry j (compressed cache)
  __host__ __device__ long long slot_of(long long p) const { return ring ? (p % cap) : p; }
  template <int M = kRowAuto>
  __device__ const uint8_t *data_ptr(int b, long long slot) const {
    return data + row<M>(b, slot) * data_stride;
  }
  template <int M = kRowAuto>
  __device__ const float *scale_ptr(int b, long long slot) const {
    return reinterpret_cast<const float *>(scale + row<M>(b, slot) * scale_stride);
  }
  template <int M = kRowAuto>
  __device__ const __nv_bfloat16 *rope_ptr(int b, long long slot) const {
    return reinterpret_cast<const __nv_bfloat16 *>(rope + row<M>(b, slot) * rope_stride);
  }
  // dequantised value of dim d of a slot (scalar path)
  template <int M = kRowAuto>
  __device__ float value(int b, long long slot, int d) const {
    const long long r = row<M>(b, slot);
    const uint8_t *dp = data + r * data_stride;
    if (fmt == CSKV_FMT_F32) return reinterpret_cast<const float *>(dp)[d];
    if (fmt == CSKV_FMT_MXFP4)
      return mxfp4_value(dp[d >> 1] >> ((d & 1) << 2), (scale + r * scale_stride)[d >> 5]);
    if (d < d_nope) {
      __nv_fp8_e4m3 c;
      c.__x = dp[d];
      return float(c) *
             reinterpret_cast<const float *>(scale + r * scale_stride)[fmt == CSKV_FMT_E4M3_VEC ? 0 : d >> 6];
    }
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(rope + r * rope_stride)[d - d_nope]);
  }
};

static_assert(sizeof(Cache) == (kChecked ? 80 : 72), "cache descriptor size");

// (field ranges are checked by the ABI: dims < 2^15, strides and blocks < 2^31)
inline Cache to_dev(const cskv_cache *c) {
  Cache v{};
  if (!c) return v;
  v.fmt = (int16_t)c->fmt; v.d_nope = (int16_t)c->d_nope; v.d_rope = (int16_t)c->d_rope;
  v.ring = (int16_t)c->ring;
  v.cap = c->cap;
  v.data = (uint8_t *)c->data; v.data_stride = (int32_t)c->data_stride;
  v.scale = (uint8_t *)c->scale; v.scale_stride = (int32_t)c->scale_stride;
  v.rope = (uint8_t *)c->rope; v.rope_stride = (int32_t)c->rope_stride;
  v.bt = c->block_table;
  v.bs_log2 = 0;
  while (c->block_table && (1LL << v.bs_log2) < c->block_size) ++v.bs_log2;
  v.nblk = c->block_table ? (int32_t)c->num_blocks : 0;
#ifdef CSKV_CHECK
  v.status = device_status_word();
#endif
  return v;
}

// E4M3 encode: round to nearest even, saturate to +-448 (finite-only format).
__device__ __forceinline__ uint8_t e4m3_encode(float x) {
  return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_decode(uint8_t code) {
  __nv_fp8_e4m3 c;
  c.__x = code;
  return float(c);
}

// Bytes of a key tile's scales that one bulk copy brings: the 16-byte groups
// of a packed scale plane (sb bytes per cache row) from the one holding the
// tile's first row to the last one that lies entirely inside the plane.  The
// copy starts `lead` bytes before the first row's scales; rows whose scales
// the copy does not hold (at most three at the very end of the cache) are
// read with plain loads.
struct ScaleSpan {
  long long src;       // first byte copied, from the plane's start
  uint32_t lead;       // bytes before the tile's first row
  uint32_t bytes;      // bytes copied (a multiple of 16, possibly 0)
};
__host__ __device__ inline ScaleSpan scale_span(long long g0, long long rows, int sb) {
  const long long b0 = g0 * sb, b1 = (g0 + rows) * sb;
  const long long a0 = b0 & ~15LL, a1 = b1 & ~15LL;
  ScaleSpan sp;
  sp.src = a0;
  sp.lead = (uint32_t)(b0 - a0);
  sp.bytes = a1 > a0 ? (uint32_t)(a1 - a0) : 0u;
  return sp;
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key):
// negative values have every bit flipped, others only the sign bit, so
// -inf < finite < +inf, with NaN patterns beyond the infinities of their
// sign (the canonical NaN of fp32 arithmetic is positive).  Written
// branch-free with an arithmetic shift: the equivalent select on the sign bit
// was measured to map NaN to its own bit pattern (the key of -0.0's
// neighbourhood) in this toolchain's code for sm_100a.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Drop a dead 128-byte line of scratch memory from L2 without writing it back
// to HBM (its contents become undefined).  `p` is 128-byte aligned.
__device__ __forceinline__ void discard_l2_line(const void *p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// Opt a kernel in to `bytes` of dynamic shared memory (host, idempotent).
// Returns false when the request does not fit next to the kernel's static
// shared memory.  Clears the error it may leave behind.
template <typename K>
inline bool ensure_dynamic_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return true;
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if ((size_t)attr.maxDynamicSharedSizeBytes >= bytes) return true;
  int dev = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (bytes + attr.sharedSizeBytes > (size_t)optin) return false;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return true;
}

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation: it may start while the previous
// kernel on the stream is finishing, runs only on-chip set-up (shared memory,
// barriers, TMEM, descriptor prefetch) before pdl_wait(), and touches global
// memory only after it.  pdl_wait() returns once every preceding grid has
// completed and its writes are visible; without a programmatic predecessor it
// returns at once.  pdl_trigger() lets the next kernel begin launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Test hook (cskv_debug_indexer_stall): mbarrier polls that bound every wait
// of a scoring launch whose first CTA leaves out its first tile (0: off).
uint32_t indexer_stall_polls();
// Polls of the multi-CTA selection's row meeting point before a CTA gives up
// (each poll backs off ~0.1-1 us, so the default is seconds).
constexpr uint32_t kDefaultBarrierSpins = 1u << 22;
uint32_t topk_barrier_spins();

// host-side launch helpers (defined in the kernel files)
int launch_compress(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                    const Cache &raw_k, const Cache &raw_v, const Cache &raw_ik,
                    const float *gate_w, const float *gate_b, int pool, int stride,
                    const Cache &out_k, const Cache &out_v, const Cache &out_ik,
                    cudaStream_t st);
int launch_compress_channel(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                            const Cache &raw_k, const Cache &raw_v, const Cache &raw_ik,
                            const float *gate_w, const float *gate_b, const float *gate_w_ik,
                            const float *gate_b_ik, int pool, int stride, const Cache &out_k,
                            const Cache &out_v, const Cache &out_ik, cudaStream_t st);

int launch_ring_store(int B, const int64_t *pos, int n, const Cache *src, const Cache *ring,
                      cudaStream_t st);

struct IndexerArgs {
  int B, Tq, H_I, d_I, stride, k;
  long long max_entries;
  const int64_t *q_pos;
  const void *q_ik; const float *q_ik_scale; const float *head_w;
  Cache ik;
  int32_t *out_idx; float *out_score;
  void *ws; size_t ws_bytes;
  unsigned int *status;    // device status word
  uint32_t stall_polls;    // test hook: 0, or the wait bound of a stalled first CTA
};
size_t indexer_ws_bytes(int B, int Tq, long long max_entries, int k);
// phases of an indexer call: scoring (with the selection histogram) and the
// top-k selection from the scores in the workspace
constexpr int kIndexerScore = 1, kIndexerSelect = 2;
int launch_indexer_topk(const IndexerArgs &a, int phases, cudaStream_t st);

struct AttnArgs {
  int B, Tq, Hq, D, Dv;
  float sm_scale;
  const int64_t *pos;      // q_pos [B][Tq] or ctx_len [B] (decode)
  int pos_is_ctx_len;      // 1: pos[b] = tokens incl. the query (decode)
  const void *q;
  Cache comp_k, comp_v;    // comp_k.data == nullptr -> window only
  int has_comp, comp_stride;
  const int32_t *sel; int k;
  long long max_entries;
  Cache win_k, win_v;
  int window;
  float *out, *lse;
  void *ws; size_t ws_bytes;
  unsigned int *status;    // device status word
};
// How one query row's key list is cut into units and units into splits (one
// CTA per split).  A split runs its units with an online softmax; with one
// split per row the kernel writes the final output, otherwise each split
// writes a partial (o, lse) that attn_merge_kernel combines.
struct AttnPlan {
  int unit;           // keys per unit
  int n_comp_units;   // units of the compressed part (the window's follow)
  int n_units;
  int per_cta;        // units per split
  int splits;         // splits per row
};
AttnPlan attn_plan(long long rows, long long max_comp, int window, int unit);
size_t attn_ws_bytes(int B, int Tq, int Hq, int Dv, long long max_entries, int window);
int launch_attention(const AttnArgs &a, cudaStream_t st);

}  // namespace cskv
