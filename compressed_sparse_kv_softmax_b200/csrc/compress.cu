// CSA / HCA softmax-gated pooling of raw tokens into compressed cache entries.
//
// Entry j pools the raw tokens at positions stride*(j+1)-pool+r (r < pool,
// positions < 0 absent) with weights a = softmax_r(gate_w . k_{p_r} + gate_b[r])
// and re-quantises the result into the cache format: per 64-element block
// scale = amax/448, E4M3 codes rounded to nearest even with saturation, BF16
// for the RoPE dims.  (CSA: 4x with overlapping windows and a learned
// positional bias, «DeepSeek-V4: 1 Million Token Context endlich nutzbar»,
// "Hybrid Attention: CSA und HCA"; HCA: 128 tokens by learned weights,
// «DeepSeek V4-Pro: Architektur, KV-Cache-Kompression und Hyper-Connections im
// Detail», "Kompression und Selektion".)
//
// (The helpers below are not inlined: the kernel runs on a cold instruction
// cache - once per 4 or 128 tokens - so its time follows the code it fetches,
// and the planes of one entry share one copy of each helper.)
//
// One CTA per (new entry, sequence).  The work is a few KB per entry and runs
// once per 4 (CSA) or 128 (HCA) tokens.  At decode a single entry is written,
// so the latency of the loads decides the time: the staged kernel copies the
// whole pooling window into shared memory with one round of 16-byte loads,
// then computes the gates (one warp per slot), the pooled sums (one thread
// per dim) and the re-quantisation (one warp per 64-element block) from
// shared memory.  Windows too large for shared memory use compress_kernel,
// which reads global memory directly.
#include <math_constants.h>

#include "cskv_internal.cuh"

namespace cskv {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// E2M1 code of x: round to nearest, ties to the even code, saturate to +-6
// (the comparisons put each tie on the even side), sign in bit 3
__device__ __forceinline__ uint32_t e2m1_encode(float x) {
  const float m = fabsf(x);
  const uint32_t c = (m > 0.25f) + (m >= 0.75f) + (m > 1.25f) + (m >= 1.75f) + (m > 2.5f) +
                     (m >= 3.5f) + (m > 5.0f);
  return c | (signbit(x) ? 8u : 0u);
}

// MXFP4 store of one warp's 32-dim block: the OCP MX shared exponent
// X = floor(log2 amax) - 2 (0 for an all-zero block), every element
// E2M1(x / 2^X), two codes per byte (even element in the low nibble)
__device__ __forceinline__ void store_mxfp4_block(uint8_t *codes, uint8_t *exps, int blk,
                                                  float v) {
  const int lane = threadIdx.x & 31;
  const float amax = warp_max(fabsf(v));
  int X = amax > 0.f ? ilogbf(amax) - 2 : 0;
  X = X < -127 ? -127 : (X > 127 ? 127 : X);
  const uint32_t c = e2m1_encode(ldexpf(v, -X));
  const uint32_t hi = __shfl_down_sync(0xffffffffu, c, 1);
  if (!(lane & 1)) codes[blk * 16 + (lane >> 1)] = (uint8_t)(c | (hi << 4));
  if (lane == 0) exps[blk] = (uint8_t)(X + 127);
}

// kPaged: the output cache may be paged (its row comes from the block
// table); the contiguous instantiation carries no paging code
template <bool kPaged>
__device__ __noinline__ void store_entry(const Cache &out, int b, long long j,
                                        const float *pooled, int D) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long orow = out.row<kPaged ? kRowAuto : kRowFlat>(b, j);
  if (out.fmt == CSKV_FMT_F32) {
    float *dst = reinterpret_cast<float *>(out.data + orow * out.data_stride);
    for (int d = tid; d < D; d += kThreads) dst[d] = pooled[d];
    return;
  }
  if (out.fmt == CSKV_FMT_MXFP4) {
    uint8_t *codes = out.data + orow * out.data_stride;
    uint8_t *exps = out.scale + orow * out.scale_stride;
    for (int blk = warp; blk < (out.d_nope >> 5); blk += kWarps)
      store_mxfp4_block(codes, exps, blk, pooled[blk * 32 + lane]);
    return;
  }
  uint8_t *codes = out.data + orow * out.data_stride;
  float *scales = reinterpret_cast<float *>(out.scale + orow * out.scale_stride);
  if (out.fmt == CSKV_FMT_E4M3_VEC) {
    // one scale for the whole vector: warp 0 finds its amax and encodes
    if (warp == 0) {
      float amax = 0.f;
      for (int d = lane; d < out.d_nope; d += 32) amax = fmaxf(amax, fabsf(pooled[d]));
      amax = warp_max(amax);
      const float s = amax > 0.f ? amax / 448.f : 1.f;
      for (int d = lane; d < out.d_nope; d += 32) codes[d] = e4m3_encode(pooled[d] / s);
      if (lane == 0) scales[0] = s;
    }
    return;
  }
  const int nb = out.d_nope >> 6;
  for (int blk = warp; blk < nb; blk += kWarps) {
    const float v0 = pooled[blk * 64 + lane];
    const float v1 = pooled[blk * 64 + 32 + lane];
    const float amax = warp_max(fmaxf(fabsf(v0), fabsf(v1)));
    const float s = amax > 0.f ? amax / 448.f : 1.f;
    codes[blk * 64 + lane] = e4m3_encode(v0 / s);
    codes[blk * 64 + 32 + lane] = e4m3_encode(v1 / s);
    if (lane == 0) scales[blk] = s;
  }
  if (out.d_rope) {
    __nv_bfloat16 *rope =
        reinterpret_cast<__nv_bfloat16 *>(out.rope + orow * out.rope_stride);
    for (int r = tid; r < out.d_rope; r += kThreads)
      rope[r] = __float2bfloat16_rn(pooled[out.d_nope + r]);
  }
}

__device__ void pool_values(const Cache &raw, int b, long long first, int pool, const float *a,
                            float *pooled) {
  const int D = raw.dims();
  for (int d = threadIdx.x; d < D; d += kThreads) {
    float acc = 0.f;
    for (int r = 0; r < pool; ++r) {
      const long long p = first + r;
      if (p < 0) continue;
      acc = fmaf(a[r], raw.value<kRowFlat>(b, raw.slot_of(p), d), acc);
    }
    pooled[d] = acc;
  }
}

// Checked build: the device-side token counts of sequence b against the
// launch and the caches (one thread; nothing in the regular build, whose
// kernels skip what the tests reject without recording it):
//  - the grid's max_new entries per sequence cover n(t_end) - n(t_begin);
//  - entry j lies below every output's cap and has a block in each;
//  - the first position it pools is still held by every ring (a ring of
//    cap slots holds positions t_end - cap .. t_end - 1).
__device__ __forceinline__ void check_entry(const int64_t *t_begin, const int64_t *t_end, int b,
                                            long long j, int pool, int stride,
                                            const Cache &raw_k, const Cache &raw_v,
                                            const Cache &raw_ik, const Cache &out_k,
                                            const Cache &out_v, const Cache &out_ik) {
  if constexpr (kChecked) {
    if (threadIdx.x != 0) return;
    const long long tb = t_begin[b], te = t_end[b], n_end = te / stride;
    if (blockIdx.x == gridDim.x - 1) out_k.check(tb / stride + (long long)gridDim.x >= n_end);
    if (j < 0 || j >= n_end) return;
    const bool in_cap = out_k.check(j < out_k.cap) && (!raw_v.data || out_v.check(j < out_v.cap)) &&
                        (!raw_ik.data || out_ik.check(j < out_ik.cap));
    if (in_cap) {
      out_k.check(out_k.mapped(b, j));
      if (raw_v.data) out_v.check(out_v.mapped(b, j));
      if (raw_ik.data) out_ik.check(out_ik.mapped(b, j));
    }
    long long lo = (long long)stride * (j + 1) - pool;
    lo = lo < 0 ? 0 : lo;
    raw_k.check(lo > te - 1 - raw_k.cap);
    if (raw_v.data) raw_v.check(lo > te - 1 - raw_v.cap);
    if (raw_ik.data) raw_ik.check(lo > te - 1 - raw_ik.cap);
  }
}

template <bool kPaged>
__global__ void __launch_bounds__(kThreads)
compress_kernel(const int64_t *__restrict__ t_begin, const int64_t *__restrict__ t_end,
                Cache raw_k, Cache raw_v,
                Cache raw_ik, const float *__restrict__ gate_w,
                const float *__restrict__ gate_b, int pool, int stride,
                Cache out_k, Cache out_v,
                Cache out_ik) {
  extern __shared__ float smem[];
  pdl_wait();
  pdl_trigger();
  float *a = smem;                 // [pool] gate logits, then weights
  float *pooled = smem + pool;     // [max dims]
  const int b = blockIdx.y;
  const long long j = t_begin[b] / stride + blockIdx.x;
  check_entry(t_begin, t_end, b, j, pool, stride, raw_k, raw_v, raw_ik, out_k, out_v, out_ik);
  if (j >= t_end[b] / stride || j < 0) return;
  // never write past a cache's capacity, whatever the device-side token counts
  // say, nor into a slot that a paged cache's block table leaves without a block
  if (j >= out_k.cap || (raw_v.data && j >= out_v.cap) || (raw_ik.data && j >= out_ik.cap))
    return;
  if (kPaged && (!out_k.mapped(b, j) || (raw_v.data && !out_v.mapped(b, j)) ||
                 (raw_ik.data && !out_ik.mapped(b, j))))
    return;
  const long long first = (long long)stride * (j + 1) - pool;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int D = raw_k.dims();

  // gate logits g_r = gate_w . k_{p_r} + gate_b[r]
  for (int r = warp; r < pool; r += kWarps) {
    const long long p = first + r;
    float acc = 0.f;
    if (p >= 0) {
      const long long slot = raw_k.slot_of(p);
      for (int d = lane; d < D; d += 32)
        acc = fmaf(gate_w[d], raw_k.value<kRowFlat>(b, slot, d), acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) a[r] = p >= 0 ? acc + gate_b[r] : -CUDART_INF_F;
  }
  __syncthreads();
  // softmax over the present slots
  if (warp == 0) {
    float m = -CUDART_INF_F;
    for (int r = lane; r < pool; r += 32) m = fmaxf(m, a[r]);
    m = warp_max(m);
    float s = 0.f;
    for (int r = lane; r < pool; r += 32) s += (a[r] == -CUDART_INF_F) ? 0.f : expf(a[r] - m);
    s = warp_sum(s);
    __syncwarp();
    for (int r = lane; r < pool; r += 32)
      a[r] = (a[r] == -CUDART_INF_F) ? 0.f : expf(a[r] - m) / s;
  }
  __syncthreads();

  pool_values(raw_k, b, first, pool, a, pooled);
  __syncthreads();
  store_entry<kPaged>(out_k, b, j, pooled, D);
  __syncthreads();
  if (raw_v.data) {
    pool_values(raw_v, b, first, pool, a, pooled);
    __syncthreads();
    store_entry<kPaged>(out_v, b, j, pooled, raw_v.dims());
    __syncthreads();
  }
  if (raw_ik.data) {
    pool_values(raw_ik, b, first, pool, a, pooled);
    __syncthreads();
    store_entry<kPaged>(out_ik, b, j, pooled, raw_ik.dims());
  }
}

// ---------------------------------------------------------------------------
// Shared-memory variant: the whole pooling window of every plane is first
// copied into shared memory with 16-byte loads issued by all threads at once,
// then the gates and pooled sums read shared memory only.

struct SlotLayout {       // bytes of one staged slot and the offsets of its parts
  int data_bytes, scale_off, rope_off, bytes;
};

__host__ __device__ inline int round16(int x) { return (x + 15) & ~15; }

__host__ __device__ inline SlotLayout slot_layout(const Cache &c) {
  SlotLayout l;
  if (c.fmt == CSKV_FMT_F32) {
    l.data_bytes = 4 * c.dims();
    l.scale_off = l.rope_off = l.bytes = round16(l.data_bytes);
    return l;
  }
  l.data_bytes = c.data_bytes();
  l.scale_off = round16(l.data_bytes);
  l.rope_off = l.scale_off + round16(c.scale_bytes());
  l.bytes = l.rope_off + round16(2 * c.d_rope);
  return l;
}

// asynchronous global -> shared copies (no register round trip), so every
// copy a thread issues is in flight at once; completed by cp.async.wait_all
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// copy n bytes (a multiple of 4) from global to shared memory, 16 bytes at a
// time when both ends allow it
__device__ inline void stage_bytes(uint8_t *dst, const uint8_t *src, int n, int t, int nt) {
  if ((((uintptr_t)src | (uintptr_t)dst) & 15) == 0 && (n & 15) == 0) {
    for (int i = t; i < (n >> 4); i += nt) cp_async16(dst + 16 * i, src + 16 * i);
  } else {
    for (int i = t; i < (n >> 2); i += nt) cp_async4(dst + 4 * i, src + 4 * i);
  }
}

// stage `pool` slots of plane set `c` for positions first .. first+pool-1;
// rows[r] is the precomputed slot row (b * cap + slot) of position first + r,
// or -1 when that position does not exist.  One warp per slot: the 16-byte
// copies of a slot are spread over its lanes.
__device__ __noinline__ void stage_window(const Cache &c, const SlotLayout &l, const long long *rows,
                             int pool, uint8_t *buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = warp; r < pool; r += nw) {
    const long long row = rows[r];
    if (row < 0) continue;
    uint8_t *dst = buf + (size_t)r * l.bytes;
    stage_bytes(dst, c.data + row * c.data_stride, l.data_bytes, lane, 32);
    if (c.fmt != CSKV_FMT_F32) {
      stage_bytes(dst + l.scale_off, c.scale + row * c.scale_stride, c.scale_bytes(), lane, 32);
      if (c.d_rope)
        stage_bytes(dst + l.rope_off, c.rope + row * c.rope_stride, 2 * c.d_rope, lane, 32);
    }
  }
}

__device__ __forceinline__ float staged_value(const Cache &c, const SlotLayout &l,
                                              const uint8_t *slot, int d) {
  if (c.fmt == CSKV_FMT_F32) return reinterpret_cast<const float *>(slot)[d];
  if (c.fmt == CSKV_FMT_MXFP4)
    return mxfp4_value(slot[d >> 1] >> ((d & 1) << 2), slot[l.scale_off + (d >> 5)]);
  if (d < c.d_nope)
    return e4m3_decode(slot[d]) *
           reinterpret_cast<const float *>(slot + l.scale_off)[c.fmt == CSKV_FMT_E4M3_VEC ? 0 : d >> 6];
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(slot + l.rope_off)[d - c.d_nope]);
}

__device__ __noinline__ void pool_staged(const Cache &c, const SlotLayout &l, const uint8_t *buf,
                            long long first, int pool, const float *a, float *pooled) {
  // the format and the slots present (positions >= 0) are fixed per entry: the
  // per-dim loops below carry no per-value branches
  const int D = c.dims(), dn = c.d_nope, bytes = l.bytes;
  const int r0 = first < 0 ? (int)-first : 0;
  if (c.fmt == CSKV_FMT_F32) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      float acc = 0.f;
      for (int r = r0; r < pool; ++r)
        acc = fmaf(a[r], reinterpret_cast<const float *>(buf + (size_t)r * bytes)[d], acc);
      pooled[d] = acc;
    }
    return;
  }
  if (c.fmt == CSKV_FMT_MXFP4) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      float acc = 0.f;
      for (int r = r0; r < pool; ++r) {
        const uint8_t *slot = buf + (size_t)r * bytes;
        acc = fmaf(a[r], mxfp4_value(slot[d >> 1] >> ((d & 1) << 2), slot[l.scale_off + (d >> 5)]),
                   acc);
      }
      pooled[d] = acc;
    }
    return;
  }
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    if (d < dn) {
      const int so = l.scale_off + (c.fmt == CSKV_FMT_E4M3_VEC ? 0 : 4 * (d >> 6));
      for (int r = r0; r < pool; ++r) {
        const uint8_t *slot = buf + (size_t)r * bytes;
        acc = fmaf(a[r] * *reinterpret_cast<const float *>(slot + so), e4m3_decode(slot[d]), acc);
      }
    } else {
      const int ro = l.rope_off + 2 * (d - dn);
      for (int r = r0; r < pool; ++r)
        acc = fmaf(a[r],
                   __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(buf + (size_t)r * bytes + ro)),
                   acc);
    }
    pooled[d] = acc;
  }
}

template <bool kPaged, bool kSmemDesc>
__global__ void __launch_bounds__(kThreads, 1)
compress_staged_kernel(const int64_t *__restrict__ t_begin, const int64_t *__restrict__ t_end,
                       Cache p_raw_k, Cache p_raw_v,
                       Cache p_raw_ik, const float *__restrict__ gate_w,
                       const float *__restrict__ gate_b, int pool, int stride,
                       Cache p_out_k, Cache p_out_v,
                       Cache p_out_ik) {
  // the cache descriptors: for a long pooling window (HCA), once in shared
  // memory, where the out-of-line helpers read them (a reference to a kernel
  // parameter makes every thread copy it to local memory, which the many
  // per-slot reads then pay for); for a short one (CSA) the per-thread copy
  // costs less than the extra barrier
  __shared__ Cache s_caches[6];
  if constexpr (kSmemDesc) {
    if (threadIdx.x == 0) {
      s_caches[0] = p_raw_k;
      s_caches[1] = p_raw_v;
      s_caches[2] = p_raw_ik;
      s_caches[3] = p_out_k;
      s_caches[4] = p_out_v;
      s_caches[5] = p_out_ik;
    }
    __syncthreads();
  }
  const Cache &raw_k = kSmemDesc ? s_caches[0] : p_raw_k;
  const Cache &raw_v = kSmemDesc ? s_caches[1] : p_raw_v;
  const Cache &raw_ik = kSmemDesc ? s_caches[2] : p_raw_ik;
  const Cache &out_k = kSmemDesc ? s_caches[3] : p_out_k;
  const Cache &out_v = kSmemDesc ? s_caches[4] : p_out_v;
  const Cache &out_ik = kSmemDesc ? s_caches[5] : p_out_ik;
  extern __shared__ __align__(16) uint8_t csm[];
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const SlotLayout lk = slot_layout(raw_k);
  const SlotLayout lv = raw_v.data ? slot_layout(raw_v) : lk;
  const SlotLayout li = raw_ik.data ? slot_layout(raw_ik) : lk;
  const int D = raw_k.dims();
  const int Dv = raw_v.data ? raw_v.dims() : 0, Di = raw_ik.data ? raw_ik.dims() : 0;
  uint8_t *bk = csm;
  uint8_t *bv = bk + (size_t)pool * lk.bytes;
  uint8_t *bi = bv + (raw_v.data ? (size_t)pool * lv.bytes : 0);
  float *gw = reinterpret_cast<float *>(bi + (raw_ik.data ? (size_t)pool * li.bytes : 0));
  float *gb = gw + round16(D);
  float *a = gb + round16(pool);
  float *pk = a + round16(pool);           // pooled key, value, indexer key
  float *pv = pk + round16(D);
  float *pi = pv + round16(Dv);
  long long *rows = reinterpret_cast<long long *>(pi + round16(Di));
  long long *rows_v = rows + pool;
  long long *rows_i = rows_v + pool;

  // the gate weights and biases travel while the token counts load
  stage_bytes(reinterpret_cast<uint8_t *>(gw), reinterpret_cast<const uint8_t *>(gate_w), 4 * D,
              tid, kThreads);
  stage_bytes(reinterpret_cast<uint8_t *>(gb), reinterpret_cast<const uint8_t *>(gate_b),
              4 * pool, tid, kThreads);
  const long long j = t_begin[b] / stride + blockIdx.x;
  check_entry(t_begin, t_end, b, j, pool, stride, raw_k, raw_v, raw_ik, out_k, out_v, out_ik);
  // never write past a cache's capacity, whatever the device-side token counts say
  if (j >= t_end[b] / stride || j < 0 || j >= out_k.cap || (raw_v.data && j >= out_v.cap) ||
      (raw_ik.data && j >= out_ik.cap) ||
      (kPaged && (!out_k.mapped(b, j) || (raw_v.data && !out_v.mapped(b, j)) ||
                  (raw_ik.data && !out_ik.mapped(b, j))))) {
    cp_async_wait_all();
    return;
  }
  const long long first = (long long)stride * (j + 1) - pool;

  // slot rows of the window's positions, one modulo per position
  for (int r = tid; r < pool; r += blockDim.x) {
    const long long p = first + r;
    rows[r] = p < 0 ? -1 : raw_k.row<kRowFlat>(b, raw_k.slot_of(p));
    if (raw_v.data) rows_v[r] = p < 0 ? -1 : raw_v.row<kRowFlat>(b, raw_v.slot_of(p));
    if (raw_ik.data) rows_i[r] = p < 0 ? -1 : raw_ik.row<kRowFlat>(b, raw_ik.slot_of(p));
  }
  __syncthreads();
  stage_window(raw_k, lk, rows, pool, bk);
  if (raw_v.data) stage_window(raw_v, lv, rows_v, pool, bv);
  if (raw_ik.data) stage_window(raw_ik, li, rows_i, pool, bi);
  cp_async_wait_all();
  __syncthreads();

  // gate logits g_r = gate_w . k_{p_r} + gate_b[r]
  for (int r = warp; r < pool; r += kWarps) {
    const long long p = first + r;
    float acc = 0.f;
    if (p >= 0) {
      const uint8_t *slot = bk + (size_t)r * lk.bytes;
      for (int d = lane; d < D; d += 32) acc = fmaf(gw[d], staged_value(raw_k, lk, slot, d), acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) a[r] = p >= 0 ? acc + gb[r] : -CUDART_INF_F;
  }
  __syncthreads();
  if (warp == 0) {
    float m = -CUDART_INF_F;
    for (int r = lane; r < pool; r += 32) m = fmaxf(m, a[r]);
    m = warp_max(m);
    float s = 0.f;
    for (int r = lane; r < pool; r += 32) s += (a[r] == -CUDART_INF_F) ? 0.f : expf(a[r] - m);
    s = warp_sum(s);
    __syncwarp();
    for (int r = lane; r < pool; r += 32)
      a[r] = (a[r] == -CUDART_INF_F) ? 0.f : expf(a[r] - m) / s;
  }
  __syncthreads();

  // pooled sums of every plane (no barrier between the planes)
  pool_staged(raw_k, lk, bk, first, pool, a, pk);
  if (raw_v.data) pool_staged(raw_v, lv, bv, first, pool, a, pv);
  if (raw_ik.data) pool_staged(raw_ik, li, bi, first, pool, a, pi);
  __syncthreads();
  // re-quantisation and stores (no shared memory is written from here on)
  store_entry<kPaged>(out_k, b, j, pk, D);
  if (raw_v.data) store_entry<kPaged>(out_v, b, j, pv, Dv);
  if (raw_ik.data) store_entry<kPaged>(out_ik, b, j, pi, Di);
}


// ---------------------------------------------------------------------------
// Per-channel gate variant: one softmax over the window's slots for every
// channel c, with logits g_{r,c} = gate_w[c] * k_{p_r}[c] + gate_b[r][c] read
// from that channel of the key alone; the value (separate-V layout) is pooled
// with the key's weights, the indexer keys with gates of their own.  The
// window is staged in shared memory as above; each thread then runs an online
// softmax over the slots for its channels (the bias rows come from L2).
__device__ __noinline__ void pool_channels(const Cache &c, const SlotLayout &l, const uint8_t *buf,
                                           const Cache *cv, const SlotLayout &lv,
                                           const uint8_t *bufv, int r0, int pool,
                                           const float *__restrict__ gw,
                                           const float *__restrict__ gb, float *pooled,
                                           float *pooled_v) {
  const int D = c.dims();
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const float w = gw[d];
    float m = -CUDART_INF_F, s = 0.f, acc = 0.f, accv = 0.f;
    for (int r = r0; r < pool; ++r) {
      const float x = staged_value(c, l, buf + (size_t)r * l.bytes, d);
      const float g = fmaf(w, x, gb[(size_t)r * D + d]);
      if (g > m) {
        const float f = expf(m - g);       // (m = -inf: f = 0, the sums are 0)
        s *= f;
        acc *= f;
        accv *= f;
        m = g;
      }
      const float e = expf(g - m);
      s += e;
      acc = fmaf(e, x, acc);
      if (cv) accv = fmaf(e, staged_value(*cv, lv, bufv + (size_t)r * lv.bytes, d), accv);
    }
    pooled[d] = acc / s;
    if (cv) pooled_v[d] = accv / s;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
compress_channel_kernel(const int64_t *__restrict__ t_begin, const int64_t *__restrict__ t_end,
                        Cache raw_k, Cache raw_v,
                        Cache raw_ik, const float *__restrict__ gate_w,
                        const float *__restrict__ gate_b, const float *__restrict__ gate_w_ik,
                        const float *__restrict__ gate_b_ik, int pool, int stride,
                        Cache out_k, Cache out_v,
                        Cache out_ik) {
  extern __shared__ __align__(16) uint8_t csm[];
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int tid = threadIdx.x;
  const SlotLayout lk = slot_layout(raw_k);
  const SlotLayout lv = raw_v.data ? slot_layout(raw_v) : lk;
  const SlotLayout li = raw_ik.data ? slot_layout(raw_ik) : lk;
  const int D = raw_k.dims();
  const int Dv = raw_v.data ? raw_v.dims() : 0, Di = raw_ik.data ? raw_ik.dims() : 0;
  uint8_t *bk = csm;
  uint8_t *bv = bk + (size_t)pool * lk.bytes;
  uint8_t *bi = bv + (raw_v.data ? (size_t)pool * lv.bytes : 0);
  float *pk = reinterpret_cast<float *>(bi + (raw_ik.data ? (size_t)pool * li.bytes : 0));
  float *pv = pk + round16(D);
  float *pi = pv + round16(Dv);
  long long *rows = reinterpret_cast<long long *>(pi + round16(Di));
  long long *rows_v = rows + pool;
  long long *rows_i = rows_v + pool;

  const long long j = t_begin[b] / stride + blockIdx.x;
  check_entry(t_begin, t_end, b, j, pool, stride, raw_k, raw_v, raw_ik, out_k, out_v, out_ik);
  // never write past a cache's capacity, whatever the device-side token counts say
  if (j >= t_end[b] / stride || j < 0 || j >= out_k.cap || (raw_v.data && j >= out_v.cap) ||
      (raw_ik.data && j >= out_ik.cap) || !out_k.mapped(b, j) ||
      (raw_v.data && !out_v.mapped(b, j)) || (raw_ik.data && !out_ik.mapped(b, j)))
    return;
  const long long first = (long long)stride * (j + 1) - pool;
  for (int r = tid; r < pool; r += blockDim.x) {
    const long long p = first + r;
    rows[r] = p < 0 ? -1 : raw_k.row<kRowFlat>(b, raw_k.slot_of(p));
    if (raw_v.data) rows_v[r] = p < 0 ? -1 : raw_v.row<kRowFlat>(b, raw_v.slot_of(p));
    if (raw_ik.data) rows_i[r] = p < 0 ? -1 : raw_ik.row<kRowFlat>(b, raw_ik.slot_of(p));
  }
  __syncthreads();
  stage_window(raw_k, lk, rows, pool, bk);
  if (raw_v.data) stage_window(raw_v, lv, rows_v, pool, bv);
  if (raw_ik.data) stage_window(raw_ik, li, rows_i, pool, bi);
  cp_async_wait_all();
  __syncthreads();

  const int r0 = first < 0 ? (int)-first : 0;
  pool_channels(raw_k, lk, bk, raw_v.data ? &raw_v : nullptr, lv, bv, r0, pool, gate_w, gate_b,
                pk, pv);
  if (raw_ik.data)
    pool_channels(raw_ik, li, bi, nullptr, li, bi, r0, pool, gate_w_ik, gate_b_ik, pi, nullptr);
  __syncthreads();
  store_entry<true>(out_k, b, j, pk, D);
  if (raw_v.data) store_entry<true>(out_v, b, j, pv, Dv);
  if (raw_ik.data) store_entry<true>(out_ik, b, j, pi, Di);
}

}  // namespace

int launch_compress(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                    const Cache &raw_k, const Cache &raw_v, const Cache &raw_ik,
                    const float *gate_w, const float *gate_b, int pool, int stride,
                    const Cache &out_k, const Cache &out_v, const Cache &out_ik,
                    cudaStream_t st) {
  if (max_new == 0 || B == 0) return CSKV_OK;
  int dmax = raw_k.dims();
  if (raw_v.data && raw_v.dims() > dmax) dmax = raw_v.dims();
  if (raw_ik.data && raw_ik.dims() > dmax) dmax = raw_ik.dims();
  dim3 grid((unsigned)max_new, (unsigned)B);
  size_t staged = (size_t)pool * slot_layout(raw_k).bytes;
  if (raw_v.data) staged += (size_t)pool * slot_layout(raw_v).bytes;
  if (raw_ik.data) staged += (size_t)pool * slot_layout(raw_ik).bytes;
  const int Dk = raw_k.dims(), Dv = raw_v.data ? raw_v.dims() : 0;
  const int Di = raw_ik.data ? raw_ik.dims() : 0;
  const size_t smem_staged =
      staged +
      sizeof(float) * (size_t)(2 * round16(Dk) + 2 * round16(pool) + round16(Dv) + round16(Di)) +
      3 * sizeof(long long) * (size_t)pool + 16;
  const bool paged = out_k.bt || (raw_v.data && out_v.bt) || (raw_ik.data && out_ik.bt);
  const bool smem_desc = pool >= 32;
  auto staged_kernel = paged ? (smem_desc ? compress_staged_kernel<true, true>
                                          : compress_staged_kernel<true, false>)
                             : (smem_desc ? compress_staged_kernel<false, true>
                                          : compress_staged_kernel<false, false>);
  if (smem_staged <= 200 * 1024 && ensure_dynamic_smem(staged_kernel, smem_staged)) {
    if (launch_pdl(staged_kernel, grid, dim3(kThreads), smem_staged, st, t_begin, t_end, raw_k,
                   raw_v, raw_ik, gate_w, gate_b, pool, stride, out_k, out_v,
                   out_ik) != cudaSuccess)
      return CSKV_ERR_CUDA;
  } else {
    const size_t smem = sizeof(float) * (size_t)(pool + dmax);
    if (launch_pdl(paged ? compress_kernel<true> : compress_kernel<false>, grid, dim3(kThreads),
                   smem, st, t_begin, t_end, raw_k, raw_v, raw_ik, gate_w, gate_b, pool, stride,
                   out_k, out_v, out_ik) != cudaSuccess)
      return CSKV_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? CSKV_OK : CSKV_ERR_CUDA;
}

int launch_compress_channel(int B, const int64_t *t_begin, const int64_t *t_end, int64_t max_new,
                            const Cache &raw_k, const Cache &raw_v, const Cache &raw_ik,
                            const float *gate_w, const float *gate_b, const float *gate_w_ik,
                            const float *gate_b_ik, int pool, int stride, const Cache &out_k,
                            const Cache &out_v, const Cache &out_ik, cudaStream_t st) {
  if (max_new == 0 || B == 0) return CSKV_OK;
  size_t staged = (size_t)pool * slot_layout(raw_k).bytes;
  if (raw_v.data) staged += (size_t)pool * slot_layout(raw_v).bytes;
  if (raw_ik.data) staged += (size_t)pool * slot_layout(raw_ik).bytes;
  const int Dk = raw_k.dims(), Dv = raw_v.data ? raw_v.dims() : 0;
  const int Di = raw_ik.data ? raw_ik.dims() : 0;
  const size_t smem = staged + sizeof(float) * (size_t)(round16(Dk) + round16(Dv) + round16(Di)) +
                      3 * sizeof(long long) * (size_t)pool + 16;
  // the staged window must fit in shared memory (HCA's 128 FP8 slots: 78 KB)
  if (smem > 200 * 1024 || !ensure_dynamic_smem(compress_channel_kernel, smem))
    return CSKV_ERR_UNSUPPORTED;
  if (launch_pdl(compress_channel_kernel, dim3((unsigned)max_new, (unsigned)B), dim3(kThreads),
                 smem, st, t_begin, t_end, raw_k, raw_v, raw_ik, gate_w, gate_b, gate_w_ik,
                 gate_b_ik, pool, stride, out_k, out_v, out_ik) != cudaSuccess)
    return CSKV_ERR_CUDA;
  return CSKV_OK;
}

}  // namespace cskv
