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
// One CTA per (new entry, sequence).  The work is a few KB per entry and runs
// once per 4 (CSA) or 128 (HCA) tokens, so the kernel is written for clarity:
// one warp per slot for the gate dot products, one thread per dim for the
// pooled sums, one warp per 64-element block for the re-quantisation.
#include <math_constants.h>

#include "cskv_internal.cuh"

namespace cskv {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ void store_entry(const Cache &out, int b, long long j, const float *pooled, int D) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (out.fmt == CSKV_FMT_F32) {
    float *dst = reinterpret_cast<float *>(out.data + out.row(b, j) * out.data_stride);
    for (int d = tid; d < D; d += kThreads) dst[d] = pooled[d];
    return;
  }
  uint8_t *codes = out.data + out.row(b, j) * out.data_stride;
  float *scales = reinterpret_cast<float *>(out.scale + out.row(b, j) * out.scale_stride);
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
        reinterpret_cast<__nv_bfloat16 *>(out.rope + out.row(b, j) * out.rope_stride);
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
      acc = fmaf(a[r], raw.value(b, raw.slot_of(p), d), acc);
    }
    pooled[d] = acc;
  }
}

__global__ void __launch_bounds__(kThreads)
compress_kernel(const int64_t *__restrict__ t_begin, const int64_t *__restrict__ t_end,
                Cache raw_k, Cache raw_v, Cache raw_ik, const float *__restrict__ gate_w,
                const float *__restrict__ gate_b, int pool, int stride, Cache out_k,
                Cache out_v, Cache out_ik) {
  extern __shared__ float smem[];
  float *a = smem;                 // [pool] gate logits, then weights
  float *pooled = smem + pool;     // [max dims]
  const int b = blockIdx.y;
  const long long j = t_begin[b] / stride + blockIdx.x;
  if (j >= t_end[b] / stride || j < 0) return;
  // never write past a cache's capacity, whatever the device-side token counts say
  if (j >= out_k.cap || (raw_v.data && j >= out_v.cap) || (raw_ik.data && j >= out_ik.cap))
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
      for (int d = lane; d < D; d += 32) acc = fmaf(gate_w[d], raw_k.value(b, slot, d), acc);
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
  store_entry(out_k, b, j, pooled, D);
  __syncthreads();
  if (raw_v.data) {
    pool_values(raw_v, b, first, pool, a, pooled);
    __syncthreads();
    store_entry(out_v, b, j, pooled, raw_v.dims());
    __syncthreads();
  }
  if (raw_ik.data) {
    pool_values(raw_ik, b, first, pool, a, pooled);
    __syncthreads();
    store_entry(out_ik, b, j, pooled, raw_ik.dims());
  }
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
  const size_t smem = sizeof(float) * (size_t)(pool + dmax);
  dim3 grid((unsigned)max_new, (unsigned)B);
  compress_kernel<<<grid, kThreads, smem, st>>>(t_begin, t_end, raw_k, raw_v, raw_ik, gate_w,
                                                gate_b, pool, stride, out_k, out_v, out_ik);
  return cudaGetLastError() == cudaSuccess ? CSKV_OK : CSKV_ERR_CUDA;
}

}  // namespace cskv
