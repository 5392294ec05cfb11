// cskv_ring_store: one new raw token per sequence into raw-token rings.
//
// The sliding window attends the last 128 raw tokens, and the compressors
// pool raw tokens, so each decode step first appends its token to the rings
// («Chinas KI-Unabhaengigkeit?: Bei Deepseek V4 haben kleine Aenderungen
// grosse Wirkung», "Komprimierte Erinnerung fuer laengere Kontexte").  One
// launch covers every (source, ring) pair: CTA (b, i) copies sequence b's
// token of pair i, plane by plane, in 16-byte units where the plane's bytes
// and addresses allow (4-byte units otherwise).
#include "cskv_internal.cuh"

namespace cskv {

namespace {

constexpr int kMaxPairs = 8;
constexpr int kThreads = 128;

struct RingPairs {
  Cache src[kMaxPairs], ring[kMaxPairs];
};

__device__ __forceinline__ void copy_bytes(uint8_t *__restrict__ dst, const uint8_t *__restrict__ src,
                                           int bytes) {
  if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | bytes) & 15) == 0) {
    for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x)
      reinterpret_cast<uint4 *>(dst)[i] = __ldg(reinterpret_cast<const uint4 *>(src) + i);
  } else {
    for (int i = threadIdx.x; i < bytes / 4; i += blockDim.x)
      reinterpret_cast<uint32_t *>(dst)[i] = __ldg(reinterpret_cast<const uint32_t *>(src) + i);
  }
}

__global__ void __launch_bounds__(kThreads)
ring_store_kernel(const RingPairs p, const int64_t *__restrict__ pos) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x, i = blockIdx.y;
  const Cache &s = p.src[i], &r = p.ring[i];
  const long long q = pos[b];
  if (!r.check(q >= 0)) return;     // (a negative position names no slot)
  const long long slot = r.slot_of(q);
  const long long rs = r.row(b, slot), ss = s.row(b, 0);
  if (s.fmt == CSKV_FMT_F32) {
    copy_bytes(r.data + rs * r.data_stride, s.data + ss * s.data_stride, 4 * s.dims());
    return;
  }
  copy_bytes(r.data + rs * r.data_stride, s.data + ss * s.data_stride, s.d_nope);
  copy_bytes(r.scale + rs * r.scale_stride, s.scale + ss * s.scale_stride, 4 * s.n_scales());
  if (s.d_rope) copy_bytes(r.rope + rs * r.rope_stride, s.rope + ss * s.rope_stride, 2 * s.d_rope);
}

}  // namespace

int launch_ring_store(int B, const int64_t *pos, int n, const Cache *src, const Cache *ring,
                      cudaStream_t st) {
  if (n > kMaxPairs) return CSKV_ERR_ARG;
  RingPairs p{};
  for (int i = 0; i < n; ++i) {
    p.src[i] = src[i];
    p.ring[i] = ring[i];
  }
  return launch_pdl(ring_store_kernel, dim3((unsigned)B, (unsigned)n), dim3(kThreads), 0, st, p,
                    pos) == cudaSuccess
             ? CSKV_OK
             : CSKV_ERR_CUDA;
}

}  // namespace cskv
