// indexer_topk_noalloc: the lightning-indexer top-k without a caller workspace.
//
// Some callers cannot hand the library a workspace: code that runs where
// cudaMalloc is not allowed or not safe (a host framework that owns all device
// memory through its own pool and exposes no scratch to plug-ins, a real-time
// loop that forbids allocation after start-up, a custom-op interface with no
// workspace argument).  For them this entry point keeps its scratch in a
// fixed-size array in the library's own device memory instead.
//
// The scratch array below lives in every GPU that loads the library for as
// long as the process runs.  Its address is looked up once per device
// (cudaGetSymbolAddress, with that device current) on the first call made on
// that device; make that first call before any stream capture.  All calls
// share the one array, so calls that overlap on the GPU (different streams,
// or different host threads, on the same device) race on it and must be
// serialised by the caller.  Nothing in it has to start at zero: each call's
// scoring writes every score slot its selection reads (a scoring CTA whose
// wait ran out writes NaN there, and the selection then reports the row as
// failed), and the score histogram and counters kept between calls only
// guide the selection - a stale histogram from a call of another shape costs
// time, not correctness.
#include <mutex>

#include "cskv_internal.cuh"

namespace {

// 8 MiB.  A request fits when cskv_indexer_workspace_size(B, Tq, max_entries,
// k) <= 8 MiB: one query row at a 1,048,576-token context (262,144 CSA
// entries, k = 1,024) needs 1,131,776 bytes, so up to 7 such rows fit; a row
// at 65,536 tokens (16,384 entries, k = 512) needs 148,512 bytes, up to 56
// rows.
constexpr size_t kScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_indexer_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on error).
void *scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_indexer_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

size_t cskv_noalloc_scratch_bytes(void) { return kScratchBytes; }

int indexer_topk_noalloc(int B, int Tq, const int64_t *q_pos, const void *q_ik,
                         const float *q_ik_scale, const float *head_w, int H_I, int d_I,
                         const cskv_cache *ik, int stride, int k, int64_t max_entries,
                         int32_t *out_idx, float *out_score, cskv_stream_t stream) {
  if (B > 0 && Tq > 0 && max_entries >= 0 &&
      cskv_indexer_workspace_size(B, Tq, max_entries, k) > kScratchBytes)
    return CSKV_ERR_SCRATCH_LIMIT;
  void *ws = nullptr;
  if (B > 0 && Tq > 0) {
    ws = scratch_on_current_device();
    if (!ws) return CSKV_ERR_CUDA;
  }
  return indexer_topk(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I, ik, stride, k,
                      max_entries, out_idx, out_score, ws, kScratchBytes, stream);
}

}  // extern "C"
