// Sticky per-device status word and the test hooks of the failure paths (the
// selection's meeting-point poll limit, a stalled scoring CTA).
//
// Every wait inside a kernel of the library is bounded.  When one runs out,
// the kernel ORs a CSKV_DEV_* bit into this word, marks its results invalid
// (NaN scores or lse, failed selection rows) and returns; the host reads the
// word with cskv_check_device_errors.  The word is a file-scope __device__
// variable, so every kernel is handed its device address (looked up once per
// device with that device current) as an argument.
#include <atomic>
#include <mutex>

#include "cskv_internal.cuh"

namespace cskv {

namespace {

static __device__ __align__(16) unsigned int g_status;
static __device__ unsigned int g_status_taken;

__global__ void status_take_kernel() { g_status_taken = atomicExch(&g_status, 0u); }

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int *g_status_ptr[kMaxDevices] = {};
std::atomic<uint32_t> g_indexer_stall{0};
std::atomic<uint32_t> g_barrier_spins{kDefaultBarrierSpins};

}  // namespace

unsigned int *device_status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess || !p) {
      cudaGetLastError();
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<unsigned int *>(p);
  }
  return g_status_ptr[dev];
}

uint32_t indexer_stall_polls() { return g_indexer_stall.load(std::memory_order_relaxed); }
uint32_t topk_barrier_spins() { return g_barrier_spins.load(std::memory_order_relaxed); }

}  // namespace cskv

extern "C" {

int cskv_check_device_errors(cskv_stream_t stream, uint32_t *events) {
  using namespace cskv;
  if (events) *events = 0;
  if (!device_status_word()) return CSKV_ERR_CUDA;
  // after the stream's work, one thread swaps the word for zero (events that
  // other streams' kernels record meanwhile keep their bits for the next
  // read); the old value comes back through a second device word
  const cudaStream_t st = (cudaStream_t)stream;
  status_take_kernel<<<1, 1, 0, st>>>();
  if (cudaGetLastError() != cudaSuccess) return CSKV_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status_taken, sizeof(v), 0, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return CSKV_ERR_CUDA;
  if (events) *events = v;
  return v ? CSKV_ERR_DEVICE : CSKV_OK;
}

uint32_t cskv_debug_topk_barrier_spins(uint32_t spins) {
  return cskv::g_barrier_spins.exchange(spins);
}

uint32_t cskv_debug_indexer_stall(uint32_t polls) {
  return cskv::g_indexer_stall.exchange(polls);
}

}  // extern "C"
