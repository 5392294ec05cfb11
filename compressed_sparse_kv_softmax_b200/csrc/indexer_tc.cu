// Tensor-core (tcgen05) lightning-indexer scoring for the FP8 64-head x 128-dim layout.
#include "cskv_internal.cuh"

namespace cskv {

bool indexer_tc_supported(const IndexerArgs &a) { (void)a; return false; }

int launch_indexer_tc(const IndexerArgs &a, float *scores, long long ld, cudaStream_t st) {
  (void)a; (void)scores; (void)ld; (void)st;
  return CSKV_ERR_UNSUPPORTED;
}

}  // namespace cskv
