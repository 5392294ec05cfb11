// Tensor-core (tcgen05) hybrid attention for the 64-head x 512-dim FP8+BF16 layout.
#include "cskv_internal.cuh"

namespace cskv {

bool attn_tc_supported(const AttnArgs &a) { (void)a; return false; }
int attn_tc_chunk_keys() { return 128; }

int launch_attn_tc(const AttnArgs &a, float *part_o, float *part_lse, int n_chunks,
                   cudaStream_t st) {
  (void)a; (void)part_o; (void)part_lse; (void)n_chunks; (void)st;
  return CSKV_ERR_UNSUPPORTED;
}

}  // namespace cskv
