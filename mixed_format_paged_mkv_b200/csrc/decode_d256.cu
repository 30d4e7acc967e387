// Partial-attention kernels for head dimension 256 (templates in decode_partial.cuh).
#include "decode_partial.cuh"

namespace mkv {

cudaError_t launch_partial_d256(int K, const DecodeParams& p, int c0, int c1, bool dependent,
                               cudaStream_t s) {
  return launch_partial_kind<256>(K, p, c0, c1, dependent, s);
}

int partial_ctas_per_sm_d256(int K, int NC) { return partial_ctas_per_sm_kind<256>(K, NC); }

}  // namespace mkv
