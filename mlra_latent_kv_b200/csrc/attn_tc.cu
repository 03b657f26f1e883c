// tcgen05 split-KV latent attention (sm_100a).
#include "attn_tc.h"

namespace mlra {

bool tc_supported(int, int, int, int, int, int, int) { return false; }

cudaError_t launch_attend_tc(const void*, const void*, const void*, const int*, const int*, float*, float*, int*,
                             const AttnArgs&, cudaStream_t) {
  return cudaErrorNotSupported;
}

void tc_shutdown() {}

}  // namespace mlra
