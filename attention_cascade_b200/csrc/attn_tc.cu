// attn_tc.cu — tcgen05 / TMEM / TMA attention kernel (sm_100a).  Not built yet:
// attn_tc_supported() reports false so the CUDA-core kernel serves every case.
#include "kernels.h"

namespace jev {
bool attn_tc_supported(int) { return false; }
cudaError_t launch_attn_tc(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace jev
