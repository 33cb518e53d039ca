// Kernel instantiations for dstate = 16.
#include "rssm_gdn.cuh"

namespace rssm {
template cudaError_t g_dispatch_n<16>(bool, int, int, const GArgs &, size_t, cudaStream_t);
template cudaError_t g_prep_dispatch_n<16>(int, const GArgs &, cudaStream_t);
}  // namespace rssm
