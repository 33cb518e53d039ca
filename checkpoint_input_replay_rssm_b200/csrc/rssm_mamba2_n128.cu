// Kernel instantiations for dstate = 128.
#include "rssm_mamba2.cuh"

namespace rssm {
template cudaError_t m2_dispatch_n<128>(bool, int, int, const M2Args &, size_t, cudaStream_t);
}  // namespace rssm
