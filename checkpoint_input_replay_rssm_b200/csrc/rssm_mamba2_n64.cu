// Kernel instantiations for dstate = 64.
#include "rssm_mamba2.cuh"

namespace rssm {
template cudaError_t m2_dispatch_n<64>(int, int, int, const M2Args &, const M2FoldLay &, size_t, int, cudaStream_t);
}  // namespace rssm
