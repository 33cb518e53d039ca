// Replay-read kernel instantiations for dstate = 32.
#include "rssm_read.cuh"

namespace rssm {
template cudaError_t read_dispatch_n<32>(int, int, const ReadArgs &, size_t, cudaStream_t);
}  // namespace rssm
