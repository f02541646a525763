// Decode-batch kernel instance: batch class 2 (up to 2 activation row(s)).
#include "decode_kernel.cuh"

namespace biloco {
template cudaError_t launch_decode<2>(const CUtensorMap&, const DecodeParams&, cudaStream_t, const LaunchOpts&);
}  // namespace biloco
