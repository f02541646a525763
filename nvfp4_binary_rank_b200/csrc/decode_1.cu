// Decode-batch kernel instance: batch class 1 (up to 1 activation row(s)).
#include "decode_kernel.cuh"

namespace biloco {
template cudaError_t launch_decode<1>(const CUtensorMap&, const DecodeParams&, cudaStream_t, const LaunchOpts&);
}  // namespace biloco
