// Decode-batch kernel instance: batch class 4 (up to 4 activation row(s)).
#include "decode_kernel.cuh"

namespace biloco {
template cudaError_t launch_decode<4>(const CUtensorMap&, const DecodeParams&, cudaStream_t, const LaunchOpts&);
}  // namespace biloco
