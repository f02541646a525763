// Decode-batch kernel instance: batch class 16 (up to 16 activation row(s)).
#include "decode_kernel.cuh"

namespace biloco {
template cudaError_t launch_decode<16>(const CUtensorMap&, const DecodeParams&, cudaStream_t, const LaunchOpts&);
}  // namespace biloco
