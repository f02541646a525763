// Decode-batch kernel instance: batch class 32 (17 to 32 activation rows).
#include "decode_kernel.cuh"

namespace biloco {
template cudaError_t launch_decode<32>(const CUtensorMap&, const DecodeParams&, cudaStream_t, const LaunchOpts&);
}  // namespace biloco
