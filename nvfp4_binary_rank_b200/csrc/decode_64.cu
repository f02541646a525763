// Decode-batch kernel instance: batch class 64 (33 to 64 activation rows).
#include "decode_kernel.cuh"

namespace biloco {
template cudaError_t launch_decode<64>(const CUtensorMap&, const DecodeParams&, cudaStream_t, const LaunchOpts&);
}  // namespace biloco
