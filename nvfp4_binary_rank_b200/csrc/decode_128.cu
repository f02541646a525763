// Decode-batch kernel instance: batch class 128 (65 to 128 activation rows).
#include "decode_kernel.cuh"

namespace biloco {
template cudaError_t launch_decode<128>(const CUtensorMap&, const DecodeParams&, cudaStream_t, const LaunchOpts&);
}  // namespace biloco
