// Decode-batch kernel instance: batch class 8 (up to 8 activation row(s)).
#include "decode_kernel.cuh"

namespace biloco {
template cudaError_t launch_decode<8>(const CUtensorMap&, const DecodeParams&, cudaStream_t, const LaunchOpts&);
}  // namespace biloco
