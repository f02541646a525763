// General fused kernel instance: MMA tile width 64, 4 stages, batch class 32.
#include "fused_kernel.cuh"

namespace biloco {
template cudaError_t launch_fused<64, 4, 32>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                             const CUtensorMap&, const FusedParams&, cudaStream_t,
                                             const LaunchOpts&);
}  // namespace biloco
