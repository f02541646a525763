// General fused kernel instance: MMA tile width 128, 3 stages, batch class 32.
#include "fused_kernel.cuh"

namespace biloco {
template cudaError_t launch_fused<128, 3, 32>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                             const CUtensorMap&, const FusedParams&, cudaStream_t,
                                             const LaunchOpts&);
}  // namespace biloco
