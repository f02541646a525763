// General fused kernel instance: MMA tile width 16, 5 stages, batch class 1.
#include "fused_kernel.cuh"

namespace biloco {
template cudaError_t launch_fused<16, 5, 1>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                             const CUtensorMap&, const FusedParams&, cudaStream_t,
                                             const LaunchOpts&);
}  // namespace biloco
