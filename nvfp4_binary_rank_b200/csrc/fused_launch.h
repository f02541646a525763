// Launcher of the general fused kernel.  One template, instantiated once per
// (MMA tile width BN, stages ST, batch class MC) in its own translation unit
// (fused_<BN>_<MC>.cu) so that the instances compile in parallel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fused_params.h"
#include "launch_common.h"

namespace biloco {

// Launches fused_kernel<BN, ST, MC> on fp.G CTAs (all resident together).
template <int BN, int ST, int MC>
cudaError_t launch_fused(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                         const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, const LaunchOpts& o);

#define BILOCO_FUSED_EXTERN(BN, ST, MC)                                                                    \
  extern template cudaError_t launch_fused<BN, ST, MC>(const CUtensorMap&, const CUtensorMap&,            \
                                                       const CUtensorMap&, const CUtensorMap&,            \
                                                       const FusedParams&, cudaStream_t, const LaunchOpts&);
BILOCO_FUSED_EXTERN(16, 5, 1)
BILOCO_FUSED_EXTERN(16, 5, 2)
BILOCO_FUSED_EXTERN(16, 5, 4)
BILOCO_FUSED_EXTERN(16, 5, 8)
BILOCO_FUSED_EXTERN(16, 5, 16)
BILOCO_FUSED_EXTERN(32, 3, 32)
BILOCO_FUSED_EXTERN(64, 4, 32)
BILOCO_FUSED_EXTERN(128, 3, 32)
#undef BILOCO_FUSED_EXTERN

}  // namespace biloco
