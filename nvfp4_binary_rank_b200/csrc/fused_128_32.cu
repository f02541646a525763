// Fused kernel instance: 128-column MMA tile, 3 stages, batch class 32.
#include <mutex>

#include "fused_kernel.cuh"
#include "fused_launch.h"

namespace biloco {

cudaError_t launch_fused_128_32(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl) {
  using L = Layout<128, 3>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(fused_kernel<128, 3, 32>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(fp.G));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fused_kernel<128, 3, 32>, tw, tx, txs, tv, fp);
}

}  // namespace biloco
