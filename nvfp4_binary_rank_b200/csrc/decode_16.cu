// Decode-batch kernel instance: up to 16 activation row(s).
#include <mutex>

#include "decode_kernel.cuh"
#include "decode_launch.h"

namespace biloco {

static_assert(decode::kMaxUnits == kDecodeMaxUnits && decode::kRowsMax == kDecodeMaxRows,
              "host and kernel limits agree");

cudaError_t launch_decode_16(const CUtensorMap& tw, const DecodeParams& dp, cudaStream_t s) {
  using L = decode::Layout<16>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(decode::decode_kernel<16>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(dp.G));
  cfg.blockDim = dim3(decode::kThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode::decode_kernel<16>, tw, dp);
}

}  // namespace biloco
