// Launch of the library's grid-synchronising GEMM kernels.
//
// Both GEMM kernels exchange data between CTAs behind grid-wide arrival
// counters (the activation image, z, the split-K tickets' partners), so every
// CTA of a grid must be resident at the same time.  The host guarantees the part
// it can: one CTA per SM fits (occupancy query, done once per kernel) and the
// grid is no larger than the SM count.  Two launch forms:
//   * programmatic dependent launch (the default): the grid may start while the
//     kernel before it on the stream finishes, so its weight stream overlaps that
//     kernel's tail.  Co-residency then also needs the GPU not to be shared with
//     long-running kernels on other streams; if CTAs cannot all start, the
//     waiting ones give up after their bounded wait and report
//     BILOCO_ERR_TIMEOUT.
//   * cooperative launch (opt-in): the driver starts the grid only when all of
//     its CTAs can be resident together, whatever else runs on the GPU.  Where
//     the driver accepts both attributes together the grid keeps programmatic
//     overlap as well; otherwise it is launched cooperative only.
#pragma once

#include <atomic>
#include <mutex>

#include <cuda_runtime.h>

namespace biloco {

struct LaunchOpts {
  bool pdl = true;           // programmatic stream serialisation
  bool cooperative = false;  // cudaLaunchAttributeCooperative
};

// Per kernel: the shared-memory opt-in and the residency check, done once.
struct KernelSetup {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  int blocks_per_sm = 0;
  int num_sms = 0;
  std::atomic<int> coop_with_pdl{-1};    // -1 untried, 0 rejected, 1 accepted
};

template <typename Kernel>
cudaError_t prepare_kernel(KernelSetup& ks, Kernel kernel, int threads, int smem) {
  std::call_once(ks.once, [&] {
    ks.err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (ks.err != cudaSuccess) return;
    ks.err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ks.blocks_per_sm, kernel, threads, smem);
    if (ks.err != cudaSuccess) return;
    int dev = 0;
    ks.err = cudaGetDevice(&dev);
    if (ks.err != cudaSuccess) return;
    ks.err = cudaDeviceGetAttribute(&ks.num_sms, cudaDevAttrMultiProcessorCount, dev);
  });
  return ks.err;
}

// Launches `kernel` on `grid` CTAs that must all be resident together.
// Returns cudaErrorCooperativeLaunchTooLarge when they cannot be, on any GPU state.
template <typename Kernel, typename... Args>
cudaError_t launch_resident(KernelSetup& ks, Kernel kernel, int grid, int threads, int smem,
                            cudaStream_t s, const LaunchOpts& o, Args&&... args) {
  cudaError_t e = prepare_kernel(ks, kernel, threads, smem);
  if (e != cudaSuccess) return e;
  if (ks.blocks_per_sm < 1 || grid > ks.blocks_per_sm * ks.num_sms)
    return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  const bool coop = o.cooperative;
  const bool pdl = o.pdl && (!coop || ks.coop_with_pdl.load() != 0);
  if (coop) {
    attr[n].id = cudaLaunchAttributeCooperative;
    attr[n].val.cooperative = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (coop && pdl) {
    if (e == cudaSuccess) {
      ks.coop_with_pdl.store(1);
    } else if (e != cudaErrorCooperativeLaunchTooLarge) {
      // the driver rejects the pair: launch cooperative only, now and later
      cudaGetLastError();
      ks.coop_with_pdl.store(0);
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    }
  }
  return e;
}

}  // namespace biloco
