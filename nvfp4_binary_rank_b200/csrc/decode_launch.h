// Launcher of the decode-batch kernel.  One template, instantiated once per
// batch class (1, 2, 4, 8, 16, 32, 64 and 128 activation rows) in its own
// translation unit (decode_<class>.cu) so that the classes compile in parallel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "decode_params.h"
#include "launch_common.h"

namespace biloco {

// The host's view of the batch classes; the kernel checks each against its own
// constants where it is compiled.
constexpr int kDecodeMaxRows = 128;
constexpr int decode_class(int M) {
  return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
}
// MMA N of the FP4 product (activation rows, padded), and rows of a split-K slot.
constexpr int decode_bn(int M) { return M <= 16 ? 16 : decode_class(M); }
// Units of 128 weight rows x 256 K elements one CTA can hold (the operand cache of
// the classes up to 16 rows; the classes from 32 rows stream their activation
// chunks).
constexpr int decode_max_units(int M) { return M <= 16 ? 16 : 64; }
// Bytes per 256-element K chunk of the quantised activation image: 16 rows of
// codes and 256 B of scales, or (32+ rows) one code row per activation row of
// the class and four 512-byte scale atoms.
constexpr int decode_img_bytes(int M) { return M <= 16 ? 16 * 128 + 256 : decode_bn(M) * 128 + 4 * 512; }
// Bytes of the z tiles of the tensor-core U side: 16 chunks of 64 ranks x
// max(16, 2 class) rows x 128 B (the classes below 16 rows use the 16-row size).
constexpr int decode_ztile_bytes(int M) { return 16 * (M <= 16 ? 32 : 2 * decode_class(M)) * 128; }

// Launches decode_kernel<MC> on dp.G CTAs (all resident together).
template <int MC>
cudaError_t launch_decode(const CUtensorMap& tw, const DecodeParams& dp, cudaStream_t s,
                          const LaunchOpts& o);

extern template cudaError_t launch_decode<1>(const CUtensorMap&, const DecodeParams&, cudaStream_t,
                                             const LaunchOpts&);
extern template cudaError_t launch_decode<2>(const CUtensorMap&, const DecodeParams&, cudaStream_t,
                                             const LaunchOpts&);
extern template cudaError_t launch_decode<4>(const CUtensorMap&, const DecodeParams&, cudaStream_t,
                                             const LaunchOpts&);
extern template cudaError_t launch_decode<8>(const CUtensorMap&, const DecodeParams&, cudaStream_t,
                                             const LaunchOpts&);
extern template cudaError_t launch_decode<16>(const CUtensorMap&, const DecodeParams&, cudaStream_t,
                                              const LaunchOpts&);
extern template cudaError_t launch_decode<32>(const CUtensorMap&, const DecodeParams&, cudaStream_t,
                                              const LaunchOpts&);
extern template cudaError_t launch_decode<64>(const CUtensorMap&, const DecodeParams&, cudaStream_t,
                                              const LaunchOpts&);
extern template cudaError_t launch_decode<128>(const CUtensorMap&, const DecodeParams&, cudaStream_t,
                                               const LaunchOpts&);

}  // namespace biloco
