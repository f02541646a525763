// Launchers of the decode-batch kernel instances (batch classes 1, 2, 4, 8 and
// 16 activation rows; each in its own translation unit).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "decode_params.h"

namespace biloco {

// Units of 128 weight rows x 256 K elements one CTA of the decode kernel can hold.
constexpr int kDecodeMaxUnits = 16;
constexpr int kDecodeMaxRows = 16;
// Bytes per 256-element K chunk of the kernel's quantised activation image
// (16 rows x 128 B of codes, 256 B of scales).
constexpr int kDecodeQImgBytes = 16 * 128 + 256;

cudaError_t launch_decode_1(const CUtensorMap& tw, const DecodeParams& dp, cudaStream_t s);
cudaError_t launch_decode_2(const CUtensorMap& tw, const DecodeParams& dp, cudaStream_t s);
cudaError_t launch_decode_4(const CUtensorMap& tw, const DecodeParams& dp, cudaStream_t s);
cudaError_t launch_decode_8(const CUtensorMap& tw, const DecodeParams& dp, cudaStream_t s);
cudaError_t launch_decode_16(const CUtensorMap& tw, const DecodeParams& dp, cudaStream_t s);

}  // namespace biloco
