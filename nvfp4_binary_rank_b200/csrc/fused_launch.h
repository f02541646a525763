// Launchers of the fused kernel instances (one per MMA tile width and batch
// class; each lives in its own translation unit so they compile in parallel).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fused_params.h"

namespace biloco {

cudaError_t launch_fused_16_1(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl);
cudaError_t launch_fused_16_2(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl);
cudaError_t launch_fused_16_4(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl);
cudaError_t launch_fused_16_8(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl);
cudaError_t launch_fused_16_16(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl);
cudaError_t launch_fused_32_32(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl);
cudaError_t launch_fused_64_32(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl);
cudaError_t launch_fused_128_32(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                               const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl);

}  // namespace biloco
