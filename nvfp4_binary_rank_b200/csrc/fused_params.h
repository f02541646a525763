// Parameters of the fused kernel, shared by the host launcher and the kernel.
#pragma once

#include <cstdint>

namespace biloco {

struct FusedParams {
  const uint8_t* w_sf;
  const uint8_t* x_sf;
  const float* gscale;
  const uint32_t* Ubits;
  const uint32_t* Vbits;
  const float* alpha;
  const uint16_t* x;
  uint16_t* y;
  float* zpart;        // [KC][M][rpad]
  float* zfin;         // [M][rpad]
  float* slots;        // [2 G][BN][128]
  uint32_t* z_ready;
  uint32_t* z_seen;
  uint32_t* tickets;   // [T] split-K tickets
  uint32_t* vtick;     // [T] V-side finaliser tickets
  int* status;
  int M, N, K, r;
  int KC, T, U, G, KW, rpad, RW;
  int mode;            // BILOCO_MODE_SHARED_Z or BILOCO_MODE_LOCAL_Z
  int inq;             // 1: activation quantised in-kernel (no pre-pass)
  int zdirect;         // 1: consumers sum the chunk partials themselves
  int fast;            // 1: the producer stages each unit's x chunk and V rows by TMA
  int unit_alu;        // 1: the CUDA-core warps have per-unit work (quantise and/or V side)
  int bxr;             // rows of the staged x box (16 or 32)
  int drop;            // failure-path self test (not used by this kernel)
};

}  // namespace biloco
