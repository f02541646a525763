// Parameters of the decode-batch kernel (M <= 16), shared by its host launcher
// and the kernel.
#pragma once

#include <cstdint>

namespace biloco {

struct DecodeParams {
  const uint8_t* w_sf;     // weight scales, tile layout
  const float* gscale;     // weight tensor scale g
  const uint32_t* Ubits;   // [N][RW]
  const uint32_t* Vbits;   // [r][KW]
  const float* alpha;      // [r]
  const uint16_t* x;       // [M][K] BF16
  uint16_t* y;             // [M][N] BF16
  float* z;                // [M][rpad] scratch: z = alpha . (V^T x)
  uint8_t* ztiles;         // [16][32][128 B] scratch: z as BF16 high/low MMA tiles (4+ rows)
  uint8_t* xq;             // [KC][2304 B] scratch: quantised activation image (8+ rows)
  float* vpart;            // [G][16][128] scratch: V-side partial sums per piece (8+ rows)
  float* slots;            // [2 G][16][128] scratch: split-K partials
  uint32_t* z_ready;       // CTAs that published their z slice
  uint32_t* done;          // CTAs that finished (the last one resets the grid counters)
  uint32_t* tickets;       // [T] split-K arrivals per weight tile
  uint32_t* q_ready;       // CTAs that published their part of the activation image
  uint32_t* v_ready;       // 32-row class: CTAs that published their V pieces' partial sums
  int* status;             // first device-side error
  int M, N, K, r;
  int KC, T, U, G, KW, RW, rpad;
  int drop;                // failure-path self test: 1 skips the z arrivals, 2 the image arrivals
  int lut;                 // 1-2 rows: U z from the signed-sum table of z instead of sign-adds
};

}  // namespace biloco
