// Host-side declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "launch_common.h"

namespace biloco {

// Library-owned scratch of one (device, stream) pair.  All regions live in one
// cudaMalloc block; counters and the status word are zeroed when allocated.
struct Scratch {
  int device = -1;
  cudaStream_t stream = nullptr;
  void* base = nullptr;
  size_t bytes = 0;
  // carved regions
  int* status = nullptr;            // first device-side error of this stream
  uint32_t* counters = nullptr;     // rank-block arrivals, z ready/seen, tile tickets
  size_t counter_words = 0;
  uint8_t* act_fp4 = nullptr;       // [M][K/2]
  uint8_t* act_sf = nullptr;        // KC * 2048 scale atoms
  float* zpart = nullptr;           // [KC][M][rpad] z partial sums per 256-element chunk
  float* zfin = nullptr;            // [M][rpad] finished z
  float* slots = nullptr;           // [2 G][BN][128] split-K partials
};

struct ScratchNeed {
  size_t act_fp4, act_sf, zpart, zfin, slots, counter_words;
};

// Returns nullptr on allocation failure.
Scratch* get_scratch(cudaStream_t stream, const ScratchNeed& need);

int num_sms();

// Launchers (return cudaError_t values).
cudaError_t launch_quant_act_rowmajor(const uint16_t* x, int M, int K, uint8_t* codes, uint8_t* sf,
                                      cudaStream_t s);
cudaError_t launch_prep_act(const uint16_t* x, int M, int K, uint8_t* codes, uint8_t* sf_atoms,
                            cudaStream_t s);
cudaError_t launch_pack_weight(const float* R, int N, int K, uint8_t* W_fp4, uint8_t* W_sf,
                               float* gscale, cudaStream_t s);
cudaError_t launch_pack_signs(const float* S, int rows, int cols, uint32_t* bits, cudaStream_t s);
cudaError_t launch_wait_timeout(int* status, cudaStream_t s);

struct GemmArgs {
  const uint16_t* x;
  const uint8_t* W_fp4;
  const uint8_t* W_sf;
  const float* gscale;
  const uint32_t* Ubits;
  const uint32_t* Vbits;
  const float* alpha;
  uint16_t* y;
  int M, N, K, r;
  int mode;   // resolved: 1 shared z, 2 local z
  int drop;   // failure-path self test: grid arrivals the decode kernel skips
  int arith;  // resolved correction arithmetic: BILOCO_CORR_SIGNS or BILOCO_CORR_LUT
};

// Host checks of biloco_gemm's arguments (include/biloco.h); fills `a` with the
// resolved z schedule.  Returns BILOCO_OK or the error code, launching nothing.
int check_gemm_args(const void* x_bf16, const uint8_t* W_fp4, const uint8_t* W_sf, const float* gscale,
                    const uint32_t* Ubits, const uint32_t* Vbits, const float* alpha, void* y_bf16,
                    int M, int N, int K, int r, GemmArgs* a);

// Shape decomposition of one call: tiles, chunks, grid, kernel options and the
// scratch the call needs.
struct GemmPlan {
  int KC, T, U, G, KW, rpad, BN, bxr;
  bool inq, zdirect, shared_z, unit_alu, fast;
  bool decode;   // the decode-batch kernel (M <= 8, shared z) runs the call
  ScratchNeed need;
};
GemmPlan plan_gemm(const GemmArgs& a);

// Launches the call's kernels on `s`; `sc` holds at least `p.need`, with its
// status word and counters zero.  Returns a BILOCO_* status.
int launch_gemm(const GemmArgs& a, const GemmPlan& p, const Scratch& sc, cudaStream_t s);

// Validated arguments; per-stream scratch, then launch_gemm.  Returns a BILOCO_* status.
int run_gemm(const GemmArgs& a, cudaStream_t s);
int resolve_mode(int M, int N, int K, int r, int requested);
int resolve_arith(int M, int N, int K, int r, int requested);

// Status word of biloco_gemm_noalloc's static scratch on the current device:
// returned and, if non-zero, cleared together with its counters (synchronous).
int noalloc_take_status();
int gemm_kernel_count_for(const GemmArgs& a);

// Launch form of the GEMM kernels (biloco_set_launch).
LaunchOpts current_launch_opts();

}  // namespace biloco
