// Activation quantiser, weight packer and sign packer (BiLoCo README, sections
// "Decomposition" and "Kernel": NVFP4 residual and activation, pack_signs).
//
// All three are bandwidth-bound elementwise passes: one thread per 16-element
// block (two 16-byte loads, one 8-byte store), one warp per 32 sign bits.
#include <cstdint>
#include <cuda_runtime.h>

#include "internal.h"
#include "nvfp4_dev.cuh"
#include "ptx.cuh"

namespace biloco {

namespace {

constexpr int kQuantThreads = 256;

// Load the 16 BF16 values of block `blk` of row `m` (16-byte aligned).
__device__ __forceinline__ void load_bf16_block(const uint16_t* x, int K, int m, int blk,
                                                float (&v)[16]) {
  const uint4* p = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K + blk * 16);
  bf16x16_to_f32(__ldg(p), __ldg(p + 1), v);
}

__global__ void __launch_bounds__(kQuantThreads)
quant_act_rowmajor_kernel(const uint16_t* __restrict__ x, int M, int K, uint8_t* __restrict__ codes,
                          uint8_t* __restrict__ sf) {
  const int nb = K / 16;
  const long long id = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (id >= static_cast<long long>(M) * nb) return;
  const int m = static_cast<int>(id / nb), b = static_cast<int>(id % nb);
  float v[16];
  load_bf16_block(x, K, m, b, v);
  uint2 c;
  const uint32_t s = quant_act_block_fast(v, c);
  *reinterpret_cast<uint2*>(codes + static_cast<size_t>(m) * (K / 2) + b * 8) = c;
  sf[static_cast<size_t>(m) * nb + b] = static_cast<uint8_t>(s);
}

// Same quantiser, scales written into the GEMM's scale atoms.  Triggers the
// dependent fused kernel at entry so that its prologue and weight stream overlap.
// The scales of the blocks past K in the last 256-element chunk are written as
// zero: the tensor cores read them against zero codes, and the scratch they sit
// in may hold an earlier call's bytes.
__global__ void __launch_bounds__(kQuantThreads)
prep_act_kernel(const uint16_t* __restrict__ x, int M, int K, uint8_t* __restrict__ codes,
                uint8_t* __restrict__ sf_atoms) {
  griddep_launch_dependents();
  const int nb = K / 16;
  const int nb_pad = (K + 255) / 256 * 16;
  const long long id = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (id >= static_cast<long long>(M) * nb_pad) return;
  const int m = static_cast<int>(id / nb_pad), b = static_cast<int>(id % nb_pad);
  if (b >= nb) {
    sf_atoms[sf_atom_offset(static_cast<uint32_t>(m), static_cast<uint32_t>(b))] = 0;
    return;
  }
  float v[16];
  load_bf16_block(x, K, m, b, v);
  uint2 c;
  const uint32_t s = quant_act_block_fast(v, c);
  *reinterpret_cast<uint2*>(codes + static_cast<size_t>(m) * (K / 2) + b * 8) = c;
  sf_atoms[sf_atom_offset(static_cast<uint32_t>(m), static_cast<uint32_t>(b))] = static_cast<uint8_t>(s);
}

// ---- weight packer: amax(|R|) -> g -> codes and tile-layout scales

__global__ void __launch_bounds__(kQuantThreads)
amax_kernel(const float4* __restrict__ R, long long n4, uint32_t* __restrict__ amax_bits) {
  float a = 0.0f;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(R + i);
    a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  // non-negative floats order like their bit patterns
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(a));
}

__global__ void gscale_kernel(float* gscale) {
  const float amax = __uint_as_float(*reinterpret_cast<uint32_t*>(gscale));
  *gscale = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);     // 2688 = 6 * 448
}

__global__ void __launch_bounds__(kQuantThreads)
quant_weight_kernel(const float* __restrict__ R, int N, int K, const float* __restrict__ gscale,
                    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  const int nb = K / 16;
  const int KC = (K + 255) / 256;
  const int nb_pad = KC * 16;                       // scale slots per row incl. the zero tail
  const long long id = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (id >= static_cast<long long>(N) * nb_pad) return;
  const int n = static_cast<int>(id / nb_pad), b = static_cast<int>(id % nb_pad);
  const size_t tile_base = static_cast<size_t>(n / 128) * KC * 2048;
  uint8_t* sf_byte = sf + tile_base + sf_atom_offset(static_cast<uint32_t>(n & 127), b);
  if (b >= nb) {                                    // K is not a multiple of 256
    *sf_byte = 0;
    return;
  }
  const float g = __ldg(gscale);
  const float4* p = reinterpret_cast<const float4*>(R + static_cast<size_t>(n) * K + b * 16);
  float v[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 q = __ldg(p + j);
    v[4 * j] = q.x; v[4 * j + 1] = q.y; v[4 * j + 2] = q.z; v[4 * j + 3] = q.w;
  }
  const float d = __fmul_rn(6.0f, g);
  const uint32_t s = e4m3_from_f32(__fdiv_rn(amax16(v), d));
  const float S = __fmul_rn(e4m3_to_f32(s), g);
  *reinterpret_cast<uint2*>(codes + static_cast<size_t>(n) * (K / 2) + b * 8) = encode_block16(v, S);
  *sf_byte = static_cast<uint8_t>(s);
}

// ---- sign packer: one warp per output word

__global__ void __launch_bounds__(kQuantThreads)
pack_signs_kernel(const float* __restrict__ S, int rows, int cols, uint32_t* __restrict__ bits) {
  const int words = (cols + 31) / 32;
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<long long>(rows) * words) return;     // whole warp leaves together
  const int row = static_cast<int>(wid / words), w = static_cast<int>(wid % words);
  const int col = w * 32 + lane;
  const bool neg = (col < cols) && (__ldg(S + static_cast<size_t>(row) * cols + col) < 0.0f);
  const uint32_t word = __ballot_sync(0xffffffffu, neg);
  if (lane == 0) bits[static_cast<size_t>(row) * words + w] = word;
}

unsigned grid_for(long long threads) {
  return static_cast<unsigned>((threads + kQuantThreads - 1) / kQuantThreads);
}

}  // namespace

cudaError_t launch_quant_act_rowmajor(const uint16_t* x, int M, int K, uint8_t* codes, uint8_t* sf,
                                      cudaStream_t s) {
  const long long n = static_cast<long long>(M) * (K / 16);
  quant_act_rowmajor_kernel<<<grid_for(n), kQuantThreads, 0, s>>>(x, M, K, codes, sf);
  return cudaGetLastError();
}

cudaError_t launch_prep_act(const uint16_t* x, int M, int K, uint8_t* codes, uint8_t* sf_atoms,
                            cudaStream_t s) {
  const long long n = static_cast<long long>(M) * ((K + 255) / 256 * 16);
  prep_act_kernel<<<grid_for(n), kQuantThreads, 0, s>>>(x, M, K, codes, sf_atoms);
  return cudaGetLastError();
}

cudaError_t launch_pack_weight(const float* R, int N, int K, uint8_t* W_fp4, uint8_t* W_sf,
                               float* gscale, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(gscale, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  const long long n4 = static_cast<long long>(N) * K / 4;
  const unsigned g = static_cast<unsigned>(num_sms()) * 8u;
  amax_kernel<<<g, kQuantThreads, 0, s>>>(reinterpret_cast<const float4*>(R), n4,
                                          reinterpret_cast<uint32_t*>(gscale));
  gscale_kernel<<<1, 1, 0, s>>>(gscale);
  const long long nblk = static_cast<long long>(N) * ((K + 255) / 256) * 16;
  quant_weight_kernel<<<grid_for(nblk), kQuantThreads, 0, s>>>(R, N, K, gscale, W_fp4, W_sf);
  return cudaGetLastError();
}

// Failure-path self test: one warp waits, through the same bounded mbarrier wait
// the GEMM kernels use, on a phase nothing will complete.  The wait gives up after
// its wall-clock limit, and the kernel records the timeout in `status` and returns.
__global__ void wait_timeout_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(smem_u32(&bar), 0, &abort_flag)) record_error(status, kDevErrTimeout);
}

cudaError_t launch_wait_timeout(int* status, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(status);
  return cudaGetLastError();
}

cudaError_t launch_pack_signs(const float* S, int rows, int cols, uint32_t* bits, cudaStream_t s) {
  const long long warps = static_cast<long long>(rows) * ((cols + 31) / 32);
  pack_signs_kernel<<<grid_for(warps * 32), kQuantThreads, 0, s>>>(S, rows, cols, bits);
  return cudaGetLastError();
}

}  // namespace biloco
