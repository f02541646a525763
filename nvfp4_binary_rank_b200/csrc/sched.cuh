// Device-side scheduling helpers shared by the fused kernels: the stream-K
// split of the weight units over CTAs, warp reductions, and bounded waits that
// turn a lost arrival into an error status instead of a hung GPU.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace biloco {

// Stream-K bookkeeping in 32-bit unsigned arithmetic: the host limits T * KC to
// 2^24 units and G to the SM count, so every product stays below 2^32.
__device__ __forceinline__ int owner_cta(uint32_t u, int G, int U) {
  return static_cast<int>(((u + 1u) * static_cast<uint32_t>(G) - 1u) / static_cast<uint32_t>(U));
}
__device__ __forceinline__ int first_unit(int h, int G, int U) {
  return static_cast<int>(static_cast<uint32_t>(h) * static_cast<uint32_t>(U) / static_cast<uint32_t>(G));
}

// Reduce V per-lane values over the 32 lanes of a warp (recursive halving).
// Afterwards lane l holds in v[j] (j < max(1, V/32)) the total of entry
// reduce_out_index<V>(l, j).
template <int V>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[V], int lane) {
  int half = V / 2;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (half >= 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int j = 0; j < (V > 1 ? V / 2 : 1); ++j) {
        if (j < half) {
          const float send = upper ? v[j] : v[j + half];
          const float keep = upper ? v[j + half] : v[j];
          v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      half >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}
template <int V>
__device__ __forceinline__ int reduce_out_index(int lane, int j) {
  if constexpr (V >= 32) {
    return (V / 32) * lane + j;
  } else {
    constexpr int kLog = (V >= 16) ? 4 : (V >= 8) ? 3 : (V >= 4) ? 2 : (V >= 2) ? 1 : 0;
    return lane >> (5 - kLog);
  }
}

struct Ctl {
  volatile int* abort_flag;
  int* status;
};

__device__ __forceinline__ void fail(const Ctl& c) {
  *c.abort_flag = 1;
  record_error(c.status, kDevErrTimeout);
}

// Bounded spin on a global counter (every calling lane polls).
__device__ __forceinline__ bool spin_until_geq(const uint32_t* p, uint32_t target, const Ctl& c) {
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_gpu(p) < target) {
    if (*c.abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(32);
  }
  return true;
}

// Every thread of a named-barrier group waits on an mbarrier phase; the group
// then agrees (barrier + OR) on whether anyone gave up, so all leave together.
__device__ __forceinline__ bool group_wait(uint32_t bar, uint32_t parity, int bar_id, int nthreads,
                                           const Ctl& c) {
  // one lane per warp polls (the others would only load the shared-memory pipe)
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, c.abort_flag);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  const bool any_fail = named_barrier_or(bar_id, nthreads, !ok);
  if (any_fail) fail(c);
  return !any_fail;
}

}  // namespace biloco
