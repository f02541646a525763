// Fused NVFP4 GEMM + binary-sign low-rank correction for one B200 (sm_100a).
//
//   y[m, n] = g * sum_k FP4(x)[m, k] FP4(R)[n, k]  +  sum_i U[n, i] z[m, i],
//   z[m, i] = alpha_i * sum_k V[k, i] x[m, k]
//
// (BiLoCo README, section "Kernel": FP4 GEMM on the tensor cores, z = alpha.(V x)
// on the CUDA cores from bit-packed V, U z expanded in the epilogue before the
// BF16 store, all in one launch.)
//
// Work decomposition ("swap-AB" + stream-K):
//   * The MMA's M dimension (128) runs over weight rows n, its N dimension (BN)
//     over activation rows m, so a decode batch of 1..32 rows wastes nothing on
//     padding to 128 activation rows.
//   * A "unit" is one 128-row weight tile times 256 elements of K: 16 KB of E2M1
//     codes (one 128-byte swizzled row per weight row) plus 2 KB of scales.  The
//     T * KC units are split into G contiguous ranges, one per CTA (G <= #SMs), so
//     every SM streams the same number of weight bytes.  A CTA's range covers
//     parts of at most a few tiles ("segments"); a tile cut between several CTAs
//     is summed through FP32 partial slots by the last CTA to arrive (ticket).
//   * The sign correction of a tile is split over the same contributors by rank
//     blocks in proportion to their share of the tile's K, so the CUDA-core work
//     is balanced exactly like the weight stream.
//
// Warp roles (14 warps):
//   warp 0      TMA producer: weight codes (2-D tiled, 128B swizzle), weight scales
//               (bulk copy of pre-tiled atoms), activation codes and scales
//   warp 1      TMEM allocator and tcgen05 MMA issuer (kind::mxf4nvf4, block16)
//   warps 2-5   epilogue: tcgen05.ld of the accumulator, g * acc + correction,
//               BF16 store or split-K partial + ticket
//   warps 6-13  CUDA-core sign correction: the V side (z slices) at entry and the
//               U side per segment
//
// z schedules:
//   shared z (mode 1)  every CTA computes one (K block, 16-rank block) slice of
//                      V^T x, publishes it to scratch and bumps an arrival counter;
//                      the last arrival of a rank block sums its K blocks, applies
//                      alpha and marks the block ready.  Tiles wait (bounded) for
//                      all rank blocks before their U side.
//   local z  (mode 2)  every CTA computes, over the whole K, the z ranks its own
//                      segments need; no cross-CTA traffic.
//
// Every wait (mbarrier or global counter) is bounded; on expiry the kernel records
// BILOCO_ERR_TIMEOUT in the stream's status word, drains its own copies and MMAs,
// frees its TMEM and returns.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/biloco.h"
#include "internal.h"
#include "nvfp4_dev.cuh"
#include "ptx.cuh"

namespace biloco {

namespace {

constexpr int kWarps = 14;
constexpr int kThreads = kWarps * 32;
constexpr int kEpiWarp0 = 2;
constexpr int kEpiThreads = 128;
constexpr int kAluWarp0 = 6;
constexpr int kAluWarps = 8;
constexpr int kAluThreads = kAluWarps * 32;
constexpr int kTileRows = 128;             // weight rows per tile = MMA M
constexpr int kUnitK = 256;                // K elements per unit
constexpr int kUnitBytesA = kTileRows * 128;
constexpr int kSfBytes = 2048;             // 4 scale atoms of 512 B per unit
constexpr int kRB = 16;                    // ranks per rank block
constexpr int kMP = 32;                    // activation rows per CUDA-core pass
constexpr int kMpad = 36;                  // padded row stride (floats) of staged tiles
constexpr int kXWords = 8;                 // 32-element words per staged x sub-block
constexpr int kZChunkBlocks = 8;           // rank blocks per staged z chunk
constexpr int kTmemCols = 512;
constexpr int kSfTmemBase = 256;           // TMEM column of the scale-factor regions

constexpr int kBarAlu = 1;                 // named barrier ids (0 is __syncthreads)
constexpr int kBarEpi = 2;

struct FusedParams {
  const uint8_t* w_sf;
  const uint8_t* x_sf;
  const float* gscale;
  const uint32_t* Ubits;
  const uint32_t* Vbits;
  const float* alpha;
  const uint16_t* x;
  const float* xsum32;
  uint16_t* y;
  float* zpart;
  float* zfin;
  float* zbsum;
  float* slots;
  uint32_t* rb_count;
  uint32_t* z_ready;
  uint32_t* z_seen;
  uint32_t* tickets;
  int* status;
  int M, N, K, r;
  int KC, T, U, G, KW, KB, IB, rpad, RW;
  int mode;
};

template <int BN, int ST>
struct Layout {
  static constexpr int kA = 0;
  static constexpr int kB = kA + ST * kUnitBytesA;
  static constexpr int kSFA = kB + ST * BN * 128;
  static constexpr int kSFB = kSFA + ST * kSfBytes;
  static constexpr int kXS = kSFB + ST * kSfBytes;                 // x sub-block [256][kMpad]
  static constexpr int kXSBytes = kXWords * 32 * kMpad * 4;
  static constexpr int kZS = kXS + kXSBytes;                        // z chunk [128][kMpad]
  static constexpr int kZSBytes = kZChunkBlocks * kRB * kMpad * 4;
  static constexpr int kZB = kZS + kZSBytes;                        // zbsum chunk [8][32]
  static constexpr int kVS = kZB + kZChunkBlocks * kMP * 4;         // V bits [16][8]
  static constexpr int kCorr = kVS + kRB * kXWords * 4;             // corr [2][32][128]
  static constexpr int kRed = kCorr + 2 * kMP * kTileRows * 4;      // k-split partials [8][64]
  static constexpr int kVOut = kRed + kAluWarps * 64 * 4;           // V-side result [32][16]
  static constexpr int kBar = kVOut + kMP * kRB * 4;
  static constexpr int kNumBars = 2 * ST + 7;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTotal = kMisc + 64;
  static constexpr int kAlloc = kTotal + 1024;
  static_assert(kB % 1024 == 0 && (BN * 128) % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kAlloc <= 232448, "shared memory budget");
};

// ------------------------------------------------------------------ small helpers

__device__ __forceinline__ int owner_cta(long long u, int G, int U) {
  return static_cast<int>(((u + 1) * G - 1) / U);
}
__device__ __forceinline__ int first_unit(int h, int G, int U) {
  return static_cast<int>(static_cast<long long>(h) * U / G);
}

// Predicated packed add: acc += (a, b) when flag != 0.
__device__ __forceinline__ void padd2(uint64_t& acc, float a, float b, uint32_t flag) {
  asm("{\n\t.reg .pred p;\n\t.reg .b64 t;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "mov.b64 t, {%2, %3};\n\t"
      "@p add.rn.f32x2 %0, %0, t;\n\t}"
      : "+l"(acc)
      : "r"(flag), "f"(a), "f"(b));
}
__device__ __forceinline__ void padd1(float& acc, float a, uint32_t flag) {
  asm("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %1, 0;\n\t@p add.rn.f32 %0, %0, %2;\n\t}"
      : "+f"(acc)
      : "r"(flag), "f"(a));
}
__device__ __forceinline__ float lo_f(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_f(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v >> 32));
}

// Reduce V per-lane values over the 32 lanes of a warp.  Afterwards lane l holds
// the totals of entries  out_index(l, j)  in v[j], j < max(1, V/32).
template <int V>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[V], int lane) {
  int half = V / 2;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (half >= 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int j = 0; j < V / 2; ++j) {
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
    // log2(V) halving steps used lane bits 4 .. 5-log2(V)
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

// Bounded spin on a global counter.
__device__ __forceinline__ bool spin_until_geq(const uint32_t* p, uint32_t target, const Ctl& c) {
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_gpu(p) < target) {
    if (*c.abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(64);
  }
  return true;
}

// One elected thread of a named-barrier group waits on an mbarrier; the whole
// group learns the outcome.  Returns false (uniformly) on timeout / abort.
__device__ __forceinline__ bool group_wait(uint32_t bar, uint32_t parity, bool elected, int bar_id,
                                           int nthreads, volatile int* shared_ok, const Ctl& c) {
  if (elected) {
    const bool ok = mbar_wait(bar, parity, c.abort_flag);
    if (!ok) fail(c);
    *shared_ok = ok ? 1 : 0;
  }
  named_barrier(bar_id, nthreads);
  const bool ok = *shared_ok != 0;
  named_barrier(bar_id, nthreads);     // everyone has read shared_ok before it is reused
  return ok;
}

// ------------------------------------------------------------------ V side

// P[m][i] = sum over words [w0, w1) of sum_{k in word, V[k][i0+i] = -1} x[m0+m][k]
// for i < 16, m < mcnt (<= 32); returned through red (smem) as res[m * 16 + i]
// in `out` (smem, [32][16]).  All 256 correction threads call this together.
template <int MG>
__device__ void vside_partial(const FusedParams& p, int m0, int mcnt, int i0, int nr, int w0, int w1,
                              float* x_s, uint32_t* v_s, float* red_s, float* out, int a, int lane,
                              int tid) {
  constexpr int kVals = 8 * MG;           // 8 ranks x MG rows per lane
  const int mgc = (mcnt + MG - 1) / MG;   // m groups
  const int groups = 2 * mgc;             // x 2 rank groups of 8
  int KS = 8 / groups;                    // k splits so that tasks == 8 warps
  if (KS < 1) KS = 1;
  const int tasks = groups * KS;
  const bool active = a < tasks;
  const int ks = a % KS, rest = a / KS, mg = rest % mgc, rg = rest / mgc;

  uint64_t acc2[8][(MG >= 2) ? MG / 2 : 1];
  float acc1[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    acc1[g] = 0.0f;
#pragma unroll
    for (int j = 0; j < ((MG >= 2) ? MG / 2 : 1); ++j) acc2[g][j] = 0ull;
  }
  const uint32_t lane_bit = 1u << lane;

  for (int ws = w0; ws < w1; ws += kXWords) {
    const int nw = min(kXWords, w1 - ws);
    named_barrier(kBarAlu, kAluThreads);          // previous sub-block consumed
    {
      const int kk = tid;                          // 256 threads <-> 256 k
      const bool in = kk < nw * 32;
      for (int m = 0; m < mcnt; ++m) {
        float v = 0.0f;
        if (in) v = bf16_bits_to_f32(__ldg(p.x + static_cast<size_t>(m0 + m) * p.K + ws * 32 + kk));
        x_s[kk * kMpad + m] = v;
      }
      if (tid < kRB * kXWords) {
        const int i = tid / kXWords, wl = tid % kXWords;
        uint32_t bits = 0;
        if (i < nr && wl < nw) bits = __ldg(p.Vbits + static_cast<size_t>(i0 + i) * p.KW + ws + wl);
        v_s[i * kXWords + wl] = bits;
      }
    }
    named_barrier(kBarAlu, kAluThreads);
    if (active) {
      const int wa = (ks * kXWords) / KS, wb = ((ks + 1) * kXWords) / KS;
      for (int wl = wa; wl < min(wb, nw); ++wl) {
        const float* xr = x_s + (wl * 32 + lane) * kMpad + mg * MG;
        float xv[MG];
        if constexpr (MG >= 4) {
#pragma unroll
          for (int j = 0; j < MG; j += 4) {
            const float4 q = *reinterpret_cast<const float4*>(xr + j);
            xv[j] = q.x; xv[j + 1] = q.y; xv[j + 2] = q.z; xv[j + 3] = q.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < MG; ++j) xv[j] = xr[j];
        }
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint32_t flag = v_s[(rg * 8 + g) * kXWords + wl] & lane_bit;
          if constexpr (MG >= 2) {
#pragma unroll
            for (int j = 0; j < MG / 2; ++j) padd2(acc2[g][j], xv[2 * j], xv[2 * j + 1], flag);
          } else {
            padd1(acc1[g], xv[0], flag);
          }
        }
      }
    }
  }
  // reduce over lanes, then over the k splits (fixed order)
  float vals[kVals];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    if constexpr (MG >= 2) {
#pragma unroll
      for (int j = 0; j < MG / 2; ++j) {
        vals[g * MG + 2 * j] = lo_f(acc2[g][j]);
        vals[g * MG + 2 * j + 1] = hi_f(acc2[g][j]);
      }
    } else {
      vals[g] = acc1[g];
    }
  }
  warp_reduce_scatter<kVals>(vals, lane);
  constexpr int kOut = (kVals >= 32) ? kVals / 32 : 1;
  if (active) {
#pragma unroll
    for (int j = 0; j < kOut; ++j) {
      const int e = reduce_out_index<kVals>(lane, j);
      // lanes that share an index after a partial reduction hold equal totals
      red_s[a * 64 + e] = vals[j];
    }
  }
  named_barrier(kBarAlu, kAluThreads);
  // out[m][i] for i < 16, m < mcnt: sum the KS partial tasks in order
  for (int idx = tid; idx < kMP * kRB; idx += kAluThreads) {
    const int m = idx / kRB, i = idx % kRB;
    float s = 0.0f;
    if (m < mcnt) {
      const int mgi = m / MG, mm = m % MG, rgi = i / 8, gg = i % 8;
      const int task0 = (rgi * mgc + mgi) * KS;
      for (int k2 = 0; k2 < KS; ++k2) s += red_s[(task0 + k2) * 64 + gg * MG + mm];
    }
    out[idx] = s;
  }
  named_barrier(kBarAlu, kAluThreads);
}

__device__ void vside_dispatch(const FusedParams& p, int m0, int mcnt, int i0, int nr, int w0, int w1,
                               float* x_s, uint32_t* v_s, float* red_s, float* out, int a, int lane,
                               int tid) {
  if (mcnt > 4)
    vside_partial<8>(p, m0, mcnt, i0, nr, w0, w1, x_s, v_s, red_s, out, a, lane, tid);
  else if (mcnt > 2)
    vside_partial<4>(p, m0, mcnt, i0, nr, w0, w1, x_s, v_s, red_s, out, a, lane, tid);
  else if (mcnt > 1)
    vside_partial<2>(p, m0, mcnt, i0, nr, w0, w1, x_s, v_s, red_s, out, a, lane, tid);
  else
    vside_partial<1>(p, m0, mcnt, i0, nr, w0, w1, x_s, v_s, red_s, out, a, lane, tid);
}

// ------------------------------------------------------------------ U side

// corr[rs][m][n] for the 128 rows of tile t, m in [m0, m0 + mcnt), ranks of
// rank blocks [b_lo, b_hi).  z comes from z_s (staged [i][kMpad]) and its block
// sums from zb_s.  Task a: rows 32 (a & 3) + lane; (a >> 2) selects the m half
// (mcnt > 16) or the rank-block parity (mcnt <= 16).
template <int MG>
__device__ void uside_chunk_accumulate(const FusedParams& p, int t, int blk0, int nblk,
                                       const float* z_s, uint64_t (&acc2)[MG >= 2 ? MG / 2 : 1],
                                       float& acc1, int mbase, int rs, int RS, int a, int lane) {
  const int n = t * kTileRows + (a & 3) * 32 + lane;
  const uint32_t* urow = p.Ubits + static_cast<size_t>(n) * p.RW;
  for (int bl = 0; bl < nblk; ++bl) {
    const int blk = blk0 + bl;
    if (RS == 2 && (blk & 1) != rs) continue;
    const uint32_t word = __ldg(urow + (blk >> 1)) >> ((blk & 1) * 16);
    const float* zr = z_s + (bl * kRB) * kMpad + mbase;
#pragma unroll
    for (int ii = 0; ii < kRB; ++ii) {
      const uint32_t flag = word & (1u << ii);
      if constexpr (MG >= 4) {
#pragma unroll
        for (int j = 0; j < MG; j += 4) {
          const float4 q = *reinterpret_cast<const float4*>(zr + ii * kMpad + j);
          padd2(acc2[j / 2], q.x, q.y, flag);
          padd2(acc2[j / 2 + 1], q.z, q.w, flag);
        }
      } else if constexpr (MG == 2) {
        const float2 q = *reinterpret_cast<const float2*>(zr + ii * kMpad);
        padd2(acc2[0], q.x, q.y, flag);
      } else {
        padd1(acc1, zr[ii * kMpad], flag);
      }
    }
  }
}

template <int MG>
__device__ bool uside_pass(const FusedParams& p, int t, int b_lo, int b_hi, int m0, int mcnt,
                           float* z_s, float* zb_s, float* corr_s, float* x_s, uint32_t* v_s,
                           float* red_s, float* vout, int a, int lane, int tid) {
  const int RS = (mcnt > 16) ? 1 : 2;
  const int rs = (RS == 2) ? (a >> 2) : 0;
  const int mbase = (RS == 1) ? (a >> 2) * 16 : 0;      // m offset within the pass
  const int mwidth = (RS == 1) ? 16 : MG;
  uint64_t acc2[MG >= 2 ? MG / 2 : 1];
#pragma unroll
  for (int j = 0; j < (MG >= 2 ? MG / 2 : 1); ++j) acc2[j] = 0ull;
  float acc1 = 0.0f;
  float zsum[MG];
#pragma unroll
  for (int j = 0; j < MG; ++j) zsum[j] = 0.0f;

  for (int c0 = b_lo; c0 < b_hi; c0 += kZChunkBlocks) {
    const int nblk = min(kZChunkBlocks, b_hi - c0);
    named_barrier(kBarAlu, kAluThreads);     // previous chunk consumed
    if (p.mode == BILOCO_MODE_SHARED_Z) {
      // stage z[m][16 c0 .. 16 (c0 + nblk)) -> z_s[i][m], block sums -> zb_s[bl][m]
      const int nr = nblk * kRB;
      for (int idx = tid; idx < nr * kMP; idx += kAluThreads) {
        const int m = idx / nr, i = idx % nr;
        float v = 0.0f;
        if (m < mcnt) v = __ldcg(p.zfin + static_cast<size_t>(m0 + m) * p.rpad + c0 * kRB + i);
        z_s[i * kMpad + m] = v;
      }
      for (int idx = tid; idx < nblk * kMP; idx += kAluThreads) {
        const int bl = idx / kMP, m = idx % kMP;
        zb_s[bl * kMP + m] = (m < mcnt) ? __ldcg(p.zbsum + static_cast<size_t>(c0 + bl) * p.M + m0 + m)
                                        : 0.0f;
      }
      named_barrier(kBarAlu, kAluThreads);
    } else {
      // local z: compute each rank block over the whole K right here
      for (int bl = 0; bl < nblk; ++bl) {
        const int blk = c0 + bl;
        const int i0 = blk * kRB, nr = min(kRB, p.r - i0);
        vside_dispatch(p, m0, mcnt, i0, nr, 0, p.KW, x_s, v_s, red_s, vout, a, lane, tid);
        // z = alpha_i * (sum_k x - 2 P)
        for (int idx = tid; idx < kMP * kRB; idx += kAluThreads) {
          const int m = idx / kRB, i = idx % kRB;
          float z = 0.0f;
          if (m < mcnt && i < nr) {
            float xs = 0.0f;
            for (int w = 0; w < p.KW; ++w)
              xs += __ldg(p.xsum32 + static_cast<size_t>(m0 + m) * p.KW + w);
            z = __fmul_rn(__ldg(p.alpha + i0 + i), xs - 2.0f * vout[idx]);
          }
          z_s[(bl * kRB + i) * kMpad + m] = z;
        }
        named_barrier(kBarAlu, kAluThreads);
        for (int idx = tid; idx < kMP; idx += kAluThreads) {
          float s = 0.0f;
          for (int i = 0; i < kRB; ++i) s += z_s[(bl * kRB + i) * kMpad + idx];
          zb_s[bl * kMP + idx] = s;
        }
        named_barrier(kBarAlu, kAluThreads);
      }
    }
    // accumulate this chunk
    uside_chunk_accumulate<MG>(p, t, c0, nblk, z_s, acc2, acc1, mbase, rs, RS, a, lane);
#pragma unroll
    for (int j = 0; j < MG; ++j) {
      if (j < mwidth) {
        float s = 0.0f;
        for (int bl = 0; bl < nblk; ++bl)
          if (RS == 1 || ((c0 + bl) & 1) == rs) s += zb_s[bl * kMP + mbase + j];
        zsum[j] += s;
      }
    }
  }
  // corr = zsum - 2 * acc, written as corr_s[rs][m][row]
  const int row = (a & 3) * 32 + lane;
  float accf[MG];
#pragma unroll
  for (int j = 0; j < MG; ++j) {
    if constexpr (MG >= 2) accf[j] = (j & 1) ? hi_f(acc2[j / 2]) : lo_f(acc2[j / 2]);
    else accf[j] = acc1;
  }
#pragma unroll
  for (int j = 0; j < MG; ++j) {
    const int m = mbase + j;
    if (j < mwidth && m < kMP) {
      corr_s[(rs * kMP + m) * kTileRows + row] = zsum[j] - 2.0f * accf[j];
      if (RS == 1) corr_s[(1 * kMP + m) * kTileRows + row] = 0.0f;
    }
  }
  return true;
}

__device__ void uside_dispatch(const FusedParams& p, int t, int b_lo, int b_hi, int m0, int mcnt,
                               float* z_s, float* zb_s, float* corr_s, float* x_s, uint32_t* v_s,
                               float* red_s, float* vout, int a, int lane, int tid) {
  if (mcnt > 8)
    uside_pass<16>(p, t, b_lo, b_hi, m0, mcnt, z_s, zb_s, corr_s, x_s, v_s, red_s, vout, a, lane, tid);
  else if (mcnt > 4)
    uside_pass<8>(p, t, b_lo, b_hi, m0, mcnt, z_s, zb_s, corr_s, x_s, v_s, red_s, vout, a, lane, tid);
  else if (mcnt > 2)
    uside_pass<4>(p, t, b_lo, b_hi, m0, mcnt, z_s, zb_s, corr_s, x_s, v_s, red_s, vout, a, lane, tid);
  else if (mcnt > 1)
    uside_pass<2>(p, t, b_lo, b_hi, m0, mcnt, z_s, zb_s, corr_s, x_s, v_s, red_s, vout, a, lane, tid);
  else
    uside_pass<1>(p, t, b_lo, b_hi, m0, mcnt, z_s, zb_s, corr_s, x_s, v_s, red_s, vout, a, lane, tid);
}

// ------------------------------------------------------------------ the kernel

template <int BN, int ST>
__global__ void __launch_bounds__(kThreads, 1)
fused_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
             const __grid_constant__ FusedParams p) {
  using L = Layout<BN, ST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[ST + s]); };
  auto accf_bar = [&](int b) { return smem_u32(&bars[2 * ST + b]); };
  auto acce_bar = [&](int b) { return smem_u32(&bars[2 * ST + 2 + b]); };
  const uint32_t corrf_bar = smem_u32(&bars[2 * ST + 4]);
  const uint32_t corre_bar = smem_u32(&bars[2 * ST + 5]);
  const uint32_t drain_bar = smem_u32(&bars[2 * ST + 6]);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* epi_ok = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  volatile int* alu_ok = reinterpret_cast<volatile int*>(smem + L::kMisc + 12);
  volatile int* epi_last = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);
  volatile int* alu_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 20);
  const Ctl ctl{abort_flag, p.status};

  const int g = blockIdx.x;
  const int u0 = first_unit(g, p.G, p.U), u1 = first_unit(g + 1, p.G, p.U);
  const int t_first = u0 / p.KC, t_last = (u1 - 1) / p.KC;
  const int nseg = t_last - t_first + 1;
  const int npass = (p.M + kMP - 1) / kMP;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), kEpiThreads);
    }
    mbar_init(corrf_bar, kAluThreads);
    mbar_init(corre_bar, kEpiThreads);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_x);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const int nunits = u1 - u0;
      const int pre = min(ST, nunits);
      const uint32_t stage_bytes = kUnitBytesA + BN * 128 + 2 * kSfBytes;
      // weight bytes do not depend on the activation quantiser: start them first
      for (int k = 0; k < pre; ++k) {
        const int u = u0 + k, t = u / p.KC, c = u % p.KC;
        mbar_arrive_expect_tx(full_bar(k), stage_bytes);
        tma_load_2d(smem_u32(smem + L::kA + k * kUnitBytesA), &tmap_w, full_bar(k), c * 128,
                    t * kTileRows);
        bulk_load(smem_u32(smem + L::kSFA + k * kSfBytes),
                  p.w_sf + (static_cast<size_t>(t) * p.KC + c) * kSfBytes, kSfBytes, full_bar(k));
      }
      griddep_wait();
      for (int k = 0; k < pre; ++k) {
        const int c = (u0 + k) % p.KC;
        tma_load_2d(smem_u32(smem + L::kB + k * BN * 128), &tmap_x, full_bar(k), c * 128, 0);
        bulk_load(smem_u32(smem + L::kSFB + k * kSfBytes), p.x_sf + static_cast<size_t>(c) * kSfBytes,
                  kSfBytes, full_bar(k));
      }
      int issued = pre;
      for (int k = pre; k < nunits; ++k) {
        const int s = k % ST;
        if (!mbar_wait(empty_bar(s), ((k / ST) - 1) & 1, abort_flag)) {
          fail(ctl);
          break;
        }
        const int u = u0 + k, t = u / p.KC, c = u % p.KC;
        mbar_arrive_expect_tx(full_bar(s), stage_bytes);
        tma_load_2d(smem_u32(smem + L::kA + s * kUnitBytesA), &tmap_w, full_bar(s), c * 128,
                    t * kTileRows);
        bulk_load(smem_u32(smem + L::kSFA + s * kSfBytes),
                  p.w_sf + (static_cast<size_t>(t) * p.KC + c) * kSfBytes, kSfBytes, full_bar(s));
        tma_load_2d(smem_u32(smem + L::kB + s * BN * 128), &tmap_x, full_bar(s), c * 128, 0);
        bulk_load(smem_u32(smem + L::kSFB + s * kSfBytes), p.x_sf + static_cast<size_t>(c) * kSfBytes,
                  kSfBytes, full_bar(s));
        ++issued;
      }
      // never leave the CTA with copies in flight: wait for the last fills
      for (int k = max(0, issued - ST); k < issued; ++k) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(full_bar(k % ST), (k / ST) & 1)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(p.status, kDevErrTimeout);
            break;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                             (static_cast<uint32_t>(kTileRows >> 4) << 24);
      int k = 0;
      bool ok = true;
      for (int seg = 0; seg < nseg && ok; ++seg) {
        const int t = t_first + seg;
        const int ua = max(u0, t * p.KC), ub = min(u1, (t + 1) * p.KC);
        const int b = seg & 1;
        if (seg >= 2 && !mbar_wait(acce_bar(b), ((seg >> 1) - 1) & 1, abort_flag)) {
          fail(ctl);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * BN);
        for (int u = ua; u < ub; ++u, ++k) {
          const int s = k % ST;
          if (!mbar_wait(full_bar(s), (k / ST) & 1, abort_flag)) {
            fail(ctl);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + kSfTmemBase + s * 32, sfb_t = sfa_t + 16;
          const uint32_t sfa_s = smem_u32(smem + L::kSFA + s * kSfBytes);
          const uint32_t sfb_s = smem_u32(smem + L::kSFB + s * kSfBytes);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tc_cp_32x128b_warpx4(sfa_t + 4 * j, smem_desc(sfa_s + 512 * j, 0, 128, 0));
            tc_cp_32x128b_warpx4(sfb_t + 4 * j, smem_desc(sfb_s + 512 * j, 0, 128, 0));
          }
          const uint64_t adesc = smem_desc(smem_u32(smem + L::kA + s * kUnitBytesA), 16, 1024, 2);
          const uint64_t bdesc = smem_desc(smem_u32(smem + L::kB + s * BN * 128), 16, 1024, 2);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tc_mma_nvf4(d_tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sfa_t + 4 * j, sfb_t + 4 * j,
                        (u > ua || j > 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(s));
        }
        if (ok) tc_commit(accf_bar(b));
      }
      // drain: every MMA and scale copy issued so far must finish before TMEM is freed
      tc_commit(drain_bar);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain_bar, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          record_error(p.status, kDevErrTimeout);
          break;
        }
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ---------------------------------------------------------------- epilogue
    const int et = threadIdx.x - kEpiWarp0 * 32;      // 0..127
    const int q = warp & 3;                            // TMEM lane quarter of this warp
    const int row = q * 32 + lane;                     // weight row within the tile
    const float gs = __ldg(p.gscale);
    int corr_round = 0;
    for (int seg = 0; seg < nseg; ++seg) {
      const int t = t_first + seg;
      const int b = seg & 1;
      const int hf = owner_cta(static_cast<long long>(t) * p.KC, p.G, p.U);
      const int hl = owner_cta(static_cast<long long>(t + 1) * p.KC - 1, p.G, p.U);
      const bool sole = hf == hl;
      const int which = (t == t_first) ? 0 : 1;
      float* my_slot = p.slots + static_cast<size_t>(2 * g + which) * BN * kTileRows;
      if (!group_wait(accf_bar(b), (seg >> 1) & 1, et == 0, kBarEpi, kEpiThreads, epi_ok, ctl)) break;
      tc_fence_after();
      bool ok = true;
      for (int pass = 0; pass < npass; ++pass) {
        const int m0 = pass * kMP, mcnt = min(kMP, p.M - m0);
        float v[kMP];
        {
          uint32_t raw[16];
          const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(b * BN + m0);
          tmem_ld16(taddr, raw);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(raw[j]);
          if (BN >= 32) {
            tmem_ld16(taddr + 16, raw);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[16 + j] = __uint_as_float(raw[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[16 + j] = 0.0f;
          }
        }
#pragma unroll
        for (int j = 0; j < kMP; ++j) v[j] = __fmul_rn(gs, v[j]);
        if (p.r > 0) {
          if (!group_wait(corrf_bar, corr_round & 1, et == 0, kBarEpi, kEpiThreads, epi_ok, ctl)) {
            ok = false;
            break;
          }
          const float* corr_s = reinterpret_cast<const float*>(smem + L::kCorr);
#pragma unroll
          for (int j = 0; j < kMP; ++j)
            v[j] += corr_s[(0 * kMP + j) * kTileRows + row] + corr_s[(1 * kMP + j) * kTileRows + row];
          mbar_arrive(corre_bar);
          ++corr_round;
        }
        if (sole) {
          uint16_t* yb = p.y + static_cast<size_t>(t) * kTileRows + row;
#pragma unroll
          for (int j = 0; j < kMP; ++j)
            if (j < mcnt) yb[static_cast<size_t>(m0 + j) * p.N] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
        } else {
#pragma unroll
          for (int j = 0; j < kMP; ++j)
            if (j < mcnt) my_slot[static_cast<size_t>(m0 + j) * kTileRows + row] = v[j];
        }
      }
      tc_fence_before();
      mbar_arrive(acce_bar(b));
      if (!ok) break;
      if (!sole) {
        __threadfence();
        named_barrier(kBarEpi, kEpiThreads);
        if (et == 0) {
          const uint32_t contributors = static_cast<uint32_t>(hl - hf + 1);
          const uint32_t old = atomicAdd(p.tickets + t, 1u);
          const bool last = (old == contributors - 1);
          if (last) atomicExch(p.tickets + t, 0u);
          __threadfence();
          *epi_last = last ? 1 : 0;
        }
        named_barrier(kBarEpi, kEpiThreads);
        const bool last = *epi_last != 0;
        named_barrier(kBarEpi, kEpiThreads);
        if (last) {
          for (int m = 0; m < p.M; ++m) {
            float s = 0.0f;
            for (int h = hf; h <= hl; ++h) {
              const int wh = (t == first_unit(h, p.G, p.U) / p.KC) ? 0 : 1;
              s += __ldcg(p.slots + (static_cast<size_t>(2 * h + wh) * BN + m) * kTileRows + row);
            }
            p.y[static_cast<size_t>(m) * p.N + static_cast<size_t>(t) * kTileRows + row] =
                __bfloat16_as_ushort(__float2bfloat16_rn(s));
          }
        }
      }
    }
  } else if (warp >= kAluWarp0 && warp < kAluWarp0 + kAluWarps && p.r > 0) {
    // ---------------------------------------------------------------- sign correction
    const int tid = threadIdx.x - kAluWarp0 * 32;   // 0..255
    const int a = warp - kAluWarp0;                  // task slot 0..7
    float* x_s = reinterpret_cast<float*>(smem + L::kXS);
    float* z_s = reinterpret_cast<float*>(smem + L::kZS);
    float* zb_s = reinterpret_cast<float*>(smem + L::kZB);
    uint32_t* v_s = reinterpret_cast<uint32_t*>(smem + L::kVS);
    float* corr_s = reinterpret_cast<float*>(smem + L::kCorr);
    float* red_s = reinterpret_cast<float*>(smem + L::kRed);
    float* vout = reinterpret_cast<float*>(smem + L::kVOut);
    bool ok = true;

    if (p.mode == BILOCO_MODE_SHARED_Z) {
      // V side: this CTA's slices (kb, ib) of V^T x
      const int items = p.KB * p.IB;
      float* part = vout;                    // [32][16] V-side result
      for (int item = g; item < items; item += p.G) {
        const int kb = item / p.IB, ib = item % p.IB;
        const int w0 = static_cast<int>(static_cast<long long>(kb) * p.KW / p.KB);
        const int w1 = static_cast<int>(static_cast<long long>(kb + 1) * p.KW / p.KB);
        const int i0 = ib * kRB, nr = min(kRB, p.r - i0);
        for (int pass = 0; pass < npass; ++pass) {
          const int m0 = pass * kMP, mcnt = min(kMP, p.M - m0);
          vside_dispatch(p, m0, mcnt, i0, nr, w0, w1, x_s, v_s, red_s, part, a, lane, tid);
          for (int idx = tid; idx < mcnt * kRB; idx += kAluThreads) {
            const int m = idx / kRB, i = idx % kRB;
            float xs = 0.0f;
            for (int w = w0; w < w1; ++w) xs += __ldg(p.xsum32 + static_cast<size_t>(m0 + m) * p.KW + w);
            p.zpart[((static_cast<size_t>(kb) * p.IB + ib) * p.M + m0 + m) * kRB + i] =
                xs - 2.0f * part[m * kRB + i];
          }
        }
        // publish; the last K block of this rank block finalises it
        __threadfence();
        named_barrier(kBarAlu, kAluThreads);
        if (tid == 0) {
          const uint32_t old = atomicAdd(p.rb_count + ib, 1u);
          const bool last = old == static_cast<uint32_t>(p.KB - 1);
          if (last) atomicExch(p.rb_count + ib, 0u);
          __threadfence();
          *alu_flag = last ? 1 : 0;
        }
        named_barrier(kBarAlu, kAluThreads);
        const bool last = *alu_flag != 0;
        named_barrier(kBarAlu, kAluThreads);
        if (last) {
          // warp-uniform trip count: the shuffles below need all 32 lanes
          for (int base = 0; base < p.M * kRB; base += kAluThreads) {
            const int idx = base + tid;
            const bool live = idx < p.M * kRB;
            const int m = idx / kRB, i = idx % kRB;
            float z = 0.0f;
            if (live) {
              float s = 0.0f;
              for (int kb2 = 0; kb2 < p.KB; ++kb2)
                s += __ldcg(p.zpart + ((static_cast<size_t>(kb2) * p.IB + ib) * p.M + m) * kRB + i);
              z = (i < nr) ? __fmul_rn(__ldg(p.alpha + i0 + i), s) : 0.0f;
              p.zfin[static_cast<size_t>(m) * p.rpad + i0 + i] = z;
            }
            // block sum over the 16 ranks (16 consecutive threads share m)
            float bs = z;
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) bs += __shfl_xor_sync(0xffffffffu, bs, o);
            if (live && i == 0) p.zbsum[static_cast<size_t>(ib) * p.M + m] = bs;
          }
          __threadfence();
          named_barrier(kBarAlu, kAluThreads);
          if (tid == 0) atomicAdd(p.z_ready, 1u);
        }
      }
      // wait until every rank block is final, then count ourselves out
      if (tid == 0) {
        bool okw = spin_until_geq(p.z_ready, static_cast<uint32_t>(p.IB), ctl);
        if (!okw) fail(ctl);
        *alu_ok = okw ? 1 : 0;
        if (okw) {
          const uint32_t old = atomicAdd(p.z_seen, 1u);
          if (old == static_cast<uint32_t>(p.G - 1)) {
            atomicExch(p.z_ready, 0u);
            atomicExch(p.z_seen, 0u);
          }
        }
      }
      named_barrier(kBarAlu, kAluThreads);
      ok = *alu_ok != 0;
      named_barrier(kBarAlu, kAluThreads);
    }

    // U side, one (segment, pass) at a time, handed to the epilogue through corr_s
    const int IBn = (p.r + kRB - 1) / kRB;
    int corr_round = 0;
    for (int seg = 0; seg < nseg && ok; ++seg) {
      const int t = t_first + seg;
      const int ua = max(u0, t * p.KC) - t * p.KC, ub = min(u1, (t + 1) * p.KC) - t * p.KC;
      const int b_lo = static_cast<int>(static_cast<long long>(IBn) * ua / p.KC);
      const int b_hi = static_cast<int>(static_cast<long long>(IBn) * ub / p.KC);
      for (int pass = 0; pass < npass; ++pass) {
        const int m0 = pass * kMP, mcnt = min(kMP, p.M - m0);
        if (corr_round > 0 &&
            !group_wait(corre_bar, (corr_round - 1) & 1, tid == 0, kBarAlu, kAluThreads, alu_ok, ctl)) {
          ok = false;
          break;
        }
        uside_dispatch(p, t, b_lo, b_hi, m0, mcnt, z_s, zb_s, corr_s, x_s, v_s, red_s, vout, a, lane, tid);
        mbar_arrive(corrf_bar);
        ++corr_round;
      }
    }
    if (ok && corr_round > 0)
      group_wait(corre_bar, (corr_round - 1) & 1, tid == 0, kBarAlu, kAluThreads, alu_ok, ctl);
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D byte tensor [rows][inner_bytes], box [box_rows][128 B], 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner_bytes, rows};
  const cuuint64_t strides[1] = {inner_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int ST>
cudaError_t launch_fused(const CUtensorMap& tw, const CUtensorMap& tx, const FusedParams& fp,
                         cudaStream_t s) {
  using L = Layout<BN, ST>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(fused_kernel<BN, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(fp.G));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fused_kernel<BN, ST>, tw, tx, fp);
}

int pick_bn(int M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

}  // namespace

int resolve_mode(int M, int N, int K, int r, int requested) {
  (void)M; (void)N; (void)K; (void)r;
  if (requested == BILOCO_MODE_SHARED_Z || requested == BILOCO_MODE_LOCAL_Z) return requested;
  return BILOCO_MODE_SHARED_Z;
}

int run_gemm(const GemmArgs& a, cudaStream_t s) {
  const int M = a.M, N = a.N, K = a.K, r = a.r;
  const int KC = (K + kUnitK - 1) / kUnitK;
  const int T = N / kTileRows;
  const int U = T * KC;
  const int G = std::min(num_sms(), U);
  const int KW = K / 32;
  const int IB = (r + kRB - 1) / kRB;
  const int KB = (IB > 0) ? std::max(1, std::min(KW, G / IB)) : 1;
  const int rpad = std::max(IB, 1) * kRB;
  const int BN = pick_bn(M);

  ScratchNeed need;
  need.act_fp4 = static_cast<size_t>(M) * K / 2;
  need.act_sf = static_cast<size_t>(KC) * kSfBytes;
  need.xsum32 = static_cast<size_t>(M) * KW * 4;
  need.zpart = static_cast<size_t>(std::max(KB * IB, 1)) * M * kRB * 4;
  need.zfin = static_cast<size_t>(M) * rpad * 4;
  need.zbsum = static_cast<size_t>(std::max(IB, 1)) * M * 4;
  need.slots = static_cast<size_t>(2 * G) * BN * kTileRows * 4;
  need.counter_words = static_cast<size_t>(std::max(IB, 1)) + 2 + T;
  Scratch* sc = get_scratch(s, need);
  if (!sc) return BILOCO_ERR_NOMEM;

  cudaError_t e = launch_prep_act(a.x, M, K, sc->act_fp4, sc->act_sf, sc->xsum32, s);
  if (e != cudaSuccess) return BILOCO_ERR_CUDA;

  CUtensorMap tw, tx;
  if (!make_tmap(&tw, a.W_fp4, static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(N), kTileRows))
    return BILOCO_ERR_CUDA;
  if (!make_tmap(&tx, sc->act_fp4, static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(M), BN))
    return BILOCO_ERR_CUDA;

  FusedParams fp = {};
  fp.w_sf = a.W_sf;
  fp.x_sf = sc->act_sf;
  fp.gscale = a.gscale;
  fp.Ubits = a.Ubits;
  fp.Vbits = a.Vbits;
  fp.alpha = a.alpha;
  fp.x = a.x;
  fp.xsum32 = sc->xsum32;
  fp.y = a.y;
  fp.zpart = sc->zpart;
  fp.zfin = sc->zfin;
  fp.zbsum = sc->zbsum;
  fp.slots = sc->slots;
  fp.rb_count = sc->counters;
  fp.z_ready = sc->counters + std::max(IB, 1);
  fp.z_seen = fp.z_ready + 1;
  fp.tickets = fp.z_seen + 1;
  fp.status = sc->status;
  fp.M = M; fp.N = N; fp.K = K; fp.r = r;
  fp.KC = KC; fp.T = T; fp.U = U; fp.G = G; fp.KW = KW; fp.KB = KB; fp.IB = IB;
  fp.rpad = rpad;
  fp.RW = (r + 31) / 32;
  fp.mode = a.mode;

  switch (BN) {
    case 16: e = launch_fused<16, 6>(tw, tx, fp, s); break;
    case 32: e = launch_fused<32, 5>(tw, tx, fp, s); break;
    case 64: e = launch_fused<64, 4>(tw, tx, fp, s); break;
    default: e = launch_fused<128, 3>(tw, tx, fp, s); break;
  }
  return e == cudaSuccess ? BILOCO_OK : BILOCO_ERR_CUDA;
}

}  // namespace biloco
