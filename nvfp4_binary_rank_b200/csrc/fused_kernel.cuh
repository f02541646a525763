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
//   * The MMA's M dimension (128) runs over weight rows n and its N dimension (BN)
//     over activation rows m, so a decode batch of 1..32 rows is not padded to
//     128 activation rows.
//   * A "unit" is one 128-row weight tile times one 256-element chunk of K:
//     16 KB of E2M1 codes (a 128-byte swizzled row per weight row) plus 2 KB of
//     scales.  The T * KC units are cut into G contiguous ranges, one per CTA
//     (G <= #SMs), so every SM streams the same number of weight bytes.  A range
//     covers parts of one or a few tiles ("segments"); a tile split between CTAs
//     is summed through FP32 partial slots by the last CTA to arrive (ticket).
//   * The sign correction rides on the same units.  Unit (t, c) computes the
//     chunk-c part of V^T x for tile t's slice of the ranks (every chunk's ranks
//     are spread over the T tiles), and the U side of a tile is split over its
//     contributors in rank blocks proportional to their share of the tile's K.
//     Both halves are therefore balanced exactly like the weight stream.
//   * Small batches (M <= 8) quantise the activation chunk in the CTA that uses
//     it, straight from the staged BF16 chunk into the swizzled B tile and its
//     scale atoms; larger batches take it from a pre-pass kernel (launched before,
//     overlapped through programmatic dependent launch).
//
// Warp roles (14 warps):
//   warp 0      TMA producer: weight codes (2-D tiled, 128B swizzle), weight scales
//               (bulk copy of pre-tiled atoms), activation codes and scales
//   warp 1      TMEM allocator and tcgen05 MMA issuer (kind::mxf4nvf4, block16)
//   warps 2-5   epilogue: tcgen05.ld of the accumulator, g * acc + correction,
//               BF16 store or split-K partial + ticket
//   warps 6-13  CUDA cores: activation quantisation (small M), V side per unit,
//               U side per segment
//
// z schedules:
//   shared z (mode 1)  units publish chunk partials of V^T x; once every CTA has
//                      published (one arrival counter; for larger batches a
//                      per-tile finaliser sums the chunks first), each CTA reads the
//                      z ranks of its rank shares.
//   local z  (mode 2)  every CTA computes, over the whole K, the z ranks its own
//                      segments need; no cross-CTA traffic.
//
// Every wait (mbarrier or global counter) is bounded; on expiry the kernel records
// BILOCO_ERR_TIMEOUT in the stream's status word, drains its own copies and MMAs,
// frees its TMEM and returns.
#pragma once

#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/biloco.h"
#include "fused_launch.h"
#include "fused_params.h"
#include "nvfp4_dev.cuh"
#include "ptx.cuh"
#include "sched.cuh"

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
constexpr int kUnitK = 256;                // K elements per unit (chunk)
constexpr int kUnitBytesA = kTileRows * 128;
constexpr int kSfBytes = 2048;             // 4 scale atoms of 512 B per unit
constexpr int kRB = 16;                    // ranks per U-side rank block
constexpr int kMP = 32;                    // activation rows per CUDA-core pass
constexpr int kMpad = 36;                  // padded row stride (floats) of staged z
constexpr int kXWords = 8;                 // 32-element words per chunk
constexpr int kSubK = kXWords * 32;        // K elements per staged x chunk
constexpr int kVRanks = 32;                // V-side ranks per computed sub-range
constexpr int kVStageRanks = 64;           // V rows staged per unit by TMA (fast path)
constexpr int kZChunkBlocks = 8;           // rank blocks per staged z chunk
constexpr int kTmemCols = 512;
constexpr int kSfTmemBase = 256;           // TMEM column of the scale-factor regions
constexpr int kInKernelQuantMaxM = 8;

constexpr int kBarAlu = 1;                 // named barrier ids (0 is __syncthreads)
constexpr int kBarEpi = 2;



template <int BN, int ST>
struct Layout {
  static constexpr int kA = 0;
  static constexpr int kB = kA + ST * kUnitBytesA;
  static constexpr int kSFA = kB + ST * BN * 128;
  static constexpr int kSFB = kSFA + ST * kSfBytes;
  // per-stage x chunk + V rows staged by TMA (fast path); the cp.async fallback
  // uses the start of the same region as its double buffer
  static constexpr int kXRows = (BN <= 16) ? 16 : 32;
  static constexpr int kXBytes = kXRows * kSubK * 2;
  static constexpr int kVBytes = kVStageRanks * kXWords * 4;
  static constexpr int kXStride = kXBytes + kVBytes;
  static constexpr int kFallbackBytes = 2 * kMP * kSubK * 2 + 2 * kVRanks * kXWords * 4;
  static constexpr int kXSRegion = (BN <= 32) ? ((ST * kXStride > kFallbackBytes) ? ST * kXStride
                                                                                   : kFallbackBytes)
                                              : kFallbackBytes;
  static constexpr int kXS = kSFB + ST * kSfBytes;
  static constexpr int kXB = kXS;                                    // fallback x [2][32][256]
  static constexpr int kVB = kXB + 2 * kMP * kSubK * 2;              // fallback V [2][32][8]
  static constexpr int kZS = kXS + kXSRegion;                        // z chunk [128][kMpad]
  static constexpr int kZB = kZS + kZChunkBlocks * kRB * kMpad * 4;  // z block sums [8][32]
  static constexpr int kCorr = kZB + kZChunkBlocks * kMP * 4;        // corr [2][32][128]
  static constexpr int kRed = kCorr + 2 * kMP * kTileRows * 4;       // task partials [8][256]
  static constexpr int kVOut = kRed + kAluWarps * 256 * 4;           // V-side result [32][32]
  static constexpr int kXsw = kVOut + kMP * kVRanks * 4;             // x sums per warp [8][32]
  static constexpr int kXsum = kXsw + kAluWarps * kMP * 4;           // x sums [32]
  static constexpr int kBar = kXsum + kMP * 4;
  static constexpr int kNumBars = 3 * ST + 8;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTotal = kMisc + 64;
  static constexpr int kAlloc = kTotal + 1024;
  static_assert(kB % 1024 == 0 && (BN * 128) % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kXB % 16 == 0 && kVB % 16 == 0, "cp.async destinations need 16-byte alignment");
  static_assert(kAlloc <= 232448, "shared memory budget");
};

// ------------------------------------------------------------------ small helpers

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

// Tile t's slice of the ranks on the V side: [t r / T, (t + 1) r / T).
__device__ __forceinline__ void vside_ranks(const FusedParams& p, int t, int& i_lo, int& i_hi) {
  i_lo = static_cast<int>(static_cast<uint32_t>(t) * static_cast<uint32_t>(p.r) / static_cast<uint32_t>(p.T));
  i_hi = static_cast<int>(static_cast<uint32_t>(t + 1) * static_cast<uint32_t>(p.r) / static_cast<uint32_t>(p.T));
}

// U-side rank blocks of tile t handled by the segment covering units [ua, ub)
// of the tile (offsets within the tile): proportional to its share of K.
__device__ __forceinline__ void rank_share(const FusedParams& p, int ua, int ub, int& b_lo, int& b_hi) {
  const int IBn = (p.r + kRB - 1) / kRB;
  b_lo = static_cast<int>(static_cast<uint32_t>(IBn) * static_cast<uint32_t>(ua) / static_cast<uint32_t>(p.KC));
  b_hi = static_cast<int>(static_cast<uint32_t>(IBn) * static_cast<uint32_t>(ub) / static_cast<uint32_t>(p.KC));
}

// ------------------------------------------------------------------ staging

// Activation rows m0 .. m0+mcnt, words [ws, ws + nw) (BF16 as stored) -> xb [32][256].
__device__ __forceinline__ void stage_x(const FusedParams& p, int m0, int mcnt, int ws, int nw,
                                        uint16_t* xb, int tid) {
  const int per_row = nw * 4;                       // 16-byte pieces per row
  for (int idx = tid; idx < mcnt * per_row; idx += kAluThreads) {
    const int m = idx / per_row, piece = idx % per_row;
    cp_async16(smem_u32(xb + m * kSubK + piece * 8),
               p.x + static_cast<size_t>(m0 + m) * p.K + static_cast<size_t>(ws) * 32 + piece * 8);
  }
}
// Sign rows i0 .. i0+nr, words [ws, ws + nw) -> vb [nr][8].
__device__ __forceinline__ void stage_v(const FusedParams& p, int i0, int nr, int ws, int nw,
                                        uint32_t* vb, int tid) {
  for (int idx = tid; idx < nr * nw; idx += kAluThreads) {
    const int i = idx / nw, wl = idx % nw;
    cp_async4(smem_u32(vb + i * kXWords + wl), p.Vbits + static_cast<size_t>(i0 + i) * p.KW + ws + wl);
  }
}

// ------------------------------------------------------------------ V side

// One task (warp) over a staged chunk: for ranks 8 rg .. 8 rg + 7 of the staged
// sign rows and activation rows MG mg .. MG mg + MG-1, accumulate the x whose
// sign is -1 over words [wa, wb).  Lane l takes bit l of every word.
template <int MG>
__device__ __forceinline__ void vside_task_accumulate(const uint16_t* xb, const uint32_t* vb, int rg,
                                                      int mg, int wa, int wb, int lane,
                                                      uint64_t (&acc2)[8][(MG >= 2) ? MG / 2 : 1],
                                                      float (&acc1)[8]) {
  const uint32_t lane_bit = 1u << lane;
  const uint16_t* xs = xb + (mg * MG) * kSubK + lane;
  const uint32_t* vs = vb + (rg * 8) * kXWords;
  for (int wl = wa; wl < wb; ++wl) {
    float xv[MG];
#pragma unroll
    for (int mm = 0; mm < MG; ++mm) xv[mm] = bf16_bits_to_f32(xs[mm * kSubK + wl * 32]);
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const uint32_t flag = vs[g * kXWords + wl] & lane_bit;
      if constexpr (MG >= 2) {
#pragma unroll
        for (int q = 0; q < MG / 2; ++q) padd2(acc2[g][q], xv[2 * q], xv[2 * q + 1], flag);
      } else {
        padd1(acc1[g], xv[0], flag);
      }
    }
  }
}

// Reduce a task's accumulators over its lanes and store them in red_slot[.].
template <int MG>
__device__ __forceinline__ void vside_task_finish(uint64_t (&acc2)[8][(MG >= 2) ? MG / 2 : 1],
                                                  float (&acc1)[8], float* red_slot, bool store,
                                                  int lane) {
  constexpr int kVals = 8 * MG;
  float vals[kVals];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    if constexpr (MG >= 2) {
#pragma unroll
      for (int q = 0; q < MG / 2; ++q) {
        vals[g * MG + 2 * q] = lo_f(acc2[g][q]);
        vals[g * MG + 2 * q + 1] = hi_f(acc2[g][q]);
      }
    } else {
      vals[g] = acc1[g];
    }
  }
  warp_reduce_scatter<kVals>(vals, lane);
  constexpr int kOut = (kVals >= 32) ? kVals / 32 : 1;
  if (store) {
#pragma unroll
    for (int j = 0; j < kOut; ++j) red_slot[reduce_out_index<kVals>(lane, j)] = vals[j];
  }
}

// out[m * kVRanks + i] = sum over the staged words [0, nw) of the x[m][k] whose
// sign V[k][i] is -1, for m < mcnt (<= 32), i < nr (<= 64).  Whole group.
template <int MG>
__device__ __forceinline__ void vside_chunk(const uint16_t* xb, const uint32_t* vb, int mcnt, int nr, int nw,
                            float* red_s, float* out, int a, int lane, int tid) {
  constexpr int kPairs = (MG >= 2) ? MG / 2 : 1;
  const int mgc = (mcnt + MG - 1) / MG;
  const int rgc = (nr + 7) / 8;
  const int groups = rgc * mgc;
  int KS = kAluWarps / groups;
  if (KS < 1) KS = 1;
  const int tasks = groups * KS;
  for (int base = 0; base < tasks; base += kAluWarps) {
    const int task = base + a;
    const bool active = task < tasks;
    const int ks = task % KS, rest = task / KS, mg = rest % mgc, rg = rest / mgc;
    uint64_t acc2[8][kPairs];
    float acc1[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      acc1[g] = 0.0f;
#pragma unroll
      for (int q = 0; q < kPairs; ++q) acc2[g][q] = 0ull;
    }
    if (active) {
      const int wa = (ks * kXWords) / KS, wb = min(nw, ((ks + 1) * kXWords) / KS);
      vside_task_accumulate<MG>(xb, vb, rg, mg, wa, wb, lane, acc2, acc1);
    }
    vside_task_finish<MG>(acc2, acc1, red_s + a * 64, active, lane);
    named_barrier(kBarAlu, kAluThreads);
    // combine the k splits in order
    const int nout = min(tasks - base, kAluWarps) / KS;    // (rank group, m group) pairs this round
    for (int idx = tid; idx < nout * 8 * MG; idx += kAluThreads) {
      const int pair = idx / (8 * MG), e = idx % (8 * MG);
      const int pg = base / KS + pair;                     // global pair index
      const int mgi = pg % mgc, rgi = pg / mgc;
      const int m = mgi * MG + e % MG, i = rgi * 8 + e / MG;
      float s = 0.0f;
      for (int k2 = 0; k2 < KS; ++k2) s += red_s[(pair * KS + k2) * 64 + e];
      if (m < mcnt && i < nr) out[m * kVRanks + i] = s;
    }
    named_barrier(kBarAlu, kAluThreads);
  }
}


// xs_s[m] = sum of the staged chunk row m (fixed order: lanes, then warps).
template <int V>
__device__ __forceinline__ void chunk_xsum(const uint16_t* xb, int mcnt, int nw, float* xsw, float* xs_s, int a,
                           int lane, int tid) {
  float v[V];
  const bool in = tid < nw * 32;
#pragma unroll
  for (int m = 0; m < V; ++m) v[m] = (m < mcnt && in) ? bf16_bits_to_f32(xb[m * kSubK + tid]) : 0.0f;
  warp_reduce_scatter<V>(v, lane);
  // lanes that share an index after a partial reduction hold the same total
  xsw[a * kMP + reduce_out_index<V>(lane, 0)] = v[0];
  named_barrier(kBarAlu, kAluThreads);
  if (tid < mcnt) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kAluWarps; ++w) s += xsw[w * kMP + tid];
    xs_s[tid] = s;
  }
  named_barrier(kBarAlu, kAluThreads);
}


// ------------------------------------------------------------------ activation quantisation

// Rows m < mcnt of the staged chunk (its first nw words) -> B tile (BN rows x 128 B,
// 128-byte swizzle: 16-byte piece j of row m sits at piece j ^ (m & 7)) and the
// chunk's 4 scale atoms.  Blocks past K keep whatever finite codes the stage held;
// the weight codes there are zero-filled by TMA.
__device__ __forceinline__ void quant_chunk(const uint16_t* xb, int mcnt, int nw, uint8_t* btile, uint8_t* sfb, int tid) {
  const int nblk = 2 * nw;
  for (int idx = tid; idx < mcnt * nblk; idx += kAluThreads) {
    const int m = idx / nblk, blk = idx % nblk;
    const uint4* src = reinterpret_cast<const uint4*>(xb + m * kSubK + blk * 16);
    float v[16];
    bf16x16_to_f32(src[0], src[1], v);
    uint2 codes;
    const uint32_t s = quant_act_block_fast(v, codes);
    const int j = blk * 8;
    *reinterpret_cast<uint2*>(btile + m * 128 + ((((j >> 4) ^ (m & 7)) << 4) | (j & 15))) = codes;
    sfb[(blk >> 2) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (blk & 3)] = static_cast<uint8_t>(s);
  }
}

// ------------------------------------------------------------------ batched V side

// The V side of a batch of staged units as independent warp tasks: task =
// (unit j, group of 8 ranks rg, group of MG batch rows mg), over the unit's whole
// chunk.  Lane l takes bit l of every 32-element word; the task's 8*MG sums are
// reduced over the lanes, its row sums of x over the whole warp, and the lanes
// store zpart = sum_k x - 2 * sum_{sign -1} x directly.  No group barrier.
template <int MG, typename UnitInfo>
__device__ __forceinline__ void vside_batch(const FusedParams& p, int nb, int mcnt, int rgu, UnitInfo info,
                                            float* xs_w, int a, int lane) {
  constexpr int kPairs = (MG >= 2) ? MG / 2 : 1;
  constexpr int kVals = 8 * MG;
  const int mgc = (mcnt + MG - 1) / MG;
  const int tasks = nb * rgu * mgc;
  const uint32_t lane_bit = 1u << lane;
  for (int task = a; task < tasks; task += kAluWarps) {
    const int j = task / (rgu * mgc), rest = task % (rgu * mgc), rg = rest / mgc, mg = rest % mgc;
    const uint16_t* xc;
    const uint32_t* vrows;
    int c, i_lo, nr, nw;
    info(j, xc, vrows, c, i_lo, nr, nw);
    if (rg * 8 >= nr) continue;                      // uniform over the warp
    uint64_t acc2[8][kPairs];
    float acc1[8];
    float xacc[MG];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      acc1[g] = 0.0f;
#pragma unroll
      for (int q = 0; q < kPairs; ++q) acc2[g][q] = 0ull;
    }
#pragma unroll
    for (int mm = 0; mm < MG; ++mm) xacc[mm] = 0.0f;
    const uint16_t* xs = xc + (mg * MG) * kSubK + lane;
    const uint32_t* vs = vrows + (rg * 8) * kXWords;
    for (int w = 0; w < nw; ++w) {
      float xv[MG];
#pragma unroll
      for (int mm = 0; mm < MG; ++mm) {
        xv[mm] = bf16_bits_to_f32(xs[mm * kSubK + w * 32]);
        xacc[mm] += xv[mm];
      }
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const uint32_t flag = vs[g * kXWords + w] & lane_bit;
        if constexpr (MG >= 2) {
#pragma unroll
          for (int q = 0; q < MG / 2; ++q) padd2(acc2[g][q], xv[2 * q], xv[2 * q + 1], flag);
        } else {
          padd1(acc1[g], xv[0], flag);
        }
      }
    }
    // row sums of x over the warp (every lane gets all MG of them)
#pragma unroll
    for (int mm = 0; mm < MG; ++mm) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) xacc[mm] += __shfl_xor_sync(0xffffffffu, xacc[mm], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int mm = 0; mm < MG; ++mm) xs_w[a * kMP + mm] = xacc[mm];
    }
    float vals[kVals];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if constexpr (MG >= 2) {
#pragma unroll
        for (int q = 0; q < MG / 2; ++q) {
          vals[g * MG + 2 * q] = lo_f(acc2[g][q]);
          vals[g * MG + 2 * q + 1] = hi_f(acc2[g][q]);
        }
      } else {
        vals[g] = acc1[g];
      }
    }
    warp_reduce_scatter<kVals>(vals, lane);
    __syncwarp();
    constexpr int kOut = (kVals >= 32) ? kVals / 32 : 1;
#pragma unroll
    for (int jj = 0; jj < kOut; ++jj) {
      const int e = reduce_out_index<kVals>(lane, jj);
      const int g = e / MG, mm = e % MG;
      const int m = mg * MG + mm, i = rg * 8 + g;
      if (m < mcnt && i < nr)
        p.zpart[(static_cast<size_t>(c) * p.M + m) * p.rpad + i_lo + i] = xs_w[a * kMP + mm] - 2.0f * vals[jj];
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------------ small-batch fast path

// V side for M <= 8 with lanes over ranks: lane l < nrg takes rank g0 + l of the
// staged rows, lane 31 sums x itself (an all-ones sign word), warp a takes word a
// of the chunk.  out[m * 64 + i] = sum of the x whose sign is -1 (i < nr),
// xs[m] = sum of x over the chunk.  Whole group.
template <int MG>
__device__ __forceinline__ void vside_lane_rank(const uint16_t* xc, const uint32_t* vrows, int mcnt, int nr,
                                                int nw, float* part, float* out, float* xs, int a, int lane,
                                                int tid) {
  for (int g0 = 0; g0 < nr; g0 += 31) {
    const int nrg = min(31, nr - g0);
    float acc[MG];
#pragma unroll
    for (int mm = 0; mm < MG; ++mm) acc[mm] = 0.0f;
    if (a < nw) {
      const uint32_t word = (lane < nrg) ? vrows[(g0 + lane) * kXWords + a] : (lane == 31 ? 0xFFFFFFFFu : 0u);
      const uint16_t* xr = xc + a * 32;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const uint32_t flag = word & (1u << j);
#pragma unroll
        for (int mm = 0; mm < MG; ++mm) padd1(acc[mm], bf16_bits_to_f32(xr[mm * kSubK + j]), flag);
      }
    }
#pragma unroll
    for (int mm = 0; mm < MG; ++mm) part[(a * 32 + lane) * MG + mm] = acc[mm];
    named_barrier(kBarAlu, kAluThreads);
    if (tid < 32 * MG) {
      const int l = tid / MG, mm = tid % MG;
      float sum = 0.0f;
#pragma unroll
      for (int w = 0; w < kAluWarps; ++w) sum += part[(w * 32 + l) * MG + mm];
      if (mm < mcnt) {
        if (l < nrg) out[mm * 64 + g0 + l] = sum;
        else if (l == 31 && g0 == 0) xs[mm] = sum;
      }
    }
    named_barrier(kBarAlu, kAluThreads);
  }
}

// ------------------------------------------------------------------ local z (mode 2)

// out[m * kVRanks + i] = sum over ALL of K of the x[m0+m][k] whose sign V[k][i0+i]
// is -1 (i < nr <= 16), and xs_s[m] = sum_k x[m0+m][k].  Whole group.
template <int MG>
__device__ __forceinline__ void vside_full_k(const FusedParams& p, int m0, int mcnt, int i0, int nr, uint16_t* xb,
                             uint32_t* vb, float* red_s, float* xs_s, float* out, int a, int lane,
                             int tid) {
  constexpr int kPairs = (MG >= 2) ? MG / 2 : 1;
  const int mgc = (mcnt + MG - 1) / MG;
  const int groups = 2 * mgc;
  int KS = kAluWarps / groups;
  if (KS < 1) KS = 1;
  const int tasks = groups * KS;
  const bool active = a < tasks;
  const int ks = a % KS, rest = a / KS, mg = rest % mgc, rg = rest / mgc;
  uint64_t acc2[8][kPairs];
  float acc1[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    acc1[g] = 0.0f;
#pragma unroll
    for (int q = 0; q < kPairs; ++q) acc2[g][q] = 0ull;
  }
  float xrun = 0.0f;                                 // this thread's share of sum_k x
  const int nsb = (p.KW + kXWords - 1) / kXWords;
  stage_x(p, m0, mcnt, 0, min(kXWords, p.KW), xb, tid);
  stage_v(p, i0, nr, 0, min(kXWords, p.KW), vb, tid);
  cp_async_commit();
  for (int j = 0; j < nsb; ++j) {
    const int ws = j * kXWords, nw = min(kXWords, p.KW - ws);
    const uint16_t* xcur = xb + (j & 1) * kMP * kSubK;
    const uint32_t* vcur = vb + (j & 1) * kVRanks * kXWords;
    if (j + 1 < nsb) {
      const int ws2 = ws + kXWords, nw2 = min(kXWords, p.KW - ws2);
      stage_x(p, m0, mcnt, ws2, nw2, xb + ((j + 1) & 1) * kMP * kSubK, tid);
      stage_v(p, i0, nr, ws2, nw2, vb + ((j + 1) & 1) * kVRanks * kXWords, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    named_barrier(kBarAlu, kAluThreads);
    if (active) {
      const int wa = (ks * kXWords) / KS, wb = min(nw, ((ks + 1) * kXWords) / KS);
      vside_task_accumulate<MG>(xcur, vcur, rg, mg, wa, wb, lane, acc2, acc1);
    }
    // thread tid owns row tid / 8 and every 8th element of it for the x sum
    {
      const int m = tid >> 3, part = tid & 7;
      if (m < mcnt)
        for (int k = part; k < nw * 32; k += 8) xrun += bf16_bits_to_f32(xcur[m * kSubK + k]);
    }
    named_barrier(kBarAlu, kAluThreads);
  }
  vside_task_finish<MG>(acc2, acc1, red_s + a * 64, active, lane);
  xrun += __shfl_xor_sync(0xffffffffu, xrun, 4);
  xrun += __shfl_xor_sync(0xffffffffu, xrun, 2);
  xrun += __shfl_xor_sync(0xffffffffu, xrun, 1);
  if ((tid & 7) == 0) xs_s[tid >> 3] = xrun;
  named_barrier(kBarAlu, kAluThreads);
  for (int idx = tid; idx < kMP * kRB; idx += kAluThreads) {
    const int m = idx / kRB, i = idx % kRB;
    float s = 0.0f;
    if (m < mcnt) {
      const int mgi = m / MG, mm = m % MG, rgi = i / 8, gg = i % 8;
      const int task0 = (rgi * mgc + mgi) * KS;
      for (int k2 = 0; k2 < KS; ++k2) s += red_s[(task0 + k2) * 64 + gg * MG + mm];
    }
    out[m * kVRanks + i] = s;
  }
  named_barrier(kBarAlu, kAluThreads);
}


// ------------------------------------------------------------------ U side

struct AluBufs {
  uint16_t* xb;
  uint32_t* vb;
  float* z_s;
  float* zb_s;
  float* corr_s;
  float* red_s;
  float* vout;
  float* xsw;
  float* xs_s;
};

// corr[rs][m][row] for the 128 rows of tile t, rows m0 .. m0+mcnt of the batch and
// the ranks of rank blocks [b_lo, b_hi).  Task a: rows 32 (a & 3) + lane; (a >> 2)
// picks the upper/lower 16 batch rows (mcnt > 16) or the rank-block parity (else).
template <int MG, int MGV>
__device__ __forceinline__ void uside_pass(const FusedParams& p, int t, int b_lo, int b_hi, int m0, int mcnt,
                           const AluBufs& B, int a, int lane, int tid) {
  constexpr int kPairs = (MG >= 2) ? MG / 2 : 1;
  const int RS = (mcnt > 16) ? 1 : 2;
  const int rs = (RS == 2) ? (a >> 2) : 0;
  const int mbase = (RS == 1) ? (a >> 2) * 16 : 0;
  const int mwidth = (RS == 1) ? 16 : MG;
  const int row = (a & 3) * 32 + lane;
  const uint32_t* urow = p.Ubits + static_cast<size_t>(t * kTileRows + row) * p.RW;
  const int IBn = (p.r + kRB - 1) / kRB;
  uint64_t acc2[kPairs];
#pragma unroll
  for (int j = 0; j < kPairs; ++j) acc2[j] = 0ull;
  float acc1 = 0.0f;
  float zsum[MG];
#pragma unroll
  for (int j = 0; j < MG; ++j) zsum[j] = 0.0f;

  // chunks of 8 rank blocks starting on an even block (whole 32-bit sign words)
  for (int c0 = b_lo & ~1; c0 < b_hi; c0 += kZChunkBlocks) {
    const int nblk = min(kZChunkBlocks, IBn - c0);
    uint32_t uw[kZChunkBlocks / 2];
#pragma unroll
    for (int q = 0; q < kZChunkBlocks / 2; ++q)
      uw[q] = (2 * q < nblk && c0 + 2 * q < b_hi) ? __ldg(urow + (c0 >> 1) + q) : 0u;
    named_barrier(kBarAlu, kAluThreads);            // previous chunk consumed
    if (p.mode == BILOCO_MODE_SHARED_Z) {
      const int nr = nblk * kRB;
      const int r_lo = max(c0, b_lo) * kRB, r_hi = min(min(c0 + nblk, b_hi) * kRB, p.r);
      const int nv = max(0, r_hi - r_lo);                 // ranks of this chunk in the share
      if (p.zdirect) {
        // every chunk partial of every needed (m, rank), copied asynchronously in one
        // round (mcnt * KC <= 64, nv <= 128), then summed in chunk order
        float* zst = B.corr_s;
        const int i = tid & 127;
        if (i < nv) {
          const size_t stride = static_cast<size_t>(p.M) * p.rpad;
          const float* src = p.zpart + static_cast<size_t>(m0) * p.rpad + r_lo + i;
          for (int cc = tid >> 7; cc < p.KC; cc += 2)
            for (int m = 0; m < mcnt; ++m)
              cp_async4(smem_u32(zst + (cc * mcnt + m) * nv + i), src + cc * stride + static_cast<size_t>(m) * p.rpad);
        }
        cp_async_commit();
        cp_async_wait<0>();
        named_barrier(kBarAlu, kAluThreads);
        for (int m = tid >> 7; m < kMP; m += 2) {
          const int rank = c0 * kRB + i;
          float v = 0.0f;
          if (i < nr && m < mcnt && rank >= r_lo && rank < r_hi) {
            float sum = 0.0f;
            for (int cc = 0; cc < p.KC; ++cc) sum += zst[(cc * mcnt + m) * nv + rank - r_lo];
            v = __fmul_rn(__ldg(p.alpha + rank), sum);
          }
          if (i < nr) B.z_s[i * kMpad + m] = v;
        }
      } else {
        const int i = tid & 127;
        for (int m = tid >> 7; m < kMP; m += 2) {
          const int rank = c0 * kRB + i;
          float v = 0.0f;
          if (i < nr && m < mcnt && rank >= r_lo && rank < r_hi)
            v = __ldcg(p.zfin + static_cast<size_t>(m0 + m) * p.rpad + rank);
          if (i < nr) B.z_s[i * kMpad + m] = v;
        }
      }
    } else {
      // local z: each needed rank block over the whole K, computed right here
      for (int bl = 0; bl < nblk; ++bl) {
        const int blk = c0 + bl;
        if (blk < b_lo || blk >= b_hi) continue;      // uniform over the group
        const int i0 = blk * kRB, nr = min(kRB, p.r - i0);
        vside_full_k<MGV>(p, m0, mcnt, i0, nr, B.xb, B.vb, B.red_s, B.xs_s, B.vout, a, lane, tid);
        for (int idx = tid; idx < kMP * kRB; idx += kAluThreads) {
          const int m = idx / kRB, i = idx % kRB;
          float z = 0.0f;
          if (m < mcnt && i < nr)
            z = __fmul_rn(__ldg(p.alpha + i0 + i), B.xs_s[m] - 2.0f * B.vout[m * kVRanks + i]);
          B.z_s[(bl * kRB + i) * kMpad + m] = z;
        }
        named_barrier(kBarAlu, kAluThreads);
      }
    }
    named_barrier(kBarAlu, kAluThreads);
    // block sums of the staged z, then the sign accumulation
    for (int idx = tid; idx < nblk * kMP; idx += kAluThreads) {
      const int bl = idx / kMP, m = idx % kMP;
      float s = 0.0f;
#pragma unroll
      for (int i = 0; i < kRB; ++i) s += B.z_s[(bl * kRB + i) * kMpad + m];
      B.zb_s[bl * kMP + m] = s;
    }
    named_barrier(kBarAlu, kAluThreads);
#pragma unroll
    for (int bl = 0; bl < kZChunkBlocks; ++bl) {
      const int blk = c0 + bl;
      if (bl >= nblk || blk < b_lo || blk >= b_hi) continue;
      if (RS == 2 && (blk & 1) != rs) continue;
      const uint32_t word = uw[bl >> 1] >> ((bl & 1) * 16);
      const float* zr = B.z_s + (bl * kRB) * kMpad + mbase;
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
#pragma unroll
      for (int j = 0; j < MG; ++j)
        if (j < mwidth) zsum[j] += B.zb_s[bl * kMP + mbase + j];
    }
  }
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
      B.corr_s[(rs * kMP + m) * kTileRows + row] = zsum[j] - 2.0f * accf[j];
      if (RS == 1) B.corr_s[(1 * kMP + m) * kTileRows + row] = 0.0f;
    }
  }
}


// Warm L2 with the sign rows of U this CTA's U side will read.
__device__ __forceinline__ void prefetch_u_rows(const FusedParams& p, int u0, int u1, int tid) {
  const int t_first = u0 / p.KC, t_last = (u1 - 1) / p.KC;
  for (int t = t_first; t <= t_last && t < t_first + 2; ++t) {
    int b_lo, b_hi;
    rank_share(p, max(u0, t * p.KC) - t * p.KC, min(u1, (t + 1) * p.KC) - t * p.KC, b_lo, b_hi);
    if (b_hi <= b_lo) continue;
    const int wlo = b_lo / 2, whi = (b_hi + 1) / 2;
    for (int row = tid; row < kTileRows; row += kAluThreads)
      for (int w = wlo; w < whi; w += 32)
        prefetch_l2(p.Ubits + static_cast<size_t>(t * kTileRows + row) * p.RW + w);
  }
}

// ------------------------------------------------------------------ the kernel

template <int BN, int ST, int MC>
__global__ void __launch_bounds__(kThreads, 1)
fused_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
             const __grid_constant__ CUtensorMap tmap_xs, const __grid_constant__ CUtensorMap tmap_v,
             const __grid_constant__ FusedParams p) {
  using L = Layout<BN, ST>;
  constexpr int MGV = (MC < 8) ? MC : 8;       // V side: batch rows per task
  constexpr int MGU = (MC < 16) ? MC : 16;     // U side: batch rows per task
  constexpr int XV = (MC < 32) ? MC : 32;      // x sums: rows per warp reduction
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
  auto xfull_bar = [&](int s) { return smem_u32(&bars[2 * ST + 7 + s]); };
  const uint32_t done_bar = smem_u32(&bars[3 * ST + 7]);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* epi_last = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);
  volatile int* alu_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 20);
  const Ctl ctl{abort_flag, p.status};

  const int g = blockIdx.x;
  const int u0 = first_unit(g, p.G, p.U), u1 = first_unit(g + 1, p.G, p.U);
  const int t_first = u0 / p.KC, t_last = (u1 - 1) / p.KC;
  const int nseg = t_last - t_first + 1;
  const int nunits = u1 - u0;
  const int npass = (p.M + kMP - 1) / kMP;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_w);
    if (!p.inq) prefetch_tmap(&tmap_x);
    if (p.fast) {
      prefetch_tmap(&tmap_xs);
      if (p.r > 0) prefetch_tmap(&tmap_v);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(full_bar(s), p.inq ? 2 : 1);     // + the quantiser's arrival when in-kernel
      mbar_init(empty_bar(s), p.fast ? 2 : 1);   // + the CUDA cores releasing the staged x
      mbar_init(xfull_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), kEpiThreads);
    }
    mbar_init(corrf_bar, kAluThreads);
    mbar_init(corre_bar, kEpiThreads);
    mbar_init(drain_bar, 1);
    mbar_init(done_bar, kWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Programmatic dependent launch.  The next kernel on the stream may start
  // taking SMs as soon as this one's CTAs leave them.  This kernel, in turn,
  // waits for the kernel before it only where that kernel's results or this
  // call's scratch are touched: every warp but the producer waits here, and the
  // producer first requests the weight bytes of its first stages (no kernel of
  // this library writes the weight operand).
  if (threadIdx.x == 0) griddep_launch_dependents();
  if (warp >= 2) griddep_wait();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const int pre = min(ST, nunits);
      const uint32_t stage_bytes = kUnitBytesA + kSfBytes + (p.inq ? 0u : BN * 128 + kSfBytes);
      const bool vstage = p.fast && p.r > 0 && p.mode == BILOCO_MODE_SHARED_Z;
      const uint32_t xstage_bytes = static_cast<uint32_t>(p.bxr * kSubK * 2) + (vstage ? L::kVBytes : 0u);
      auto issue_x = [&](int k, int s) {
        const int u = u0 + k, t = u / p.KC, c = u % p.KC;
        mbar_arrive_expect_tx(xfull_bar(s), xstage_bytes);
        tma_load_2d(smem_u32(smem + L::kXS + s * L::kXStride), &tmap_xs, xfull_bar(s), c * kSubK, 0);
        if (vstage) {
          int i_lo, i_hi;
          vside_ranks(p, t, i_lo, i_hi);
          tma_load_2d(smem_u32(smem + L::kXS + s * L::kXStride + L::kXBytes), &tmap_v, xfull_bar(s),
                      c * kXWords, i_lo);
        }
      };
      // the weight bytes of the first stages before waiting for the previous
      // kernel, then the activation (and V rows) those stages need
      for (int k = 0; k < pre; ++k) {
        const int u = u0 + k, t = u / p.KC, c = u % p.KC;
        mbar_arrive_expect_tx(full_bar(k), stage_bytes);
        tma_load_2d(smem_u32(smem + L::kA + k * kUnitBytesA), &tmap_w, full_bar(k), c * 128,
                    t * kTileRows);
        bulk_load(smem_u32(smem + L::kSFA + k * kSfBytes),
                  p.w_sf + (static_cast<size_t>(t) * p.KC + c) * kSfBytes, kSfBytes, full_bar(k));
      }
      griddep_wait();
      if (p.fast)
        for (int k = 0; k < pre; ++k) issue_x(k, k);
      if (!p.inq) {
        for (int k = 0; k < pre; ++k) {
          const int c = (u0 + k) % p.KC;
          tma_load_2d(smem_u32(smem + L::kB + k * BN * 128), &tmap_x, full_bar(k), c * 128, 0);
          bulk_load(smem_u32(smem + L::kSFB + k * kSfBytes), p.x_sf + static_cast<size_t>(c) * kSfBytes,
                    kSfBytes, full_bar(k));
        }
      }
      int issued = pre;
      for (int k = pre; k < nunits; ++k) {
        const int s = k % ST;
        if (!mbar_wait(empty_bar(s), ((k / ST) - 1) & 1, abort_flag)) {
          fail(ctl);
          break;
        }
        const int u = u0 + k, t = u / p.KC, c = u % p.KC;
        if (p.fast) issue_x(k, s);
        mbar_arrive_expect_tx(full_bar(s), stage_bytes);
        tma_load_2d(smem_u32(smem + L::kA + s * kUnitBytesA), &tmap_w, full_bar(s), c * 128,
                    t * kTileRows);
        bulk_load(smem_u32(smem + L::kSFA + s * kSfBytes),
                  p.w_sf + (static_cast<size_t>(t) * p.KC + c) * kSfBytes, kSfBytes, full_bar(s));
        if (!p.inq) {
          tma_load_2d(smem_u32(smem + L::kB + s * BN * 128), &tmap_x, full_bar(s), c * 128, 0);
          bulk_load(smem_u32(smem + L::kSFB + s * kSfBytes), p.x_sf + static_cast<size_t>(c) * kSfBytes,
                    kSfBytes, full_bar(s));
        }
        ++issued;
      }
      // never leave the CTA with copies in flight: wait for the last fills
      for (int k = max(0, issued - ST); k < issued; ++k) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(full_bar(k % ST), (k / ST) & 1) ||
               (p.fast && !mbar_try_wait(xfull_bar(k % ST), (k / ST) & 1))) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(p.status, kDevErrTimeout);
            break;
          }
        }
      }
    }
    __syncwarp();
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
            tc_cp_32x128b_warpx4(sfa_t + 4 * j, make_sdesc(sfa_s + 512 * j, 0, 128, 0));
            tc_cp_32x128b_warpx4(sfb_t + 4 * j, make_sdesc(sfb_s + 512 * j, 0, 128, 0));
          }
          const SmemDesc adesc = make_sdesc(smem_u32(smem + L::kA + s * kUnitBytesA), 16, 1024, 2);
          const SmemDesc bdesc = make_sdesc(smem_u32(smem + L::kB + s * BN * 128), 16, 1024, 2);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tc_mma_nvf4(d_tmem, sdesc_at(adesc, 2 * j), sdesc_at(bdesc, 2 * j), idesc, sfa_t + 4 * j, sfb_t + 4 * j,
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
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                            // TMEM lane quarter of this warp
    const int row = q * 32 + lane;                     // weight row within the tile
    const float gs = __ldg(p.gscale);
    int corr_round = 0;
    for (int seg = 0; seg < nseg; ++seg) {
      const int t = t_first + seg;
      const int b = seg & 1;
      const int hf = owner_cta(static_cast<uint32_t>(t * p.KC), p.G, p.U);
      const int hl = owner_cta(static_cast<uint32_t>((t + 1) * p.KC - 1), p.G, p.U);
      const bool sole = hf == hl;
      const int which = (t == t_first) ? 0 : 1;
      float* my_slot = p.slots + static_cast<size_t>(2 * g + which) * BN * kTileRows;
      if (!group_wait(accf_bar(b), (seg >> 1) & 1, kBarEpi, kEpiThreads, ctl)) break;
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
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(raw[j]);
          if (BN >= 32) {
            tmem_ld16(taddr + 16, raw);
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
          if (!group_wait(corrf_bar, corr_round & 1, kBarEpi, kEpiThreads, ctl)) {
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
            if (j < mcnt)
              yb[static_cast<size_t>(m0 + j) * p.N] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
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
        // publish this partial; the last contributor of the tile sums all of them
        __threadfence();
        named_barrier(kBarEpi, kEpiThreads);
        if (warp == kEpiWarp0) {
          if (lane == 0) {
            const uint32_t contributors = static_cast<uint32_t>(hl - hf + 1);
            const uint32_t old = atomicAdd(p.tickets + t, 1u);
            const bool last = (old == contributors - 1);
            if (last) atomicExch(p.tickets + t, 0u);
            __threadfence();
            *epi_last = last ? 1 : 0;
          }
          __syncwarp();
        }
        named_barrier(kBarEpi, kEpiThreads);
        const bool last = *epi_last != 0;
        named_barrier(kBarEpi, kEpiThreads);
        if (last) {
          // this row's partials of every contributor in rounds of 32 independent
          // loads, each batch row summed in contributor order
          const int nh = hl - hf + 1;
          // every contributor after the first starts its range inside tile t, so only
          // the first one may hold this tile in its second slot
          const int wh_first = (t == first_unit(hf, p.G, p.U) / p.KC) ? 0 : 1;
          auto slot_of = [&](int h) { return 2 * h + ((h == hf) ? wh_first : 0); };
          if (nh <= 32) {
            const int rows_per_round = 32 / nh;
            for (int m0 = 0; m0 < p.M; m0 += rows_per_round) {
              const int mrows = min(p.M - m0, rows_per_round);
              float part[32];
              {
                int e = 0, mm = 0;
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                  part[q] = 0.0f;
                  if (mm < mrows) {
                    part[q] = __ldcg(p.slots + (static_cast<size_t>(slot_of(hf + e)) * BN + m0 + mm) * kTileRows + row);
                  }
                  if (++e == nh) { e = 0; ++mm; }
                }
              }
              int e = 0, mm = 0;
              float sum = 0.0f;
#pragma unroll
              for (int q = 0; q < 32; ++q) {
                if (mm < mrows) {
                  sum += part[q];
                  if (e == nh - 1) {
                    p.y[static_cast<size_t>(m0 + mm) * p.N + static_cast<size_t>(t) * kTileRows + row] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(sum));
                    sum = 0.0f;
                  }
                }
                if (++e == nh) { e = 0; ++mm; }
              }
            }
          } else {
            for (int m = 0; m < p.M; ++m) {
              float tot = 0.0f;
              for (int h0 = hf; h0 <= hl; h0 += 32) {
                float part[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                  part[q] = 0.0f;
                  const int h = h0 + q;
                  if (h <= hl)
                    part[q] = __ldcg(p.slots + (static_cast<size_t>(slot_of(h)) * BN + m) * kTileRows + row);
                }
#pragma unroll
                for (int q = 0; q < 32; ++q) tot += part[q];
              }
              p.y[static_cast<size_t>(m) * p.N + static_cast<size_t>(t) * kTileRows + row] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(tot));
            }
          }
        }
      }
    }
  } else if (warp >= kAluWarp0 && warp < kAluWarp0 + kAluWarps && (p.r > 0 || p.inq)) {
    // ---------------------------------------------------------------- CUDA-core work
    const int tid = threadIdx.x - kAluWarp0 * 32;   // 0..255
    const int a = warp - kAluWarp0;                  // task slot 0..7
    AluBufs B;
    B.xb = reinterpret_cast<uint16_t*>(smem + L::kXB);
    B.vb = reinterpret_cast<uint32_t*>(smem + L::kVB);
    B.z_s = reinterpret_cast<float*>(smem + L::kZS);
    B.zb_s = reinterpret_cast<float*>(smem + L::kZB);
    B.corr_s = reinterpret_cast<float*>(smem + L::kCorr);
    B.red_s = reinterpret_cast<float*>(smem + L::kRed);
    B.vout = reinterpret_cast<float*>(smem + L::kVOut);
    B.xsw = reinterpret_cast<float*>(smem + L::kXsw);
    B.xs_s = reinterpret_cast<float*>(smem + L::kXsum);
    const bool shared_z = p.r > 0 && p.mode == BILOCO_MODE_SHARED_Z;
    bool ok = true;

    if (p.r > 0) prefetch_u_rows(p, u0, u1, tid);
    if (p.inq) {
      // B tile rows >= M and unused scale bytes stay zero for the whole launch
      constexpr int kPer = (BN * 128 + kSfBytes) / 16;
      for (int idx = tid; idx < ST * kPer; idx += kAluThreads) {
        const int s = idx / kPer, o = idx % kPer;
        uint4* dst = (o < BN * 8) ? reinterpret_cast<uint4*>(smem + L::kB + s * BN * 128) + o
                                  : reinterpret_cast<uint4*>(smem + L::kSFB + s * kSfBytes) + (o - BN * 8);
        *dst = make_uint4(0u, 0u, 0u, 0u);
      }
    }

    if (p.fast) {
      // ---- on the x chunks and V rows the producer staged, a batch of up to ST
      // units at a time (one per stage): quantise all of them (small M), release
      // them to the MMA, then the V side of each, then free the stages.
      for (int k0 = 0; k0 < nunits && ok; k0 += ST) {
        const int nb = min(ST, nunits - k0);
        for (int j = 0; j < nb && ok; ++j) {
          const int k = k0 + j;
          if (!group_wait(xfull_bar(k % ST), (k / ST) & 1, kBarAlu, kAluThreads, ctl)) ok = false;
        }
        if (!ok) break;
        const int mcnt = p.M;                          // fast path: M <= 32, one pass
        if (p.inq) {
          // one thread per element pair; the 8 pairs of a 16-element block sit in 8
          // consecutive lanes (block max by shuffles)
          const int per_unit = mcnt * 128;
          for (int idx = tid; idx < nb * per_unit; idx += kAluThreads) {
            const int j = idx / per_unit, rem = idx % per_unit, m = rem >> 7, pr = rem & 127;
            const int k = k0 + j, s = k % ST, c = (u0 + k) % p.KC;
            const int nw = min(kXWords, p.KW - c * kXWords);
            const uint32_t w2 = *reinterpret_cast<const uint32_t*>(smem + L::kXS + s * L::kXStride +
                                                                   m * (kSubK * 2) + pr * 4);
            const float v0 = bf16_bits_to_f32(w2 & 0xFFFFu), v1 = bf16_bits_to_f32(w2 >> 16);
            float amax = fmaxf(fabsf(v0), fabsf(v1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
            const uint32_t sb = e4m3_from_f32(__fdiv_rn(amax, 6.0f));
            const float S = e4m3_to_f32(sb);
            const E2M1Thresholds th = e2m1_thresholds(S);
            const uint32_t byte = e2m1_code_bf16(v0, th, S == 0.0f) | (e2m1_code_bf16(v1, th, S == 0.0f) << 4);
            if (pr < nw * 16) {
              smem[L::kB + s * BN * 128 + m * 128 + ((((pr >> 4) ^ (m & 7)) << 4) | (pr & 15))] =
                  static_cast<uint8_t>(byte);
              if ((pr & 7) == 0)
                smem[L::kSFB + s * kSfBytes + (pr >> 5) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 +
                     ((pr >> 3) & 3)] = static_cast<uint8_t>(sb);
            }
          }
          fence_proxy_async_smem();
          named_barrier(kBarAlu, kAluThreads);
          if (a == 0) {
            if (lane < nb) mbar_arrive(full_bar((k0 + lane) % ST));
            __syncwarp();
          }
        }
        if (shared_z) {
          const int rgu = (p.r + p.T - 1) / p.T / 8 + 1;         // rank groups of 8 per unit (upper bound)
          auto info = [&](int j, const uint16_t*& xc, const uint32_t*& vrows, int& c, int& i_lo, int& nr,
                          int& nw) {
            const int k = k0 + j, u = u0 + k, t = u / p.KC, s = k % ST;
            c = u % p.KC;
            nw = min(kXWords, p.KW - c * kXWords);
            xc = reinterpret_cast<const uint16_t*>(smem + L::kXS + s * L::kXStride);
            vrows = reinterpret_cast<const uint32_t*>(smem + L::kXS + s * L::kXStride + L::kXBytes);
            int i_hi;
            vside_ranks(p, t, i_lo, i_hi);
            nr = i_hi - i_lo;
          };
          vside_batch<MGV>(p, nb, mcnt, rgu, info, B.xsw, a, lane);
        }
        named_barrier(kBarAlu, kAluThreads);           // every read of the batch's slots is done
        if (a == 0) {
          if (lane < nb) mbar_arrive(empty_bar((k0 + lane) % ST));
          __syncwarp();
        }
      }
    } else if (p.unit_alu) {
      // ---- per unit: stage the chunk, quantise it (small M), V side (shared z).
      // A job is (unit, batch pass, V rank sub-range); the next job is prefetched.
      auto nsub_of = [&](int t) {
        if (!shared_z) return 1;
        int i_lo, i_hi;
        vside_ranks(p, t, i_lo, i_hi);
        return max(1, (i_hi - i_lo + kVRanks - 1) / kVRanks);
      };
      auto stage_job = [&](int k, int jk, int buf) {
        const int u = u0 + k, t = u / p.KC, c = u % p.KC;
        const int nw = min(kXWords, p.KW - c * kXWords);
        const int nsub = nsub_of(t);
        const int pass = jk / nsub, sub = jk % nsub;
        const int m0 = pass * kMP, mcnt = min(kMP, p.M - m0);
        stage_x(p, m0, mcnt, c * kXWords, nw, B.xb + buf * kMP * kSubK, tid);
        if (shared_z) {
          int i_lo, i_hi;
          vside_ranks(p, t, i_lo, i_hi);
          const int r0 = i_lo + sub * kVRanks, nr = min(kVRanks, i_hi - r0);
          if (nr > 0) stage_v(p, r0, nr, c * kXWords, nw, B.vb + buf * kVRanks * kXWords, tid);
        }
      };
      int buf = 0;
      stage_job(0, 0, 0);
      cp_async_commit();
      for (int k = 0; k < nunits && ok; ++k) {
        const int u = u0 + k, t = u / p.KC, c = u % p.KC, s = k % ST;
        const int nw = min(kXWords, p.KW - c * kXWords);
        const int nsub = nsub_of(t);
        const int njobs = npass * nsub;
        int i_lo = 0, i_hi = 0;
        if (shared_z) vside_ranks(p, t, i_lo, i_hi);
        for (int jk = 0; jk < njobs && ok; ++jk) {
          const bool more = (jk + 1 < njobs) || (k + 1 < nunits);
          if (more) {
            if (jk + 1 < njobs) stage_job(k, jk + 1, buf ^ 1);
            else stage_job(k + 1, 0, buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
          } else {
            cp_async_wait<0>();
          }
          named_barrier(kBarAlu, kAluThreads);
          const uint16_t* xcur = B.xb + buf * kMP * kSubK;
          const int pass = jk / nsub, sub = jk % nsub;
          const int m0 = pass * kMP, mcnt = min(kMP, p.M - m0);
          if (p.inq && jk == 0) {
            // the stage must be free before its B tile is rewritten
            if (k >= ST && !group_wait(empty_bar(s), ((k / ST) - 1) & 1, kBarAlu, kAluThreads, ctl)) {
              ok = false;
              break;
            }
            quant_chunk(xcur, mcnt, nw, smem + L::kB + s * BN * 128, smem + L::kSFB + s * kSfBytes, tid);
            fence_proxy_async_smem();
            named_barrier(kBarAlu, kAluThreads);
            if (a == 0) {
              if (lane == 0) mbar_arrive(full_bar(s));
              __syncwarp();
            }
          }
          if (shared_z) {
            const int r0 = i_lo + sub * kVRanks, nr = min(kVRanks, i_hi - r0);
            if (sub == 0) chunk_xsum<XV>(xcur, mcnt, nw, B.xsw, B.xs_s, a, lane, tid);
            if (nr > 0) {
              vside_chunk<MGV>(xcur, B.vb + buf * kVRanks * kXWords, mcnt, nr, nw, B.red_s, B.vout, a, lane,
                               tid);
              for (int idx = tid; idx < mcnt * nr; idx += kAluThreads) {
                const int m = idx / nr, i = idx % nr;
                p.zpart[(static_cast<size_t>(c) * p.M + m0 + m) * p.rpad + r0 + i] =
                    B.xs_s[m] - 2.0f * B.vout[m * kVRanks + i];
              }
            }
          }
          named_barrier(kBarAlu, kAluThreads);     // buffer `buf` may be refilled
          buf ^= 1;
        }
      }
      if (!ok) cp_async_wait<0>();
    }

    if (shared_z && ok) {
      // ---- publish the chunk partials; finalise (larger M) or count in (direct)
      __threadfence();
      named_barrier(kBarAlu, kAluThreads);
      if (p.zdirect) {
        if (a == 0) {
          if (lane == 0) atomicAdd(p.z_ready, 1u);
          __syncwarp();
        }
      } else {
        for (int seg = 0; seg < nseg; ++seg) {
          const int t = t_first + seg;
          if (a == 0) {
            if (lane == 0) {
              const int hf = owner_cta(static_cast<uint32_t>(t * p.KC), p.G, p.U);
              const int hl = owner_cta(static_cast<uint32_t>((t + 1) * p.KC - 1), p.G, p.U);
              const uint32_t old = atomicAdd(p.vtick + t, 1u);
              const bool last = old == static_cast<uint32_t>(hl - hf);
              if (last) atomicExch(p.vtick + t, 0u);
              __threadfence();
              *alu_flag = last ? 1 : 0;
            }
            __syncwarp();
          }
          named_barrier(kBarAlu, kAluThreads);
          const bool last = *alu_flag != 0;
          named_barrier(kBarAlu, kAluThreads);
          if (last) {
            int i_lo, i_hi;
            vside_ranks(p, t, i_lo, i_hi);
            const int nr = i_hi - i_lo;
            const int per_c = p.M * nr;                     // values per chunk partial
            const size_t stride = static_cast<size_t>(p.M) * p.rpad;
            float* acc_s = B.corr_s;                        // running sums [M][nr]
            float* stg = B.corr_s + 4096;                   // one round of partials
            const int cpr = max(1, 4096 / max(per_c, 1));   // chunks per round
            for (int idx = tid; idx < per_c; idx += kAluThreads) acc_s[idx] = 0.0f;
            for (int c0r = 0; c0r < p.KC; c0r += cpr) {
              const int ncr = min(cpr, p.KC - c0r);
              const int total = ncr * per_c;
              float tmp[16];
#pragma unroll
              for (int q = 0; q < 16; ++q) {
                const int idx = tid + q * kAluThreads;
                tmp[q] = 0.0f;
                if (idx < total) {
                  const int cc = idx / per_c, rem = idx % per_c, m = rem / nr, i = rem % nr;
                  tmp[q] = __ldcg(p.zpart + (c0r + cc) * stride + static_cast<size_t>(m) * p.rpad + i_lo + i);
                }
              }
#pragma unroll
              for (int q = 0; q < 16; ++q) {
                const int idx = tid + q * kAluThreads;
                if (idx < total) stg[idx] = tmp[q];
              }
              named_barrier(kBarAlu, kAluThreads);
              for (int idx = tid; idx < per_c; idx += kAluThreads) {
                float sum = acc_s[idx];
                for (int cc = 0; cc < ncr; ++cc) sum += stg[cc * per_c + idx];
                acc_s[idx] = sum;
              }
              named_barrier(kBarAlu, kAluThreads);
            }
            for (int idx = tid; idx < per_c; idx += kAluThreads) {
              const int m = idx / nr, i = i_lo + idx % nr;
              p.zfin[static_cast<size_t>(m) * p.rpad + i] = __fmul_rn(__ldg(p.alpha + i), acc_s[idx]);
            }
            __threadfence();
            named_barrier(kBarAlu, kAluThreads);
            if (a == 0) {
              if (lane == 0) atomicAdd(p.z_ready, 1u);
              __syncwarp();
            }
          }
        }
      }
      // wait until every partial (or every finished tile slice) is visible
      const uint32_t target = static_cast<uint32_t>(p.zdirect ? p.G : p.T);
      bool okw = true;
      if (a == 0) {
        if (lane == 0) okw = spin_until_geq(p.z_ready, target, ctl);
        okw = __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
        if (lane == 0 && okw) {
          const uint32_t old = atomicAdd(p.z_seen, 1u);
          if (old == static_cast<uint32_t>(p.G - 1)) {
            atomicExch(p.z_ready, 0u);
            atomicExch(p.z_seen, 0u);
          }
        }
        __syncwarp();
      }
      const bool any_fail = named_barrier_or(kBarAlu, kAluThreads, !okw);
      if (any_fail) fail(ctl);
      ok = !any_fail;
    }

    if (p.r > 0) {
      // ---- U side, one (segment, pass) at a time, handed to the epilogue via corr_s
      int corr_round = 0;
      for (int seg = 0; seg < nseg && ok; ++seg) {
        const int t = t_first + seg;
        int b_lo, b_hi;
        rank_share(p, max(u0, t * p.KC) - t * p.KC, min(u1, (t + 1) * p.KC) - t * p.KC, b_lo, b_hi);
        for (int pass = 0; pass < npass; ++pass) {
          const int m0 = pass * kMP, mcnt = min(kMP, p.M - m0);
          if (corr_round > 0 &&
              !group_wait(corre_bar, (corr_round - 1) & 1, kBarAlu, kAluThreads, ctl)) {
            ok = false;
            break;
          }
          uside_pass<MGU, MGV>(p, t, b_lo, b_hi, m0, mcnt, B, a, lane, tid);
          mbar_arrive(corrf_bar);
          ++corr_round;
        }
      }
      if (ok && corr_round > 0) group_wait(corre_bar, (corr_round - 1) & 1, kBarAlu, kAluThreads, ctl);
    }
  }

  // ------------------------------------------------------------------ teardown
  // Each warp reports once it no longer touches TMEM or the staging buffers;
  // warp 1 frees TMEM after all of them (bounded wait).
  __syncwarp();
  tc_fence_before();
  if (lane == 0) mbar_arrive(done_bar);
  if (warp == 1) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(done_bar, 0)) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        record_error(p.status, kDevErrTimeout);
        break;
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace
}  // namespace biloco

namespace biloco {

template <int BN, int ST, int MC>
cudaError_t launch_fused(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                         const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, const LaunchOpts& o) {
  static KernelSetup ks;
  return launch_resident(ks, fused_kernel<BN, ST, MC>, fp.G, kThreads, Layout<BN, ST>::kAlloc, s, o, tw, tx,
                         txs, tv, fp);
}

}  // namespace biloco
