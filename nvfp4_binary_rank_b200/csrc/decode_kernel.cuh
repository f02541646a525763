// Fused NVFP4 GEMM + binary-sign low-rank correction for batches of up to 128
// activation rows (decode and small prefill batches) on one B200 (sm_100a).
//
//   y[m, n] = g * sum_k FP4(x)[m, k] FP4(R)[n, k]  +  sum_i U[n, i] z[m, i],
//   z[m, i] = alpha_i * sum_k V[k, i] x[m, k]
//
// (BiLoCo README, section "Kernel": FP4 GEMM on the tensor cores, z = alpha.(V x)
// on the CUDA cores from bit-packed V, U z expanded before the BF16 store, one
// launch.)
//
// The weight is cut into units of 128 rows x 256 K elements, split over G <= #SMs
// CTAs in contiguous ranges (stream-K), exactly like the general kernel.  What
// differs is the order of the work after the wait on the previous kernel of the
// stream, which is what bounds a decode call:
//   * Weight stages are requested before that wait: no kernel of this library
//     writes the weight operand.
//   * Up to 16 rows the activation chunks of all the CTA's units land at once in
//     an operand cache in shared memory: below 8 rows quantised by the CTA itself,
//     from 8 rows up copied from an image the CTAs quantise once between them.
//     The MMAs read the activation from there, so the stage ring carries weight
//     bytes only.  The classes of 32, 64 and 128 rows (MMA N = 32, 64, 128) stream
//     each unit's activation chunk from that image with its weight stage.
//   * z is computed in rank slices: CTA g < Z computes z for the ranks
//     [g r / Z, (g + 1) r / Z) and publishes them behind one arrival counter
//     (Z = G - 2 on large grids, see shared_work_ctas).  This is the "side CTAs +
//     arrival flag" schedule of the README's mode table.  Below 8 rows the slice
//     is summed over the whole of K on the CUDA cores; from 8, V^T x runs on the
//     tensor cores in pieces of 128 ranks x a K slice whose partial sums the slice
//     owners add up.
//   * U z: from 4 rows up (tensor-core U side) every contributor of a weight tile
//     expands its share of U z for the tile (the 64-rank chunks in proportion to
//     its units of the tile) and adds it to the partial it publishes, so the
//     completing CTA (the sole owner, or the last split-K contributor to arrive)
//     only sums partials.  Below 4 rows the completing CTA alone expands U z for
//     the tile, in parallel with summing the partials, so the other CTAs publish
//     without waiting for z and exit early.
//
// Warp roles (14 warps): warp 0 TMA producer; warp 1 TMEM allocator and MMA
// issuer (tcgen05 kind::mxf4nvf4, block16); warps 2-5 epilogue (one weight row
// per thread); warps 6-13 CUDA cores (activation quantisation, V side, U side).
//
// Every wait is bounded.  On expiry the kernel records BILOCO_ERR_TIMEOUT in
// the status word, and the warps that share barriers leave together.
#pragma once

#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/biloco.h"
#include "decode_launch.h"
#include "decode_params.h"
#include "nvfp4_dev.cuh"
#include "ptx.cuh"
#include "sched.cuh"

namespace biloco {
namespace decode {

constexpr int kWarps = 14;
constexpr int kThreads = kWarps * 32;
constexpr int kEpiWarp0 = 2;
constexpr int kEpiThreads = 128;
constexpr int kAluWarp0 = 6;
constexpr int kAluWarps = 8;
constexpr int kAluThreads = kAluWarps * 32;
constexpr int kFinThreads = kEpiThreads + kAluThreads;
constexpr int kRowsMax = 128;             // activation rows handled (the largest class)
constexpr int kTileRows = 128;            // weight rows per tile = MMA M
constexpr int kUnitK = 256;               // K elements per unit
constexpr int kUnitBytesA = kTileRows * 128;
constexpr int kSfBytes = 2048;            // 4 scale atoms of 512 B per unit
constexpr int kMaxRanks = 1024;
constexpr int kTmemCols = 512;
constexpr int kVAtoms = 3;                // K atoms (64 elements) per V-side MMA batch
constexpr int kUChunk = 64;               // ranks per U-side MMA chunk (one 128-byte BF16 row)
constexpr int kUChunksMax = 16;           // r <= 1024
constexpr uint32_t kStageTx = kUnitBytesA + kSfBytes;

// named barriers (0 is __syncthreads)
constexpr int kBarAlu = 1;
constexpr int kBarEpi = 2;
constexpr int kBarFin = 3;                // epilogue + CUDA cores: finisher decision
constexpr int kBarFin2 = 4;               // epilogue + CUDA cores: correction ready
constexpr int kBarZ = 5;                  // epilogue + CUDA cores: z staged (1-2 rows)

// Per batch class (MC = most activation rows): weight stages and V-side ranks
// per pass (the larger classes trade stages for their z and register
// footprint).
template <int MC>
struct Cfg {
  // Up to 16 rows the activation chunks of all of a CTA's units sit in an operand
  // cache in shared memory (at most kMaxUnits units per CTA).  From 32 rows the
  // classes stream them instead: each stage carries one weight unit and the
  // matching activation chunk (codes and scale atoms) from the grid's activation
  // image, and both sets of block scales go to TMEM per stage.
  static constexpr bool kStream = MC > 16;
  static constexpr int kBN = kStream ? MC : 16;            // MMA N (activation rows, padded)
  static constexpr int kMaxUnits = kStream ? 64 : 16;      // units per CTA
  static constexpr int kStages = kStream ? (MC >= 128 ? 3 : 5) : ((MC >= 16) ? 4 : 6);
  static constexpr int kRankGroup = 4;                     // ranks per V-side pass
  // V-side load ring depth (blocks in flight per warp); below 8 rows a warp walks
  // only two or three K blocks
  static constexpr int kVStages = (MC >= 8) ? 3 : 2;
  // U side on the tensor cores from 4 rows up; below, per-thread sign-adds are
  // cheaper than the chunked MMA chain (measured on B200)
  static constexpr bool kTensorU = MC >= 4;
  // with the tensor-core U side every contributor of a tile adds its share of U z
  // to its partial; below, the completing CTA alone expands U z for the tile, so
  // the other CTAs exit early and free their SMs for the next kernel (each choice
  // measured faster on B200 for its classes)
  static constexpr bool kUShares = kTensorU;
  // from 8 rows up the CTAs quantise the activation once between them (a global
  // image behind an arrival counter) instead of each CTA quantising the chunks of
  // all its units
  static constexpr bool kGlobalQ = MC >= 8;
  // from 8 rows the V side runs on the tensor cores, cut into pieces of 128 ranks
  // x a slice of K, with the partial sums reduced across CTAs (at 8 rows 13-22%
  // faster than the CUDA-core loop, measured on B200; below 8 that loop stays)
  static constexpr bool kTensorV = MC >= 8;
  // The U side's product: up to 32 rows the high and low BF16 parts of z go to
  // separate TMEM columns (one MMA of N = 2 MC per K step, added by the epilogue);
  // from 64 rows both parts accumulate into the same MC columns (two MMAs of N = MC),
  // which halves the product's tensor memory.  The 128-row class keeps one product
  // buffer (its accumulators take half of TMEM), the others two.
  static constexpr bool kUSum = MC >= 64;
  static constexpr int kUBufs = MC >= 128 ? 1 : 2;
  // z tiles of the tensor-core U side held in shared memory at once (64 ranks
  // each); the streamed classes cycle larger ranks through them
  static constexpr int kZSlots = !kStream ? 16 : (MC <= 32 ? 8 : (MC <= 64 ? 3 : 2));
  // from 64 rows the epilogue reads the accumulator and the U-side product 16
  // columns at a time (a thread cannot hold a whole row of either)
  static constexpr bool kChunkedEpi = MC > 32;
};

// Global activation image (8+ rows), per 256-element K chunk:
//  * classes 8 and 16: the 16 x 128 B code rows exactly as the operand cache holds
//    them (128-byte swizzle), then 256 B of block scales, 64 B per 64-element K
//    step (row m at byte 4 m, block b of the step at byte b);
//  * classes 32, 64, 128: the MC x 128 B code rows (128-byte swizzle), then the
//    block scales as four 512-byte scale atoms, one per K step, in the layout the
//    tensor memory copy expects: 32 lines of 16 bytes, row m's four scales at
//    bytes 16 (m % 32) + 4 (m / 32) .. + 3 (bytes no row of the class uses are
//    zero).  A stage's activation part is one bulk copy of it.
template <int MC>
struct QImg {
  static constexpr int kCodes = Cfg<MC>::kBN * 128;
  static constexpr int kBytes = kCodes + (Cfg<MC>::kStream ? 4 * 512 : 256);
};

template <int MC>
struct Layout {
  static constexpr int kStages = Cfg<MC>::kStages;
  static constexpr int kRankGroup = Cfg<MC>::kRankGroup;
  static constexpr int kBN = Cfg<MC>::kBN;
  static constexpr int kMaxUnits = Cfg<MC>::kMaxUnits;
  static constexpr bool kStream = Cfg<MC>::kStream;
  // a stage: the weight unit's codes and scale atoms, and (streamed classes) the
  // activation chunk's codes and scale atoms
  static constexpr int kStageA = 0;
  static constexpr int kStageSFA = kUnitBytesA;
  static constexpr int kStageB = kStageSFA + kSfBytes;
  static constexpr int kStageSFB = kStageB + kBN * 128;
  static constexpr int kStageBytes = kStageSFB + kSfBytes;
  static_assert(kStageBytes == kUnitBytesA + kSfBytes + QImg<MC>::kBytes || !kStream,
                "a stage's activation part is one image chunk");
  static constexpr int kA = 0;                                        // [ST][128][128 B] (cache classes)
  static constexpr int kSFA = kA + kStages * kUnitBytesA;              // [ST][2 KB]
  static constexpr int kB = kSFA + kStages * kSfBytes;                 // [NU][16][128 B] operand cache
  static constexpr int kSFB = kB + kMaxUnits * kBN * 128;              // [NU][4 steps][32 rows] u32
  static constexpr int kCacheEnd = kSFB + kMaxUnits * 512;
  // first byte past the stages (streamed) or the operand cache
  static constexpr int kFree = kStream ? kStages * kStageBytes : kCacheEnd;
  // U side on the tensor cores: A = the tile's U signs as +-1 BF16, 64 ranks per
  // chunk (two buffers); B = z as BF16 high and low parts, kUN rows per chunk
  static constexpr int kUN = (2 * MC < 16) ? 16 : 2 * MC;               // MMA N of the U side
  static constexpr int kUA = kFree;                                     // [2][128][128 B]
  static constexpr int kUZ = kUA + 2 * kTileRows * 128;                // [kZSlots][kUN][128 B]
  // without the tensor-core U side: z staged as floats, the two half sums, and the
  // signed-sum table of z (16 entries per 4 ranks)
  static constexpr int kZ = kFree;                                     // [MC][1024] floats
  static constexpr int kCorr = kZ + MC * kMaxRanks * 4;                // [2][MC][128] floats
  static constexpr int kLut = kCorr + 2 * MC * kTileRows * 4;          // [MC][256 groups][16] floats
  static constexpr int kUEnd = Cfg<MC>::kTensorU ? kUZ + Cfg<MC>::kZSlots * kUN * 128
                                                 : kLut + MC * kMaxRanks * 16;
  static constexpr int kVRed = kUEnd;                                  // [8][MC * ranks] floats
  static constexpr int kVRedBytes = Cfg<MC>::kTensorV ? 0 : kAluWarps * MC * kRankGroup * 4;
  static constexpr int kBar = kVRed + kVRedBytes;
  static constexpr int kNumBars = 2 * kStages + 18;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kFinFlags = kMisc + 32;                         // [kMaxUnits + 1] ints
  static constexpr int kTotal = kFinFlags + (kMaxUnits + 1) * 4;
  static constexpr int kAlloc = kTotal + 1024;
  // TMEM columns.  Cache classes: accumulators [0, 32), activation scales per unit
  // [32, 288), weight scales per stage [288, 384), the two U-side product buffers
  // [384, 384 + 2 kUN), the V-side product [448, 464).  Streamed classes:
  // accumulators [0, 2 MC), weight and activation scales per stage, then the U-side
  // product buffers (kUBufs x kUCols) and the V-side product (MC columns; from 64
  // rows it shares the first U-side buffer: the V pieces are read out before this
  // CTA's z exists, and no U-side MMA runs before z does).
  static constexpr int kUCols = Cfg<MC>::kUSum ? MC : kUN;             // columns per U-side buffer
  static constexpr int kTmSfb = kStream ? 2 * kBN + kStages * 16 : 32;
  static constexpr int kTmSfa = kStream ? 2 * kBN : kTmSfb + kMaxUnits * 16;
  static constexpr int kTmU = kStream ? kTmSfb + kStages * 16 : 384;
  static constexpr int kTmV = kStream ? (Cfg<MC>::kUSum ? kTmU : kTmU + Cfg<MC>::kUBufs * kUCols) : 448;
  static_assert(!Cfg<MC>::kTensorU || kTmU + Cfg<MC>::kUBufs * kUCols <= (Cfg<MC>::kUSum ? kTmemCols : kTmV),
                "U-side product buffers");
  static_assert(kTmV + kBN <= kTmemCols, "tensor memory budget");
  static_assert(kStream || kTmSfa + kStages * 16 <= kTmU, "tensor memory budget");
  static_assert(kSFA % 1024 == 0 && kB % 1024 == 0 && kUA % 1024 == 0 && kUZ % 1024 == 0 &&
                kStageBytes % 1024 == 0 && kStageB % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kAlloc <= 232448, "shared memory budget");
  // the tensor-core V side's buffers alias the U side's (unused until z is complete)
  static_assert(!Cfg<MC>::kTensorV || kVAtoms * (kTileRows + kBN) * 128 <= kUEnd - kUA,
                "V-side buffers fit the U side's");
};

// One z value's two BF16 parts into the global tile image of the U side's B
// operand: chunk i / 64 of kUN rows x 128 bytes, element i % 64 of row m (high)
// and row MC + m (low), 128-byte swizzle (16-byte piece j of row q at j ^ (q & 7)).
__device__ __forceinline__ void store_ztile(uint8_t* tiles, int kUN, int MC, int m, int i, __nv_bfloat16 hi,
                                            __nv_bfloat16 lo) {
  const int c = i >> 6, byte = (i & 63) * 2;
  uint8_t* tile = tiles + static_cast<size_t>(c) * kUN * 128;
  const int rl = MC + m;
  *reinterpret_cast<uint16_t*>(tile + m * 128 + ((((byte >> 4) ^ (m & 7)) << 4) | (byte & 15))) =
      __bfloat16_as_ushort(hi);
  *reinterpret_cast<uint16_t*>(tile + rl * 128 + ((((byte >> 4) ^ (rl & 7)) << 4) | (byte & 15))) =
      __bfloat16_as_ushort(lo);
}

// V side: how the 8 CUDA-core warps share the rows and the K blocks (256
// elements each).  A warp owns kRows = min(MC, 4) rows, row0, row0 + kStep, ..
// (kStep = MC / kRows row groups), and the kSplit = 8 / kStep warps of one row
// group split K between them.
template <int MC>
struct VSplit {
  static constexpr int kRows = (MC >= 4) ? 4 : MC;          // rows per warp
  static constexpr int kStep = MC / kRows;                  // row groups
  static constexpr int kSplit = kAluWarps / kStep;          // warps per row group (K split)
  __device__ static int row0(int a) { return a % kStep; }
  __device__ static int kb0(int a) { return a / kStep; }
  // warp q (< kSplit) of those holding row m, and the row's slot in that warp
  __device__ static int warp_of(int m, int q) { return m % kStep + kStep * q; }
  __device__ static int slot_of(int m) { return m / kStep; }
};

// V-side partial sums of one warp: rows row0 + j kStep (j < kRows), the K blocks
// kb0, kb0 + kSplit, ..; lane l takes elements 8 l .. 8 l + 7 of a block with one
// 16-byte load per row, and the matching byte of the block's sign words (word
// 8 kb + l / 4, bits 8 (l % 4) ..).  Loads run kVStages blocks ahead.  The sign-adds
// are packed FP32 FMAs with +-1.0 multipliers (exact products, one rounding per
// add, as a plain add or subtract): one instruction covers an element pair, even
// and odd elements in the two lanes of a pair accumulator.  Each lane returns
// acc[j][i] for row row0 + j kStep and rank ig + i (ranks i >= nr are left at
// zero).  Inputs that the previous kernel of the stream may have written are read
// through L2 (ld.global.cg), never through a possibly stale L1 line.
// CTAs that share the grid-wide work (z slices, activation image items, V pieces).
// The last CTAs of a large grid are left out: they are dispatched last, onto SMs
// still held by the previous kernel's completing CTAs, and pass the dependency wait
// 0.3 to 2 us after the others (measured on B200), so any share of that work would
// hold up every reader of it.
__device__ __forceinline__ int shared_work_ctas(const DecodeParams& p) {
  return p.G >= 96 ? p.G - 16 : (p.G > 16 ? p.G - 2 : p.G);
}

// K slices per rank block of the tensor-core V side: one piece per sharing CTA
// where there are enough, at most 32 (the cross-CTA sum of a (rank, row) pair takes
// four lanes x eight partial sums).
constexpr int kVSliceMax = 32;
__device__ __forceinline__ int vside_slices(const DecodeParams& p, int RB) {
  return max(1, min(min(shared_work_ctas(p) / RB, p.K / 64), kVSliceMax));
}

// V-side partial sums of one warp: rows row0 + j kStep (j < kRows), the K blocks
// kb0, kb0 + kSplit, ..; lane l takes elements 8 l .. 8 l + 7 of a block with one
// 16-byte load per row, and the matching byte of the block's sign words (word
// 8 kb + l / 4, bits 8 (l % 4) ..).  Loads run kVStages blocks ahead.  The sign-adds
// are packed FP32 FMAs with +-1.0 multipliers (exact products, one rounding per
// add, as a plain add or subtract): one instruction covers an element pair, even
// and odd elements in the two lanes of a pair accumulator.  Each lane returns
// acc[j][i] for row row0 + j kStep and rank ig + i (ranks i >= nr are left at
// zero).  Inputs that the previous kernel of the stream may have written are read
// through L2 (ld.global.cg), never through a possibly stale L1 line.
template <int MC, int kRankGroup = Cfg<MC>::kRankGroup>
__device__ __forceinline__ void vside_rows(const DecodeParams& p, int ig, int nr, int a, int lane,
                                           float (&acc)[VSplit<MC>::kRows][kRankGroup]) {
  using VS = VSplit<MC>;
  constexpr int RPW = VS::kRows, kbs = VS::kSplit;
  const int row0 = VS::row0(a), kb0 = VS::kb0(a);
  const int nkb = (p.K + 255) / 256;
  uint64_t acc2[RPW][kRankGroup];
#pragma unroll
  for (int j = 0; j < RPW; ++j)
#pragma unroll
    for (int i = 0; i < kRankGroup; ++i) acc2[j][i] = 0ull;
  struct Stage {
    uint4 x[RPW];
    uint32_t v[kRankGroup];
  };
  auto load = [&](int kb, Stage& st) {
    const int k0 = kb * 256 + lane * 8;
    const bool kin = kb < nkb && k0 < p.K;
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
      const int m = row0 + VS::kStep * j;
      st.x[j] = (kin && m < p.M) ? __ldcg(reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(m) * p.K + k0))
                                 : make_uint4(0u, 0u, 0u, 0u);
    }
    const int w = kb * 8 + (lane >> 2);
#pragma unroll
    for (int i = 0; i < kRankGroup; ++i)
      st.v[i] = (kin && i < nr) ? __ldcg(p.Vbits + static_cast<size_t>(ig + i) * p.KW + w) : 0u;
  };
  // a ring of kVStages stages indexed statically (the loop body is unrolled that
  // many times), so that no register copy waits on the load issued last
  constexpr int NS = Cfg<MC>::kVStages;
  Stage st[NS];
#pragma unroll
  for (int q = 0; q < NS; ++q) load(kb0 + q * kbs, st[q]);
  const uint32_t bshift = 8u * static_cast<uint32_t>(lane & 3);
#pragma unroll 1
  for (int t = kb0; t < nkb; t += NS * kbs) {
#pragma unroll
    for (int q = 0; q < NS; ++q) {
      if (t + q * kbs < nkb) {
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {               // element pair 2 pr, 2 pr + 1
          uint64_t x2[RPW];
#pragma unroll
          for (int j = 0; j < RPW; ++j) {
            const uint32_t w = (pr == 0) ? st[q].x[j].x : (pr == 1) ? st[q].x[j].y : (pr == 2) ? st[q].x[j].z : st[q].x[j].w;
            x2[j] = f32x2_pack(w << 16, w & 0xFFFF0000u);
          }
#pragma unroll
          for (int i = 0; i < kRankGroup; ++i) {
            if (i < nr) {
              const uint32_t bits = st[q].v[i] >> bshift;    // this lane's 8 sign bits
              const uint32_t s0 = ((bits << (31 - 2 * pr)) & 0x80000000u) | 0x3F800000u;
              const uint32_t s1 = ((bits << (30 - 2 * pr)) & 0x80000000u) | 0x3F800000u;
              const uint64_t s2 = f32x2_pack(s0, s1);
#pragma unroll
              for (int j = 0; j < RPW; ++j) acc2[j][i] = f32x2_fma(x2[j], s2, acc2[j][i]);
            }
          }
        }
      }
      load(t + (q + NS) * kbs, st[q]);
    }
  }
#pragma unroll
  for (int j = 0; j < RPW; ++j)
#pragma unroll
    for (int i = 0; i < kRankGroup; ++i) acc[j][i] = f32x2_sum(acc2[j][i]);
}

// Signed-sum table of z for the CUDA-core U side (the LUT form of the correction
// arithmetic): for every row m and group g of four ranks, entry b (0..15) is
// sum_j (bit j of b ? -z[4 g + j] : z[4 g + j]), so that the four sign bits of a
// weight row select the row's contribution of those ranks with one load.  Built
// from the staged z (zero past r) by `nthreads` threads.
template <int MC>
__device__ __forceinline__ void build_z_table(const float* zs, float* lut, int M, int RW, int tid, int nthreads) {
  const int groups = 8 * RW;
  for (int idx = tid; idx < M * groups; idx += nthreads) {
    const int m = idx / groups, g = idx - m * groups;
    const float4 z = *reinterpret_cast<const float4*>(zs + m * kMaxRanks + 4 * g);
    float4* t = reinterpret_cast<float4*>(lut + (m * (kMaxRanks / 4) + g) * 16);
    float e[16];
#pragma unroll
    for (int b = 0; b < 16; ++b)
      e[b] = (((b & 1) ? -z.x : z.x) + ((b & 2) ? -z.y : z.y)) + (((b & 4) ? -z.z : z.z) + ((b & 8) ? -z.w : z.w));
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) t[q4] = make_float4(e[4 * q4], e[4 * q4 + 1], e[4 * q4 + 2], e[4 * q4 + 3]);
  }
}

// One rank word (32 ranks from word index w) of a weight row's U z, added into
// four interleaved sums per activation row: sign-adds on the staged z, or (lut)
// eight lookups in the signed-sum table.
template <int MC, bool kLut>
__device__ __forceinline__ void u_word_sum(const float* zs, const float* lut, uint32_t word, int w, int M,
                                           float (&acc4)[MC][4]) {
  if constexpr (kLut) {
    const float* tw = lut + w * 8 * 16;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      const uint32_t nib = (word >> (4 * nb)) & 15u;
#pragma unroll
      for (int m = 0; m < MC; ++m)
        if (m < M) acc4[m][nb & 3] += tw[m * (kMaxRanks / 4) * 16 + nb * 16 + nib];
    }
  } else {
    const float* zw = zs + w * 32;
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
#pragma unroll
      for (int m = 0; m < MC; ++m) {
        if (m < M) {
          const float4 z4 = *reinterpret_cast<const float4*>(zw + m * kMaxRanks + 4 * j4);
          const float zz[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint32_t sgn = (word << (31 - (4 * j4 + jj))) & 0x80000000u;
            acc4[m][jj] += __uint_as_float(__float_as_uint(zz[jj]) ^ sgn);
          }
        }
      }
    }
  }
}

// The operand cache starts zero: rows >= M and blocks past K stay zero.
template <int MC>
__device__ __forceinline__ void zero_cache(uint8_t* smem, int nunits, int tid, int nthreads) {
  using L = Layout<MC>;
  for (int idx = tid; idx < nunits * 160; idx += nthreads) {
    const int k = idx / 160, o = idx - k * 160;
    uint4* dst = (o < 128) ? reinterpret_cast<uint4*>(smem + L::kB + k * L::kBN * 128) + o
                           : reinterpret_cast<uint4*>(smem + L::kSFB + k * 512) + (o - 128);
    *dst = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Quantise the activation chunks of every unit of this CTA into the operand cache
// (codes in the MMA's 128-byte-swizzled rows, scales staged for TMEM): two blocks
// per thread per round, the loop rolled (the quantiser is long straight-line code;
// unrolled deeper it would crowd the instruction cache).
template <int MC>
__device__ __forceinline__ void quant_into_cache(const DecodeParams& p, uint8_t* smem, int u0, int nunits, int tid,
                                                 int nthreads) {
  using L = Layout<MC>;
  constexpr int kQB = 2;
  const int per_unit = p.M * 16;
  const int items = nunits * per_unit;
#pragma unroll 1
  for (int base = 0; base < items; base += nthreads * kQB) {
    uint4 lo[kQB], hi[kQB];
#pragma unroll
    for (int e = 0; e < kQB; ++e) {
      const int idx = base + e * nthreads + tid;
      lo[e] = hi[e] = make_uint4(0u, 0u, 0u, 0u);
      if (idx < items) {
        const int k = idx / per_unit, rem = idx - k * per_unit, m = rem >> 4, blk = rem & 15;
        const int kk = ((u0 + k) % p.KC) * kUnitK + blk * 16;
        if (kk < p.K) {
          const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(m) * p.K + kk);
          lo[e] = __ldcg(src);
          hi[e] = __ldcg(src + 1);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < kQB; ++e) {
      const int idx = base + e * nthreads + tid;
      if (idx < items) {
        const int k = idx / per_unit, rem = idx - k * per_unit, m = rem >> 4, blk = rem & 15;
        const int kk = ((u0 + k) % p.KC) * kUnitK + blk * 16;
        if (kk < p.K) {
          float v[16];
          bf16x16_to_f32(lo[e], hi[e], v);
          uint2 codes;
          const uint32_t s = quant_act_block_fast(v, codes);
          const int j = blk * 8;
          *reinterpret_cast<uint2*>(smem + L::kB + k * L::kBN * 128 + m * 128 +
                                    ((((j >> 4) ^ (m & 7)) << 4) | (j & 15))) = codes;
          smem[L::kSFB + k * 512 + (blk >> 2) * 128 + m * 4 + (blk & 3)] = static_cast<uint8_t>(s);
        }
      }
    }
  }
}

// Activation scales to TMEM, in the layout a 32x128b.warpx4 copy of scale atoms
// would give: lane i of every lane quarter holds, in column 16 k + 4 j, the four
// block scales of row i for K step j of unit k (rows >= 16 and the other three
// columns of a step are zero).  Called by one warp per lane quarter.
template <int MC>
__device__ __forceinline__ void sfb_to_tmem(const uint8_t* smem, uint32_t tmem, int nunits, uint32_t quarter,
                                            int lane) {
  using L = Layout<MC>;
  for (int k = 0; k < nunits; ++k) {
    const uint32_t* sfb = reinterpret_cast<const uint32_t*>(smem + L::kSFB + k * 512) + lane;
    uint32_t v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[4 * j] = sfb[j * 32];
      v[4 * j + 1] = v[4 * j + 2] = v[4 * j + 3] = 0u;
    }
    tmem_st16(tmem + ((quarter * 32) << 16) + L::kTmSfb + k * 16, v);
  }
  tmem_wait_st();
}

// kLut (1-2 rows): the U side adds lookups in the signed-sum table of z instead of
// sign-adds (each instance carries only its own loop: the code size of these
// kernels shows in their instruction-cache misses)
template <int MC, bool kLut>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ DecodeParams p) {
  using L = Layout<MC>;
  constexpr int kStages = Cfg<MC>::kStages, kRankGroup = Cfg<MC>::kRankGroup;
  constexpr int kBN = Cfg<MC>::kBN;
  constexpr bool kStream = Cfg<MC>::kStream;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[kStages + s]); };
  const uint32_t actr_bar = smem_u32(&bars[2 * kStages]);
  auto accf_bar = [&](int b) { return smem_u32(&bars[2 * kStages + 1 + b]); };
  auto acce_bar = [&](int b) { return smem_u32(&bars[2 * kStages + 3 + b]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * kStages + 5]);
  const uint32_t done_bar = smem_u32(&bars[2 * kStages + 6]);
  auto ubuf_bar = [&](int b) { return smem_u32(&bars[2 * kStages + 7 + b]); };
  // the U-side product of segment s lands in TMEM buffer s & 1: ud_bar(b) when it
  // is ready (tcgen05.commit), uread_bar(b) when the epilogue has read it
  auto ud_bar = [&](int b) { return smem_u32(&bars[b ? 2 * kStages + 13 : 2 * kStages + 9]); };
  auto uread_bar = [&](int b) { return smem_u32(&bars[2 * kStages + 14 + b]); };
  const uint32_t qpass_bar = smem_u32(&bars[2 * kStages + 16]);   // streamed class: the producer passed the image wait
  const uint32_t zst_bar = smem_u32(&bars[2 * kStages + 17]);     // the z tiles' bulk copies into the slots
  auto ufull_bar = [&](int b) { return smem_u32(&bars[2 * kStages + 10 + b]); };
  const uint32_t vmma_bar = smem_u32(&bars[2 * kStages + 12]);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* epi_last = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  volatile int* fin_flag = reinterpret_cast<volatile int*>(smem + L::kFinFlags);
  const Ctl ctl{abort_flag, p.status};

  const int g = blockIdx.x;
  const int u0 = first_unit(g, p.G, p.U), u1 = first_unit(g + 1, p.G, p.U);
  const int t_first = u0 / p.KC, t_last = (u1 - 1) / p.KC;
  const int nseg = t_last - t_first + 1;
  const int nunits = u1 - u0;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_w);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(actr_bar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), kEpiThreads);
    }
    mbar_init(drain_bar, 1);
    mbar_init(done_bar, kWarps);
    mbar_init(ubuf_bar(0), 1);
    mbar_init(ubuf_bar(1), 1);
    mbar_init(ud_bar(0), 1);
    mbar_init(ud_bar(1), 1);
    mbar_init(uread_bar(0), kEpiThreads);
    mbar_init(uread_bar(1), kEpiThreads);
    mbar_init(qpass_bar, 1);
    mbar_init(zst_bar, 1);
    mbar_init(ufull_bar(0), kAluThreads);
    mbar_init(ufull_bar(1), kAluThreads);
    mbar_init(vmma_bar, 1);
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

  // Programmatic dependent launch: the next kernel may take this CTA's SM as
  // soon as it leaves.  The producer streams only the weight operand and never
  // waits for the previous kernel; the epilogue and CUDA-core warps wait below.
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // (one thread; the unit's tile and chunk advance incrementally: no divisions)
    if (lane == 0) {
      int issued = 0;
      int t = u0 / p.KC, c = u0 - t * p.KC;
      int s = 0;
      uint32_t ph = 0;                                   // parity of the stage's current use
      const uint8_t* sf = p.w_sf + static_cast<size_t>(u0) * kSfBytes;
      if constexpr (!kStream) {
        for (int k = 0; k < nunits; ++k) {
          if (k >= kStages && !mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) {
            fail(ctl);
            break;
          }
          mbar_arrive_expect_tx(full_bar(s), kStageTx);
          tma_load_2d(smem_u32(smem + L::kA + s * kUnitBytesA), &tmap_w, full_bar(s), c * 128, t * kTileRows);
          bulk_load(smem_u32(smem + L::kSFA + s * kSfBytes), sf, kSfBytes, full_bar(s));
          ++issued;
          sf += kSfBytes;
          if (++c == p.KC) { c = 0; ++t; }
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      } else {
        // A stage = the weight unit (TMA tile + scale atoms) and the activation
        // chunk of the same K range (one bulk copy of its image chunk).  The weight
        // parts of the first stages are requested at once; the activation parts
        // once every CTA has published its part of the image, which this thread
        // waits for itself; always issued, so that every stage's transaction count
        // completes even after a failed wait.
        constexpr uint32_t kImg = QImg<MC>::kBytes;
        const int pre = min(nunits, kStages);
        for (int k = 0; k < pre; ++k) {
          uint8_t* st = smem + k * L::kStageBytes;
          mbar_arrive_expect_tx(full_bar(k), kStageTx + kImg);
          tma_load_2d(smem_u32(st + L::kStageA), &tmap_w, full_bar(k), c * 128, t * kTileRows);
          bulk_load(smem_u32(st + L::kStageSFA), sf, kSfBytes, full_bar(k));
          sf += kSfBytes;
          if (++c == p.KC) { c = 0; ++t; }
        }
        // every CTA has written its part of the activation image (the counter
        // belongs to this call once the previous kernel of the stream has ended)
        griddep_wait();
        bool ok = spin_until_geq(p.q_ready, static_cast<uint32_t>(p.G), ctl);
        if (!ok) fail(ctl);
        mbar_arrive(qpass_bar);                          // done with the grid counters
        fence_proxy_async_global();                      // the image was written through the generic proxy
        int ca = u0 % p.KC;
        for (int k = 0; k < pre; ++k) {
          bulk_load(smem_u32(smem + k * L::kStageBytes + L::kStageB), p.xq + static_cast<size_t>(ca) * kImg, kImg,
                    full_bar(k));
          if (++ca == p.KC) ca = 0;
        }
        issued = pre;
        s = pre % kStages;
        ph = (pre == kStages) ? 1u : 0u;
        for (int k = pre; k < nunits && ok; ++k) {
          if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) {
            fail(ctl);
            break;
          }
          uint8_t* st = smem + s * L::kStageBytes;
          mbar_arrive_expect_tx(full_bar(s), kStageTx + kImg);
          tma_load_2d(smem_u32(st + L::kStageA), &tmap_w, full_bar(s), c * 128, t * kTileRows);
          bulk_load(smem_u32(st + L::kStageSFA), sf, kSfBytes, full_bar(s));
          bulk_load(smem_u32(st + L::kStageB), p.xq + static_cast<size_t>(c) * kImg, kImg, full_bar(s));
          ++issued;
          sf += kSfBytes;
          if (++c == p.KC) { c = 0; ++t; }
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
      // never leave the CTA with copies in flight
      for (int k = max(0, issued - kStages); k < issued; ++k) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(full_bar(k % kStages), (k / kStages) & 1)) {
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
    // One thread issues every tcgen05 instruction; descriptors are built once and
    // offset per unit (the 14-bit address field counts 16-byte units and never
    // carries here).
    if (lane == 0) {
      const uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                             (static_cast<uint32_t>(kTileRows >> 4) << 24);
      // cache classes: stage s at kA + s 16 KB (codes) and kSFA + s 2 KB (scales),
      // activation unit k in the operand cache; streamed class: everything in
      // stage s at s * kStageBytes
      const SmemDesc a_desc0 = make_sdesc(smem_u32(smem + (kStream ? L::kStageA : L::kA)), 16, 1024, 2);
      const SmemDesc b_desc0 = make_sdesc(smem_u32(smem + (kStream ? L::kStageB : L::kB)), 16, 1024, 2);
      const SmemDesc sfa_desc0 = make_sdesc(smem_u32(smem + (kStream ? L::kStageSFA : L::kSFA)), 0, 128, 0);
      const SmemDesc sfb_desc0 = make_sdesc(smem_u32(smem + L::kStageSFB), 0, 128, 0);
      constexpr uint32_t kAtom = 512 >> 4;
      constexpr uint32_t kUnitSf = (kStream ? L::kStageBytes : kSfBytes) >> 4;
      constexpr uint32_t kUnitA = (kStream ? L::kStageBytes : kUnitBytesA) >> 4;
      constexpr uint32_t kUnitB = (kBN * 128) >> 4, kStageB = L::kStageBytes >> 4;
      // cache classes: the weight scales of the stages already requested go to
      // TMEM while the activation is still being quantised
      const int pre = kStream ? 0 : min(nunits, kStages);
      bool ok = true;
      for (int j = 0; j < pre && ok; ++j) {
        if (!mbar_wait(full_bar(j), 0, abort_flag)) {
          fail(ctl);
          ok = false;
          break;
        }
        tc_fence_after();
        const SmemDesc sfa_d = sdesc_at(sfa_desc0, static_cast<uint32_t>(j) * kUnitSf);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tc_cp_32x128b_warpx4(tmem + L::kTmSfa + j * 16 + 4 * q, sdesc_at(sfa_d, kAtom * q));
      }
      // the activation codes (shared memory) and scales (TMEM) are in place
      if (!kStream && ok && !mbar_wait(actr_bar, 0, abort_flag)) {
        fail(ctl);
        ok = false;
      }
      tc_fence_after();
      int k = 0, s = 0;
      uint32_t ph = 0;
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
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * kBN);
        for (int u = ua; u < ub; ++u, ++k) {
          const uint32_t sfa_t = tmem + L::kTmSfa + s * 16;
          const uint32_t sfb_t = tmem + L::kTmSfb + (kStream ? s : k) * 16;
          if (k >= pre) {
            if (!mbar_wait(full_bar(s), ph, abort_flag)) {
              fail(ctl);
              ok = false;
              break;
            }
            tc_fence_after();
            const SmemDesc sfa_d = sdesc_at(sfa_desc0, static_cast<uint32_t>(s) * kUnitSf);
#pragma unroll
            for (int q = 0; q < 4; ++q) tc_cp_32x128b_warpx4(sfa_t + 4 * q, sdesc_at(sfa_d, kAtom * q));
            if constexpr (kStream) {
              const SmemDesc sfb_d = sdesc_at(sfb_desc0, static_cast<uint32_t>(s) * kStageB);
#pragma unroll
              for (int q = 0; q < 4; ++q) tc_cp_32x128b_warpx4(sfb_t + 4 * q, sdesc_at(sfb_d, kAtom * q));
            }
          }
          const SmemDesc a_d = sdesc_at(a_desc0, static_cast<uint32_t>(s) * kUnitA);
          const SmemDesc b_d = kStream ? sdesc_at(b_desc0, static_cast<uint32_t>(s) * kStageB)
                                       : sdesc_at(b_desc0, static_cast<uint32_t>(k) * kUnitB);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tc_mma_nvf4(d_tmem, sdesc_at(a_d, 2 * j), sdesc_at(b_d, 2 * j), idesc, sfa_t + 4 * j, sfb_t + 4 * j,
                        (u > ua || j > 0) ? 1u : 0u);
          tc_commit(empty_bar(s));
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        if (ok) tc_commit(accf_bar(b));
      }
      // every MMA and scale copy issued so far must finish before TMEM is freed
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
    const int etid = threadIdx.x - kEpiWarp0 * 32;
    griddep_wait();
    const float gs = __ldcg(p.gscale);
    constexpr int kHB = (MC <= 2) ? 16 : (MC <= 4 ? 8 : (MC <= 8 ? 6 : (MC <= 16 ? 3 : 1)));   // partials loaded per batch
    // the accumulator of buffer b for this warp's lane quarter, times g
    auto load_acc = [&](int b, float (&v)[MC]) {
#pragma unroll
      for (int c0 = 0; c0 < MC; c0 += 16) {
        uint32_t raw[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * kBN + c0), raw);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (c0 + j < MC) v[c0 + j] = __fmul_rn(gs, __uint_as_float(raw[j]));
      }
    };
    if constexpr (Cfg<MC>::kChunkedEpi) {
      // 64+ rows: once the segment's FP4 product and (r > 0) this CTA's share of U z
      // are both in TMEM, read them 16 columns at a time; a sole owner stores y
      // directly, a split-K contributor publishes its partial and the last one to
      // arrive sums every contributor's partial (its own included) from the slots
      constexpr int kUB = Cfg<MC>::kUBufs;
      bool ok = true;
      for (int seg = 0; seg < nseg; ++seg) {
        const int t = t_first + seg;
        const int b = seg & 1, ubf = seg % kUB;
        const int hf = owner_cta(static_cast<uint32_t>(t * p.KC), p.G, p.U);
        const int hl = owner_cta(static_cast<uint32_t>((t + 1) * p.KC - 1), p.G, p.U);
        const bool sole = hf == hl;
        const int which = (t == t_first) ? 0 : 1;
        const int nuc = (p.r + kUChunk - 1) / kUChunk;
        const int ua = max(u0, t * p.KC), ub = min(u1, (t + 1) * p.KC);
        const bool addu = p.r > 0 && (ub - t * p.KC) * nuc / p.KC > (ua - t * p.KC) * nuc / p.KC;
        if (ok) ok = group_wait(accf_bar(b), (seg >> 1) & 1, kBarEpi, kEpiThreads, ctl);
        if (ok && p.r > 0) ok = group_wait(ud_bar(ubf), (seg / kUB) & 1, kBarEpi, kEpiThreads, ctl);
        uint16_t* yb = p.y + static_cast<size_t>(t) * kTileRows + row;
        float* my_slot = p.slots + static_cast<size_t>(2 * g + which) * kBN * kTileRows;
        if (ok) {
          tc_fence_after();
          const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
  #pragma unroll 1
          for (int c0 = 0; c0 < MC; c0 += 16) {
            uint32_t ra[16], ru[16];
            if (addu) {
              tmem_ld16x2(lane_base + static_cast<uint32_t>(b * kBN + c0), ra,
                          lane_base + L::kTmU + static_cast<uint32_t>(ubf * L::kUCols + c0), ru);
            } else {
              tmem_ld16(lane_base + static_cast<uint32_t>(b * kBN + c0), ra);
            }
  #pragma unroll
            for (int j = 0; j < 16; ++j) {
              float v = __fmul_rn(gs, __uint_as_float(ra[j]));
              if (addu) v += __uint_as_float(ru[j]);
              if (c0 + j < p.M) {
                if (sole) yb[static_cast<size_t>(c0 + j) * p.N] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                else my_slot[(c0 + j) * kTileRows + row] = v;
              }
            }
          }
          tc_fence_before();
          mbar_arrive(acce_bar(b));
        }
        // the U-side buffer may take its next product (arrived on every path, so
        // that the phases stay in step)
        if (p.r > 0) {
          tc_fence_before();
          mbar_arrive(uread_bar(ubf));
        }
        if (!ok) break;
        if (sole) continue;
        named_barrier(kBarEpi, kEpiThreads);
        if (etid == 0) {
          // release: this CTA's partial; acquire: every earlier contributor's
          const uint32_t nh = static_cast<uint32_t>(hl - hf + 1);
          const uint32_t old = atom_add_acq_rel_gpu(p.tickets + t, 1u);
          const bool last = old == nh - 1;
          if (last) atomicExch(p.tickets + t, 0u);
          *epi_last = last ? 1 : 0;
        }
        named_barrier(kBarEpi, kEpiThreads);
        const bool fin = *epi_last != 0;
        named_barrier(kBarEpi, kEpiThreads);
        if (!fin) continue;
        // every contributor's partial, summed in contributor order, 16 rows at a
        // time, two contributors per batch of loads
        const int wh_first = (t == first_unit(hf, p.G, p.U) / p.KC) ? 0 : 1;
  #pragma unroll 1
        for (int j0 = 0; j0 < MC && j0 < p.M; j0 += 16) {
          float acc[16];
  #pragma unroll
          for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.0f;
          for (int h0 = hf; h0 <= hl; h0 += 2) {
            float part[2][16];
  #pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int h = h0 + e;
              const float* sl = p.slots + static_cast<size_t>(2 * h + ((h == hf) ? wh_first : 0)) * kBN * kTileRows;
  #pragma unroll
              for (int jj = 0; jj < 16; ++jj)
                part[e][jj] = (h <= hl && j0 + jj < p.M) ? __ldcg(sl + (j0 + jj) * kTileRows + row) : 0.0f;
            }
  #pragma unroll
            for (int e = 0; e < 2; ++e)
              if (h0 + e <= hl) {
  #pragma unroll
                for (int jj = 0; jj < 16; ++jj) acc[jj] += part[e][jj];
              }
          }
  #pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (j0 + jj < p.M) yb[static_cast<size_t>(j0 + jj) * p.N] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[jj]));
        }
      }
    } else if constexpr (Cfg<MC>::kUShares) {
      bool ok = true;
      for (int seg = 0; seg < nseg; ++seg) {
        const int t = t_first + seg;
        const int b = seg & 1;
        const int hf = owner_cta(static_cast<uint32_t>(t * p.KC), p.G, p.U);
        const int hl = owner_cta(static_cast<uint32_t>((t + 1) * p.KC - 1), p.G, p.U);
        const bool sole = hf == hl;
        const int which = (t == t_first) ? 0 : 1;
        float v[MC];
        if (ok) ok = group_wait(accf_bar(b), (seg >> 1) & 1, kBarEpi, kEpiThreads, ctl);
        if (ok) {
          tc_fence_after();
          load_acc(b, v);
          tc_fence_before();
          mbar_arrive(acce_bar(b));
        }
        if constexpr (Cfg<MC>::kTensorU) {
          if (p.r > 0) {
            // This CTA's share of U z for the tile (the 64-rank chunks [cs0, cs1), the
            // split the CUDA-core warps use), from TMEM buffer b once ud_bar(b) has
            // completed for this segment; the MMAs left sum_i U[n][i] zhi[m][i] in
            // column m and sum_i U[n][i] zlo[m][i] in column MC + m of lane n.
            const int nuc = (p.r + kUChunk - 1) / kUChunk;
            const int ua = max(u0, t * p.KC), ub = min(u1, (t + 1) * p.KC);
            const int cs0 = (ua - t * p.KC) * nuc / p.KC, cs1 = (ub - t * p.KC) * nuc / p.KC;
            if (ok) ok = group_wait(ud_bar(b), (seg >> 1) & 1, kBarEpi, kEpiThreads, ctl);
            if (ok && cs1 > cs0) {
              tc_fence_after();
              const uint32_t ucol = L::kTmU + static_cast<uint32_t>(b * L::kUN);
              if constexpr (L::kUN <= 32) {
                uint32_t du[32];
                if constexpr (L::kUN > 16)
                  tmem_ld16x2(tmem + (static_cast<uint32_t>(q * 32) << 16) + ucol, *reinterpret_cast<uint32_t(*)[16]>(du),
                              tmem + (static_cast<uint32_t>(q * 32) << 16) + ucol + 16,
                              *reinterpret_cast<uint32_t(*)[16]>(du + 16));
                else
                  tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + ucol, *reinterpret_cast<uint32_t(*)[16]>(du));
    #pragma unroll
                for (int j = 0; j < MC; ++j) v[j] += __uint_as_float(du[j]) + __uint_as_float(du[MC + j]);
              } else {
                // high parts in columns [0, MC), low parts in [MC, 2 MC): 16 rows at a time
    #pragma unroll
                for (int c0 = 0; c0 < MC; c0 += 16) {
                  uint32_t hi[16], lo[16];
                  tmem_ld16x2(tmem + (static_cast<uint32_t>(q * 32) << 16) + ucol + c0, hi,
                              tmem + (static_cast<uint32_t>(q * 32) << 16) + ucol + MC + c0, lo);
    #pragma unroll
                  for (int j = 0; j < 16; ++j) v[c0 + j] += __uint_as_float(hi[j]) + __uint_as_float(lo[j]);
                }
              }
            }
            // buffer b may take segment seg + 2's product (arrived on every path, so
            // that the phases stay in step)
            tc_fence_before();
            mbar_arrive(uread_bar(b));
          }
        }
        if (!ok) break;
        float acc[MC];
        if (sole) {
  #pragma unroll
          for (int j = 0; j < MC; ++j) acc[j] = v[j];
        } else {
          // publish this partial (FP4 product and U z share); the last contributor
          // of the tile completes it
          float* my_slot = p.slots + static_cast<size_t>(2 * g + which) * kBN * kTileRows;
  #pragma unroll
          for (int j = 0; j < MC; ++j)
            if (j < p.M) my_slot[j * kTileRows + row] = v[j];
          named_barrier(kBarEpi, kEpiThreads);
          if (etid == 0) {
            // release: this CTA's partial; acquire: every earlier contributor's
            const uint32_t nh = static_cast<uint32_t>(hl - hf + 1);
            const uint32_t old = atom_add_acq_rel_gpu(p.tickets + t, 1u);
            const bool last = old == nh - 1;
            if (last) atomicExch(p.tickets + t, 0u);
            *epi_last = last ? 1 : 0;
          }
          named_barrier(kBarEpi, kEpiThreads);
          const bool fin = *epi_last != 0;
          named_barrier(kBarEpi, kEpiThreads);
          if (!fin) continue;
          // every contributor's partial, summed in contributor order (the 32-row
          // class in two halves of 16 rows, three contributors per batch of loads)
  #pragma unroll
          for (int j = 0; j < MC; ++j) acc[j] = 0.0f;
          const int wh_first = (t == first_unit(hf, p.G, p.U) / p.KC) ? 0 : 1;
          constexpr int kRC = (MC > 16) ? 16 : MC;
          constexpr int kHBc = (MC > 16) ? 3 : kHB;
  #pragma unroll
          for (int j0 = 0; j0 < MC; j0 += kRC) {
            for (int h0 = hf; h0 <= hl; h0 += kHBc) {
              float part[kHBc][kRC];
  #pragma unroll
              for (int e = 0; e < kHBc; ++e) {
                const int h = h0 + e;
                const float* sl = p.slots + static_cast<size_t>(2 * h + ((h == hf) ? wh_first : 0)) *
                                                kBN * kTileRows;
  #pragma unroll
                for (int jj = 0; jj < kRC; ++jj)
                  part[e][jj] = (h <= hl && h != g && j0 + jj < p.M) ? __ldcg(sl + (j0 + jj) * kTileRows + row) : 0.0f;
              }
  #pragma unroll
              for (int e = 0; e < kHBc; ++e) {
                const int h = h0 + e;
                if (h <= hl) {
  #pragma unroll
                  for (int jj = 0; jj < kRC; ++jj) acc[j0 + jj] += (h == g) ? v[j0 + jj] : part[e][jj];
                }
              }
            }
          }
        }
        uint16_t* yb = p.y + static_cast<size_t>(t) * kTileRows + row;
  #pragma unroll
        for (int j = 0; j < MC; ++j)
          if (j < p.M) yb[static_cast<size_t>(j) * p.N] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
      }
    } else {
      bool ok = true;
      for (int seg = 0; seg < nseg; ++seg) {
        const int t = t_first + seg;
        const int b = seg & 1;
        const int hf = owner_cta(static_cast<uint32_t>(t * p.KC), p.G, p.U);
        const int hl = owner_cta(static_cast<uint32_t>((t + 1) * p.KC - 1), p.G, p.U);
        const bool sole = hf == hl;
        const int which = (t == t_first) ? 0 : 1;
        float v[MC];
        bool fin = false;
        if (ok) ok = group_wait(accf_bar(b), (seg >> 1) & 1, kBarEpi, kEpiThreads, ctl);
        if (ok) {
          tc_fence_after();
          load_acc(b, v);
          tc_fence_before();
          mbar_arrive(acce_bar(b));
          if (sole) {
            fin = true;
          } else {
            // publish this partial; the last contributor of the tile completes it
            float* my_slot = p.slots + static_cast<size_t>(2 * g + which) * kBN * kTileRows;
  #pragma unroll
            for (int j = 0; j < MC; ++j)
              if (j < p.M) my_slot[j * kTileRows + row] = v[j];
            named_barrier(kBarEpi, kEpiThreads);
            if (etid == 0) {
              // release: this CTA's partial; acquire: every earlier contributor's
              const uint32_t nh = static_cast<uint32_t>(hl - hf + 1);
              const uint32_t old = atom_add_acq_rel_gpu(p.tickets + t, 1u);
              const bool last = old == nh - 1;
              if (last) atomicExch(p.tickets + t, 0u);
              *epi_last = last ? 1 : 0;
            }
            named_barrier(kBarEpi, kEpiThreads);
            fin = *epi_last != 0;
            named_barrier(kBarEpi, kEpiThreads);
          }
        }
        if (p.r > 0) {
          // tell the CUDA-core warps whether this tile's correction is needed here
          if (etid == 0) fin_flag[seg] = fin ? 1 : 0;
          if (named_barrier_or(kBarFin, kFinThreads, !ok)) {
            if (ok) fail(ctl);
            ok = false;
          }
        }
        if (!ok) break;
        if (!fin) continue;
        float acc[MC];
        if (sole) {
  #pragma unroll
          for (int j = 0; j < MC; ++j) acc[j] = v[j];
        } else {
          // every contributor's partial, summed in contributor order
  #pragma unroll
          for (int j = 0; j < MC; ++j) acc[j] = 0.0f;
          const int wh_first = (t == first_unit(hf, p.G, p.U) / p.KC) ? 0 : 1;
          for (int h0 = hf; h0 <= hl; h0 += kHB) {
            float part[kHB][MC];
  #pragma unroll
            for (int e = 0; e < kHB; ++e) {
              const int h = h0 + e;
              const float* sl = p.slots + static_cast<size_t>(2 * h + ((h == hf) ? wh_first : 0)) *
                                              kBN * kTileRows;
  #pragma unroll
              for (int j = 0; j < MC; ++j)
                part[e][j] = (h <= hl && h != g && j < p.M) ? __ldcg(sl + j * kTileRows + row) : 0.0f;
            }
  #pragma unroll
            for (int e = 0; e < kHB; ++e) {
              const int h = h0 + e;
              if (h <= hl) {
  #pragma unroll
                for (int j = 0; j < MC; ++j) acc[j] += (h == g) ? v[j] : part[e][j];
              }
            }
          }
        }
        if (p.r > 0) {
          // the correction in three parts: the CUDA-core warps sum the first two
          // thirds of the rank words for every row, this thread the last third for
          // its own row, once the CUDA-core warps have staged z
          static_assert(!Cfg<MC>::kTensorU, "the completing-CTA U side is the sign-add one");
          const int w2 = 2 * p.RW / 3;
          const uint32_t* ur = p.Ubits + (static_cast<size_t>(t) * kTileRows + row) * p.RW;
          uint32_t uw[16];
  #pragma unroll
          for (int w = 0; w < 16; ++w) uw[w] = (w2 + w < p.RW) ? __ldcg(ur + w2 + w) : 0u;
          if (named_barrier_or(kBarZ, kFinThreads, !ok)) ok = false;
          float own[MC];
  #pragma unroll
          for (int m = 0; m < MC; ++m) own[m] = 0.0f;
          if (ok) {
            const float* zs = reinterpret_cast<const float*>(smem + L::kZ);
            const float* lut = reinterpret_cast<const float*>(smem + L::kLut);
            float acc4[MC][4];
  #pragma unroll
            for (int m = 0; m < MC; ++m)
  #pragma unroll
              for (int jj = 0; jj < 4; ++jj) acc4[m][jj] = 0.0f;
            for (int w = 0; w < p.RW - w2; ++w) {
              uint32_t word = 0;
  #pragma unroll
              for (int e = 0; e < 16; ++e) word = (e == w) ? uw[e] : word;
              u_word_sum<MC, kLut>(zs, lut, word, w2 + w, p.M, acc4);
            }
  #pragma unroll
            for (int m = 0; m < MC; ++m) own[m] = (acc4[m][0] + acc4[m][1]) + (acc4[m][2] + acc4[m][3]);
          }
          if (named_barrier_or(kBarFin2, kFinThreads, !ok)) {
            ok = false;
            break;
          }
          const float* corr = reinterpret_cast<const float*>(smem + L::kCorr);
  #pragma unroll
          for (int j = 0; j < MC; ++j)
            acc[j] = ((acc[j] + corr[j * kTileRows + row]) + corr[(MC + j) * kTileRows + row]) + own[j];
        }
        uint16_t* yb = p.y + static_cast<size_t>(t) * kTileRows + row;
  #pragma unroll
        for (int j = 0; j < MC; ++j)
          if (j < p.M) yb[static_cast<size_t>(j) * p.N] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
      }
    }
  } else {
    // ---------------------------------------------------------------- CUDA cores
    const int tid = threadIdx.x - kAluWarp0 * 32;      // 0..255
    const int a = warp - kAluWarp0;                     // warp slot 0..7
    if constexpr (!kStream) zero_cache<MC>(smem, nunits, tid, kAluThreads);
    // this CTA's slice of the ranks for z (empty for CTAs outside the sharing set)
    const int zg = shared_work_ctas(p);
    const int i0 = g < zg ? static_cast<int>(static_cast<uint32_t>(g) * static_cast<uint32_t>(p.r) /
                                             static_cast<uint32_t>(zg))
                          : p.r;
    const int i1 = g < zg ? static_cast<int>(static_cast<uint32_t>(g + 1) * static_cast<uint32_t>(p.r) /
                                             static_cast<uint32_t>(zg))
                          : p.r;
    if (p.r > 0) {
      // warm L2 with the sign words this CTA reads later (a hint only)
      const char* vb = reinterpret_cast<const char*>(p.Vbits + static_cast<size_t>(i0) * p.KW);
      const int vlines = ((i1 - i0) * p.KW * 4 + 127) / 128;
      for (int l = tid; l < vlines; l += kAluThreads) prefetch_l2(vb + static_cast<size_t>(l) * 128);
      const int ulines = (kTileRows * p.RW * 4 + 127) / 128;
      for (int seg = 0; seg < nseg; ++seg) {
        const char* ub = reinterpret_cast<const char*>(p.Ubits + static_cast<size_t>(t_first + seg) *
                                                                     kTileRows * p.RW);
        for (int l = tid; l < ulines; l += kAluThreads) prefetch_l2(ub + static_cast<size_t>(l) * 128);
      }
    }
    griddep_wait();
    named_barrier(kBarAlu, kAluThreads);               // cache zeroed before any code lands

    // ---- 1. quantise the activation chunks of every unit of this CTA
    {
      if constexpr (!Cfg<MC>::kGlobalQ) {
        quant_into_cache<MC>(p, smem, u0, nunits, tid, kAluThreads);
      } else {
        constexpr int kImgBytes = QImg<MC>::kBytes, kImgCodes = QImg<MC>::kCodes;
        if constexpr (!kStream) {
          // CTA g < Z (Z = shared_work_ctas) quantises items [g I / Z, (g + 1) I / Z) of the I = 16 KC blocks of
          // 16 rows x 16 elements (rows >= M and blocks past K as zero codes and scales)
          // into the global image, publishes them, and after every CTA has done so
          // copies the chunks of its units into the operand cache
          const uint32_t items = static_cast<uint32_t>(p.KC) * 256u;
          const uint32_t q0 = g < zg ? static_cast<uint32_t>(static_cast<uint64_t>(g) * items / static_cast<uint32_t>(zg)) : 0u;
          const uint32_t q1 = g < zg ? static_cast<uint32_t>(static_cast<uint64_t>(g + 1) * items / static_cast<uint32_t>(zg)) : 0u;
          for (uint32_t it = q0 + static_cast<uint32_t>(tid); it < q1; it += kAluThreads) {
            const int kc = static_cast<int>(it >> 8), m = static_cast<int>((it >> 4) & 15u), blk = static_cast<int>(it & 15u);
            const int kk = kc * kUnitK + blk * 16;
            uint2 codes = make_uint2(0u, 0u);
            uint32_t sc = 0u;
            if (m < p.M && kk < p.K) {
              const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(m) * p.K + kk);
              const uint4 lo = __ldcg(src), hi = __ldcg(src + 1);
              float v[16];
              bf16x16_to_f32(lo, hi, v);
              sc = quant_act_block_fast(v, codes);
            }
            uint8_t* img = p.xq + static_cast<size_t>(kc) * kImgBytes;
            const int j = blk * 8;
            *reinterpret_cast<uint2*>(img + m * 128 + ((((j >> 4) ^ (m & 7)) << 4) | (j & 15))) = codes;
            img[kImgCodes + (blk >> 2) * 64 + m * 4 + (blk & 3)] = static_cast<uint8_t>(sc);
          }
        } else {
          // Streamed classes: items of (chunk, row, 64-element K step), I = 4 kBN KC
          // of them, CTA g < Z taking [g I / Z, (g + 1) I / Z).  An item is four
          // blocks: 32 code bytes (two 16-byte pieces of the swizzled row) and the
          // row's four scales in the step's scale atom (the 32-row class writes the
          // whole 16-byte line, twelve bytes of it zero; at 64 rows the rows below 32
          // zero the line's last eight bytes, which no row uses).  Rows >= M and
          // steps past K are written as zeros.
          constexpr uint32_t kItemsPerChunk = 4u * kBN;
          const uint32_t items = static_cast<uint32_t>(p.KC) * kItemsPerChunk;
          const uint32_t q0 = g < zg ? static_cast<uint32_t>(static_cast<uint64_t>(g) * items / static_cast<uint32_t>(zg)) : 0u;
          const uint32_t q1 = g < zg ? static_cast<uint32_t>(static_cast<uint64_t>(g + 1) * items / static_cast<uint32_t>(zg)) : 0u;
#pragma unroll 1
          for (uint32_t it = q0 + static_cast<uint32_t>(tid); it < q1; it += kAluThreads) {
            const int kc = static_cast<int>(it / kItemsPerChunk);
            const int m = static_cast<int>((it >> 2) & static_cast<uint32_t>(kBN - 1)), st = static_cast<int>(it & 3u);
            const int kk = kc * kUnitK + st * 64;
            const bool live = m < p.M && kk < p.K;
            uint4 xv[8];
            const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(live ? m : 0) * p.K + (live ? kk : 0));
#pragma unroll
            for (int e = 0; e < 8; ++e) xv[e] = live ? __ldcg(src + e) : make_uint4(0u, 0u, 0u, 0u);
            uint32_t cw[8];
            uint32_t sc4 = 0u;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              float v[16];
              bf16x16_to_f32(xv[2 * b], xv[2 * b + 1], v);
              uint2 codes;
              const uint32_t sc = quant_act_block_fast(v, codes);
              cw[2 * b] = codes.x;
              cw[2 * b + 1] = codes.y;
              sc4 |= sc << (8 * b);
            }
            uint8_t* img = p.xq + static_cast<size_t>(kc) * kImgBytes;
            // elements 64 st .. 64 st + 63 = bytes 32 st .. 32 st + 31 of the row: pieces 2 st, 2 st + 1
            *reinterpret_cast<uint4*>(img + m * 128 + (((2 * st) ^ (m & 7)) << 4)) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            *reinterpret_cast<uint4*>(img + m * 128 + (((2 * st + 1) ^ (m & 7)) << 4)) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
            uint8_t* line = img + kImgCodes + st * 512 + (m & 31) * 16;
            if constexpr (kBN == 32) {
              *reinterpret_cast<uint4*>(line) = make_uint4(sc4, 0u, 0u, 0u);
            } else {
              *reinterpret_cast<uint32_t*>(line + 4 * (m >> 5)) = sc4;
              if constexpr (kBN == 64) {
                if (m < 32) *reinterpret_cast<uint2*>(line + 8) = make_uint2(0u, 0u);
              }
            }
          }
          // the producers read the image with bulk copies (the async proxy); this
          // CTA's part is published at once, ahead of the V pieces
          fence_proxy_async_global();
          named_barrier(kBarAlu, kAluThreads);
          if (tid == 0 && !(p.drop & 2)) red_add_release_gpu(p.q_ready, 1u);
        }
        if constexpr (Cfg<MC>::kTensorV) {
          if (p.r > 0) {
            // ---- V side, part 1, on the tensor cores.  Piece (rb, s) = ranks
            // [128 rb, 128 rb + 128) x K atoms [s KA / S, (s + 1) KA / S); CTA g takes
            // pieces g, g + Z, .. (Z = shared_work_ctas).  For each, the partial sums
            //   vpart[rb][s][m][i] = sum_{k in the slice} s_ik x[m][k]
            // come from BF16 MMAs: A = the pieces' sign bits expanded to +-1 (exact,
            // ranks >= r as zero rows), B = the activation rows (rows >= M zero), D in
            // TMEM (lane = rank, column = row).  The buffers are the U side's, unused
            // until z is complete.
            const int RB = (p.r + kTileRows - 1) / kTileRows, KA = p.K / 64;
            const int S = vside_slices(p, RB);
            uint8_t* va = smem + L::kUA;                                  // [kVAtoms][128][128 B]
            uint8_t* vbt = smem + L::kUA + kVAtoms * kTileRows * 128;     // [kVAtoms][16][128 B]
            const int row = tid & (kTileRows - 1), half = tid >> 7;
            const uint32_t idesc_v = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                                     (static_cast<uint32_t>(kTileRows >> 4) << 24);
            int vuses = 0;
            for (int piece = g; g < zg && piece < RB * S; piece += zg) {
              const int rb = piece / S, sl = piece - rb * S;
              const int a0 = static_cast<int>(static_cast<int64_t>(sl) * KA / S);
              const int a1 = static_cast<int>(static_cast<int64_t>(sl + 1) * KA / S);
              const int rank = rb * kTileRows + row;
              // Batches of kVAtoms atoms.  The next batch's sign words and activation
              // pieces are requested before waiting for the current batch's MMAs, so
              // that only the first batch of a piece waits on memory.
              constexpr int kXL = (kVAtoms * kBN * 8 + kAluThreads - 1) / kAluThreads;
              auto load_batch = [&](int b0, uint32_t (&vw)[kVAtoms], uint4 (&xv)[kXL]) {
                const int nb = min(kVAtoms, a1 - b0);
#pragma unroll
                for (int j = 0; j < kVAtoms; ++j)
                  vw[j] = (j < nb && rank < p.r) ? __ldcg(p.Vbits + static_cast<size_t>(rank) * p.KW + 2 * (b0 + j) + half)
                                                 : 0u;
#pragma unroll
                for (int e = 0; e < kXL; ++e) {
                  const int idx = e * kAluThreads + tid;
                  const int j = idx / (kBN * 8), m = (idx >> 3) & (kBN - 1), c = idx & 7;
                  xv[e] = (j < nb && m < p.M)
                              ? __ldcg(reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(m) * p.K + 64 * (b0 + j) + 8 * c))
                              : make_uint4(0u, 0u, 0u, 0u);
                }
              };
              uint32_t vw[kVAtoms];
              uint4 xv[kXL];
              load_batch(a0, vw, xv);
              for (int b0 = a0; b0 < a1; b0 += kVAtoms) {
                const int nb = min(kVAtoms, a1 - b0);
#pragma unroll
                for (int j = 0; j < kVAtoms; ++j) {
                  if (j < nb) {
                    uint8_t* arow = va + j * (kTileRows * 128) + row * 128;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                      uint32_t pk[4];
#pragma unroll
                      for (int t2 = 0; t2 < 4; ++t2) {
                        const int jb = 8 * k + 2 * t2;
                        pk[t2] = (rank < p.r) ? (0x3F803F80u | (((vw[j] >> jb) & 1u) << 15) | (((vw[j] >> (jb + 1)) & 1u) << 31))
                                              : 0u;
                      }
                      const int pc = 4 * half + k;
                      *reinterpret_cast<uint4*>(arow + ((pc ^ (row & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                  }
                }
#pragma unroll
                for (int e = 0; e < kXL; ++e) {
                  const int idx = e * kAluThreads + tid;
                  const int j = idx / (kBN * 8), m = (idx >> 3) & (kBN - 1), c = idx & 7;
                  if (j < nb) *reinterpret_cast<uint4*>(vbt + j * (kBN * 128) + m * 128 + ((c ^ (m & 7)) << 4)) = xv[e];
                }
                fence_proxy_async_smem();
                named_barrier(kBarAlu, kAluThreads);
                if (b0 + kVAtoms < a1) load_batch(b0 + kVAtoms, vw, xv);   // the next batch, in flight during the MMAs
                bool okv = true;
                if (tid == 0) {
                  tc_fence_after();
                  const SmemDesc a_d = make_sdesc(smem_u32(va), 16, 1024, 2);
                  const SmemDesc b_d = make_sdesc(smem_u32(vbt), 16, 1024, 2);
                  for (int j = 0; j < nb; ++j)
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                      tc_mma_bf16(tmem + L::kTmV, sdesc_at(a_d, static_cast<uint32_t>(j) * ((kTileRows * 128) >> 4) + 2 * k4),
                                  sdesc_at(b_d, static_cast<uint32_t>(j) * ((kBN * 128) >> 4) + 2 * k4), idesc_v,
                                  (b0 > a0 || j > 0 || k4 > 0) ? 1u : 0u);
                  tc_commit(vmma_bar);
                  okv = mbar_wait(vmma_bar, vuses & 1, abort_flag);
                }
                ++vuses;
                if (named_barrier_or(kBarAlu, kAluThreads, !okv)) fail(ctl);   // buffers free again
              }
              // the piece's partial sums: warps 0..3 of this group read the four lane
              // quarters of the accumulator
              tc_fence_after();
              // (rank-major, rows contiguous: a thread holds one rank's kBN rows, and
              // the reduce below reads consecutive rows with consecutive threads)
              if (a < 4) {
                const int quarter = warp & 3;
                float4* dst = reinterpret_cast<float4*>(p.vpart + static_cast<size_t>(rb * S + sl) * kBN * kTileRows +
                                                        static_cast<size_t>(quarter * 32 + lane) * kBN);
#pragma unroll
                for (int c0 = 0; c0 < kBN; c0 += 16) {
                  uint32_t v[16];
                  tmem_ld16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + L::kTmV + c0, v);
#pragma unroll
                  for (int j = 0; j < 4; ++j)
                    dst[c0 / 4 + j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                  __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                }
              }
              tc_fence_before();
              named_barrier(kBarAlu, kAluThreads);           // TMEM read before the next piece
            }
          }
        }
        named_barrier(kBarAlu, kAluThreads);
        if constexpr (kStream) {
          // the V pieces' partial sums, behind their own counter (the image went out
          // before them, and the producer waits for it)
          if (p.r > 0) {
            bool okv = true;
            if (tid == 0) {
              red_add_release_gpu(p.v_ready, 1u);             // covers the pieces the CTA wrote
              okv = spin_until_geq(p.v_ready, static_cast<uint32_t>(p.G), ctl);
            }
            if (named_barrier_or(kBarAlu, kAluThreads, !okv)) fail(ctl);
          }
        } else {
          bool okq = true;
          if (tid == 0) {
            if (!(p.drop & 2)) red_add_release_gpu(p.q_ready, 1u);   // covers the items the CTA wrote
            okq = spin_until_geq(p.q_ready, static_cast<uint32_t>(p.G), ctl);
          }
          if (named_barrier_or(kBarAlu, kAluThreads, !okq)) fail(ctl);
          // one round of 16-byte loads: 144 per unit (128 of codes, 16 of scales)
          constexpr int kPer = kImgBytes / 16;
          constexpr int kLd = (L::kMaxUnits * kPer + kAluThreads - 1) / kAluThreads;
          uint4 buf[kLd];
#pragma unroll
          for (int e = 0; e < kLd; ++e) {
            const int idx = e * kAluThreads + tid;
            if (idx < nunits * kPer) {
              const int k = idx / kPer, o = idx - k * kPer;
              const int kc = (u0 + k) % p.KC;
              buf[e] = __ldcg(reinterpret_cast<const uint4*>(p.xq + static_cast<size_t>(kc) * kImgBytes) + o);
            }
          }
#pragma unroll
          for (int e = 0; e < kLd; ++e) {
            const int idx = e * kAluThreads + tid;
            if (idx < nunits * kPer) {
              const int k = idx / kPer, o = idx - k * kPer;
              uint8_t* dst = (o < 128) ? smem + L::kB + k * kBN * 128 + o * 16
                                       : smem + L::kSFB + k * 512 + ((o - 128) >> 2) * 128 + ((o - 128) & 3) * 16;
              *reinterpret_cast<uint4*>(dst) = buf[e];
            }
          }
        }
      }
    }
    if constexpr (!kStream) {
      fence_proxy_async_smem();
      named_barrier(kBarAlu, kAluThreads);
      // activation scales to TMEM: warps 6..9 cover the four lane quarters
      if (a < 4) sfb_to_tmem<MC>(smem, tmem, nunits, static_cast<uint32_t>(warp & 3), lane);
      tc_fence_before();
      named_barrier(kBarAlu, kAluThreads);
      if (tid == 0) mbar_arrive(actr_bar);
    }

    if (p.r > 0) {
      // ---- 2. V side: z for this CTA's rank slice over the whole of K
      float* vred = reinterpret_cast<float*>(smem + L::kVRed);
      if constexpr (!Cfg<MC>::kTensorV) {
        {
          // every warp sums its rows over its K blocks; the warps that split one row's
          // K then add their sums through shared memory
          using VS = VSplit<MC>;
          constexpr int RPW = VS::kRows;
          for (int ig = i0; ig < i1; ig += kRankGroup) {
            const int nr = min(kRankGroup, i1 - ig);
            // alpha of the (row, rank) this thread finishes below, requested with the
            // V-side loads rather than after the reduction
            const float al = (tid < p.M * nr) ? __ldcg(p.alpha + ig + tid % nr) : 0.0f;
            float acc[RPW][kRankGroup];
            vside_rows<MC>(p, ig, nr, a, lane, acc);
  #pragma unroll
            for (int j = 0; j < RPW; ++j)
  #pragma unroll
              for (int i = 0; i < kRankGroup; ++i)
  #pragma unroll
                for (int o = 16; o >= 1; o >>= 1) acc[j][i] += __shfl_xor_sync(0xffffffffu, acc[j][i], o);
            // z for row m, rank ig + i: straight into the U side's B tiles (BF16 high
            // part in row m, the BF16 rounding of the rest in row MC + m, 128-byte
            // swizzled rows) or into the fp32 z scratch
            auto put = [&](int m, int i, float sum) {
              const float zv = __fmul_rn(al, sum);
              if constexpr (Cfg<MC>::kTensorU) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(zv);
                const __nv_bfloat16 lo = __float2bfloat16_rn(zv - __bfloat162float(hi));
                store_ztile(p.ztiles, Layout<MC>::kUN, MC, m, ig + i, hi, lo);
              } else {
                p.z[static_cast<size_t>(m) * p.rpad + ig + i] = zv;
              }
            };
            // the warps of a row group add their sums through shared memory
            static_assert(VS::kSplit > 1, "every row group splits K");
            if (lane == 0) {
  #pragma unroll
              for (int j = 0; j < RPW; ++j)
  #pragma unroll
                for (int i = 0; i < kRankGroup; ++i) vred[(a * RPW + j) * kRankGroup + i] = acc[j][i];
            }
            named_barrier(kBarAlu, kAluThreads);
            if (tid < p.M * nr) {
              const int m = tid / nr, i = tid - m * nr, j = VS::slot_of(m);
              float sum = 0.0f;
  #pragma unroll
              for (int q = 0; q < VS::kSplit; ++q) sum += vred[(VS::warp_of(m, q) * RPW + j) * kRankGroup + i];
              put(m, i, sum);
            }
            named_barrier(kBarAlu, kAluThreads);             // vred is reused by the next group
          }
        }
      } else {
        // ---- V side, part 2: z for this CTA's rank slice [i0, i1), the pieces'
        // partial sums added in a fixed order (slice 0 first), times alpha.  One
        // thread per (rank, row) with the rows of a rank on consecutive threads, so
        // that each of a thread's S loads is part of one contiguous line per warp;
        // all of them are requested before the first is added.
        const int RB = (p.r + kTileRows - 1) / kTileRows;
        const int S = vside_slices(p, RB);
        const int P = (i1 - i0) * p.M;
        for (int base = 0; base < P; base += kAluThreads) {
          const int pair = base + tid;
          const bool act = pair < P;
          const int il = act ? pair / p.M : 0;
          const int i = i0 + il, m = act ? pair - il * p.M : 0;
          const float* src = p.vpart + static_cast<size_t>(i / kTileRows) * S * kBN * kTileRows +
                             static_cast<size_t>(i % kTileRows) * kBN + m;
          const float al = act ? __ldcg(p.alpha + i) : 0.0f;
          float t[kVSliceMax];
#pragma unroll
          for (int q = 0; q < kVSliceMax; ++q)
            t[q] = (act && q < S) ? __ldcg(src + static_cast<size_t>(q) * kBN * kTileRows) : 0.0f;
          float sum = 0.0f;
#pragma unroll
          for (int q = 0; q < kVSliceMax; ++q) sum += t[q];
          if (act) {
            const float zv = __fmul_rn(al, sum);
            const __nv_bfloat16 hi = __float2bfloat16_rn(zv);
            const __nv_bfloat16 lo = __float2bfloat16_rn(zv - __bfloat162float(hi));
            store_ztile(p.ztiles, Layout<MC>::kUN, MC, m, i, hi, lo);
          }
        }
      }
      if constexpr (Cfg<MC>::kTensorU) {
        // the CTA holding the last ranks clears the tiles' tail past r
        if (i1 == p.r && i0 < i1) {
          const int tail = ((p.r + kUChunk - 1) / kUChunk) * kUChunk;
          for (int idx = tid; idx < p.M * (tail - p.r); idx += kAluThreads) {
            const int m = idx / (tail - p.r), i = p.r + idx - m * (tail - p.r);
            store_ztile(p.ztiles, Layout<MC>::kUN, MC, m, i, __float2bfloat16_rn(0.0f), __float2bfloat16_rn(0.0f));
          }
        }
      }
      named_barrier(kBarAlu, kAluThreads);
      if (tid == 0 && !(p.drop & 1)) red_add_release_gpu(p.z_ready, 1u);   // covers the slice the CTA wrote

      if constexpr (Cfg<MC>::kTensorU) {
        // ---- 3. This CTA's share of U z for each of its tiles, on the tensor cores:
        // corr[n][m] = sum_i U[n][i] z[m][i] over the 64-rank chunks [cs0, cs1) of the
        // share, as one BF16 MMA chain.  A tile's contributors split its chunks in
        // proportion to their units of it, so every contributor adds its share to the
        // partial it publishes and the completing CTA only sums partials.  A = the
        // tile's sign bits expanded to +-1 BF16 (exact); B = z split into a BF16 high
        // part and the BF16 rounding of the rest (rows m and MC + m), so the product
        // keeps about 16 bits of z.  The epilogue adds both columns.
        const int nuc = (p.r + kUChunk - 1) / kUChunk;
        const int row = tid & (kTileRows - 1), half = tid >> 7;
        const uint32_t idesc_u = (1u << 4) | (1u << 7) | (1u << 10) |
                                 (static_cast<uint32_t>(L::kUCols >> 3) << 17) |
                                 (static_cast<uint32_t>(kTileRows >> 4) << 24);
        constexpr int kUB = Cfg<MC>::kUBufs;
        // this thread expands word 2 c + half of row `row` for chunk c
        auto load_words = [&](int t, uint32_t (&uw)[kUChunksMax]) {
          const uint32_t* ur = p.Ubits + (static_cast<size_t>(t) * kTileRows + row) * p.RW;
  #pragma unroll
          for (int c = 0; c < kUChunksMax; ++c) {
            const int w = 2 * c + half;
            uw[c] = (w < p.RW) ? __ldcg(ur + w) : 0u;
          }
        };
        uint32_t uw0[kUChunksMax], uw1[kUChunksMax];
        load_words(t_first, uw0);
        if (nseg > 1) load_words(t_first + 1, uw1);
        bool ok = true, zwaited = false;
        int zgroup = -1;                                 // z chunks [zgroup S, zgroup S + S) are in the slots
        int zstagings = 0;                               // thread 0: stagings done (zst_bar's phase)
        int uses0 = 0, uses1 = 0;                        // MMA rounds issued on each A buffer
        // wait (lane 0 of each warp) until the MMAs that last read A buffer `buf` are done
        auto buffer_free = [&](int buf, int uses) {
          if (uses > 0) {
            bool okb = true;
            if (lane == 0) okb = mbar_wait(ubuf_bar(buf), (uses - 1) & 1, abort_flag);
            if (__shfl_sync(0xffffffffu, okb ? 1 : 0, 0) == 0) {
              fail(ctl);
              ok = false;
            }
          }
        };
        // The B tiles of z chunks [grp S, grp S + S) (S = kZSlots) into the slots.  They
        // were written in their final layout by the CTAs that computed z (rows past 2 M
        // only feed output columns nobody reads).  The first time, wait for every slice
        // of z; later (ranks beyond S chunks), for the MMAs still reading the slots.
        auto stage_z = [&](int grp) {
          constexpr int S = Cfg<MC>::kZSlots;
          if (!zwaited) {
            bool okw = true;
            if (tid == 0) okw = spin_until_geq(p.z_ready, static_cast<uint32_t>(p.G), ctl);
            if (named_barrier_or(kBarAlu, kAluThreads, !okw)) {
              fail(ctl);
              ok = false;
            }
            zwaited = true;
          } else if constexpr (S < kUChunksMax) {
            // a reload (only the 32-row class has fewer slots than chunks)
            buffer_free(0, uses0);
            buffer_free(1, uses1);
            named_barrier(kBarAlu, kAluThreads);
          }
          // thread 0 copies the chunks' tiles into the slots with bulk copies (the
          // CTAs that computed z wrote them through the generic proxy) and waits for
          // them: it alone reads the slots (its MMAs); the other threads go on to
          // expand the chunk's signs meanwhile
          if (tid == 0) {
            constexpr uint32_t kChunkBytes = L::kUN * 128;
            const int nch = min(S, nuc - grp * S);
            fence_proxy_async_global();
            mbar_arrive_expect_tx(zst_bar, static_cast<uint32_t>(nch) * kChunkBytes);
            for (int c = 0; c < nch; ++c)
              bulk_load(smem_u32(smem + L::kUZ + c * kChunkBytes),
                        p.ztiles + static_cast<size_t>(grp * S + c) * kChunkBytes, kChunkBytes, zst_bar);
            // (not cut short by an abort: the copies must land before anything else
            // uses the slots or the CTA leaves)
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(zst_bar, zstagings & 1)) {
              if (globaltimer_ns() - t0 > kWaitLimitNs) {
                fail(ctl);
                ok = false;
                break;
              }
            }
            ++zstagings;
          }
          zgroup = grp;
        };
        // The product of segment seg goes to TMEM buffer seg % kUB.  The two sides
        // meet only through mbarriers (bounded waits): ud_bar(b) when a segment's MMAs
        // are done (committed, also for an empty share), uread_bar(b) when the
        // epilogue has read buffer b, which the next product of that buffer waits
        // for.  With two buffers the share of a CTA's second tile runs while the
        // epilogue still finishes its first.
        for (int seg = 0; seg < nseg; ++seg) {
          const int t = t_first + seg;
          const int ub_ = seg % kUB;
          const int ua = max(u0, t * p.KC), ub = min(u1, (t + 1) * p.KC);
          const int cs0 = (ua - t * p.KC) * nuc / p.KC;
          const int cs1 = (ub - t * p.KC) * nuc / p.KC;
          if (seg >= 2) load_words(t_first + seg, uw1);    // segments past the second: load now
          if (seg >= kUB && tid == 0 && !mbar_wait(uread_bar(ub_), ((seg / kUB) - 1) & 1, abort_flag)) {
            fail(ctl);
            ok = false;
          }
          // the classes whose slots hold every chunk stage z once, before their first
          // chunk; the 32-row class cycles larger ranks through its slots below
          if constexpr (Cfg<MC>::kZSlots >= kUChunksMax) {
            if (cs1 > cs0 && zgroup < 0) stage_z(0);
          }
          // chunk pairs in a rolled loop (fully unrolled, the body would make the
          // kernel's code outgrow the instruction cache; the chunk's word is picked
          // out of the registers by compare-and-select, so the word arrays stay in
          // registers), the two A buffers alternating inside a pair.  No
          // CTA-wide barrier per chunk: every thread arrives on the buffer's fill
          // barrier after writing its piece; thread 0 alone waits for the fill, issues
          // the chunk's MMAs and commits them to the buffer's free barrier, which the
          // threads wait on before they write the buffer again.
#pragma unroll 1
          for (int c2 = cs0; c2 < cs1; c2 += 2) {
#pragma unroll
          for (int buf = 0; buf < 2; ++buf) {
            const int c = c2 + buf;
            if (c < cs1) {
              if constexpr (Cfg<MC>::kZSlots < kUChunksMax) {
                if (c / Cfg<MC>::kZSlots != zgroup) stage_z(c / Cfg<MC>::kZSlots);
              }
              int& uses = buf ? uses1 : uses0;
              buffer_free(buf, uses);                      // the MMAs that read this buffer last are done
              uint32_t word = 0u;
  #pragma unroll
              for (int e = 0; e < kUChunksMax; ++e) word = (e == c) ? ((seg == 0) ? uw0[e] : uw1[e]) : word;
              uint8_t* arow = smem + L::kUA + buf * (kTileRows * 128) + row * 128;
  #pragma unroll
              for (int k = 0; k < 4; ++k) {
                uint32_t pk[4];
  #pragma unroll
                for (int t2 = 0; t2 < 4; ++t2) {
                  const int j = 8 * k + 2 * t2;
                  pk[t2] = 0x3F803F80u | (((word >> j) & 1u) << 15) | (((word >> (j + 1)) & 1u) << 31);
                }
                const int piece = 4 * half + k;
                *reinterpret_cast<uint4*>(arow + ((piece ^ (row & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              }
              fence_proxy_async_smem();
              mbar_arrive(ufull_bar(buf));
              if (tid == 0) {
                if (mbar_wait(ufull_bar(buf), uses & 1, abort_flag)) {
                  tc_fence_after();
                  const SmemDesc a_d = make_sdesc(smem_u32(smem + L::kUA + buf * (kTileRows * 128)), 16, 1024, 2);
                  const SmemDesc b_d =
                      make_sdesc(smem_u32(smem + L::kUZ + (c % Cfg<MC>::kZSlots) * L::kUN * 128), 16, 1024, 2);
                  const uint32_t d_u = tmem + L::kTmU + static_cast<uint32_t>(ub_ * L::kUCols);
  #pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    tc_mma_bf16(d_u, sdesc_at(a_d, 2 * j), sdesc_at(b_d, 2 * j), idesc_u, (c > cs0 || j > 0) ? 1u : 0u);
                    // the low parts (rows MC .. 2 MC - 1 of the tile) into the same columns
                    if constexpr (Cfg<MC>::kUSum)
                      tc_mma_bf16(d_u, sdesc_at(a_d, 2 * j), sdesc_at(b_d, (MC * 128 >> 4) + 2 * j), idesc_u, 1u);
                  }
                  tc_commit(ubuf_bar(buf));
                } else {
                  fail(ctl);
                  ok = false;
                }
              }
              ++uses;
            }
          }
          }
          if (tid == 0) tc_commit(ud_bar(ub_));             // arrives at once if nothing was issued
        }
        // the U-side MMAs must be finished before TMEM is freed (bounded wait)
        if (tid == 0 && uses0 + uses1 > 0) {
          tc_commit(ubuf_bar(0));
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(ubuf_bar(0), uses0 & 1)) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
              record_error(p.status, kDevErrTimeout);
              break;
            }
          }
        }
      } else {
        // ---- 3. U side of every tile this CTA completes
        float* zs = reinterpret_cast<float*>(smem + L::kZ);
        float* corr = reinterpret_cast<float*>(smem + L::kCorr);
        bool ok = true, staged = false;
        // thread (row, half) sums ranks [32 wa, 32 wb) of weight row `row`: the first
        // and second thirds of the words (the epilogue threads take the last third);
        // the sign words of the first two tiles are requested now, before z is complete
        const int row = tid & (kTileRows - 1), half = tid >> 7;
        const int w1 = p.RW / 3, w2 = 2 * p.RW / 3;
        const int wa = half ? w1 : 0, wb = half ? w2 : w1;
        auto load_words = [&](int t, uint32_t (&uw)[16]) {
          const uint32_t* ur = p.Ubits + (static_cast<size_t>(t) * kTileRows + row) * p.RW;
  #pragma unroll
          for (int w = 0; w < 16; ++w) uw[w] = (wa + w < wb) ? __ldcg(ur + wa + w) : 0u;
        };
        uint32_t uw0[16], uw1[16];
        load_words(t_first, uw0);
        if (nseg > 1) load_words(t_first + 1, uw1);
        for (int seg = 0; seg < nseg; ++seg) {
          if (named_barrier_or(kBarFin, kFinThreads, !ok)) {
            ok = false;
            break;
          }
          if (!fin_flag[seg]) continue;
          const int t = t_first + seg;
          if (!staged) {
            bool okw = true;
            if (tid == 0) okw = spin_until_geq(p.z_ready, static_cast<uint32_t>(p.G), ctl);
            if (named_barrier_or(kBarAlu, kAluThreads, !okw)) {
              fail(ctl);
              ok = false;
            } else {
              const int span = 32 * p.RW;
              for (int idx = tid; idx < p.M * span; idx += kAluThreads) {
                const int m = idx / span, i = idx - m * span;
                zs[m * kMaxRanks + i] = (i < p.r) ? __ldcg(p.z + static_cast<size_t>(m) * p.rpad + i) : 0.0f;
              }
              named_barrier(kBarAlu, kAluThreads);
              if constexpr (kLut) {
                build_z_table<MC>(zs, reinterpret_cast<float*>(smem + L::kLut), p.M, p.RW, tid, kAluThreads);
                named_barrier(kBarAlu, kAluThreads);
              }
              staged = true;
            }
          }
          if (named_barrier_or(kBarZ, kFinThreads, !ok)) ok = false;   // z staged for the epilogue's third
          if (ok) {
            if (seg >= 2) load_words(t, uw1);            // segments past the second: load now
            // four interleaved sums per row: a dependency chain a quarter as long
            float acc4[MC][4];
  #pragma unroll
            for (int m = 0; m < MC; ++m)
  #pragma unroll
              for (int jj = 0; jj < 4; ++jj) acc4[m][jj] = 0.0f;
            const float* lut = reinterpret_cast<const float*>(smem + L::kLut);
            for (int w = 0; w < wb - wa; ++w) {
              uint32_t word = 0;
  #pragma unroll
              for (int e = 0; e < 16; ++e) word = (e == w) ? ((seg == 0) ? uw0[e] : uw1[e]) : word;
              u_word_sum<MC, kLut>(zs, lut, word, wa + w, p.M, acc4);
            }
            float acc[MC];
  #pragma unroll
            for (int m = 0; m < MC; ++m) acc[m] = (acc4[m][0] + acc4[m][1]) + (acc4[m][2] + acc4[m][3]);
  #pragma unroll
            for (int m = 0; m < MC; ++m) corr[(half * MC + m) * kTileRows + row] = acc[m];
          }
          if (named_barrier_or(kBarFin2, kFinThreads, !ok)) {
            ok = false;
            break;
          }
        }
      }
    }
    // This CTA waits on no grid counter any more (in the streamed class its producer
    // has passed the image wait too): count it done.  The last CTA resets every
    // counter for the next call, which reads them only after its wait on this
    // kernel.  Counted here, the atomic runs while the epilogue finishes, off its
    // path; calls that use no counter (r = 0 below 8 rows) count nothing.
    if (p.r > 0 || Cfg<MC>::kGlobalQ) {
      if (tid == 0) {
        if constexpr (kStream) {
          if (!mbar_wait(qpass_bar, 0, abort_flag)) fail(ctl);
        }
        const uint32_t old = atomicAdd(p.done, 1u);
        if (old == static_cast<uint32_t>(p.G - 1)) {
          atomicExch(p.z_ready, 0u);
          atomicExch(p.q_ready, 0u);
          atomicExch(p.v_ready, 0u);
          atomicExch(p.done, 0u);
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  // Each warp reports once it no longer touches TMEM or shared memory; warp 1
  // frees TMEM after all of them (bounded wait).
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

}  // namespace decode
}  // namespace biloco

namespace biloco {

static_assert(decode::kRowsMax == kDecodeMaxRows, "host and kernel limits agree");

template <int MC>
cudaError_t launch_decode(const CUtensorMap& tw, const DecodeParams& dp, cudaStream_t s,
                          const LaunchOpts& o) {
  // the table form exists for the classes with the CUDA-core U side (1-2 rows)
  constexpr bool kHasLut = !decode::Cfg<MC>::kTensorU;
  if constexpr (kHasLut) {
    if (dp.lut) {
      static KernelSetup ks_lut;
      return launch_resident(ks_lut, decode::decode_kernel<MC, true>, dp.G, decode::kThreads,
                             decode::Layout<MC>::kAlloc, s, o, tw, dp);
    }
  }
  static_assert(decode_class(MC) == MC && decode::Cfg<MC>::kBN == decode_bn(MC) &&
                    decode::Cfg<MC>::kMaxUnits == decode_max_units(MC) &&
                    decode::QImg<MC>::kBytes == decode_img_bytes(MC) &&
                    decode::Layout<MC>::kUN * 128 * decode::kUChunksMax <= decode_ztile_bytes(MC),
                "host and kernel views of the batch class agree");
  static KernelSetup ks;
  return launch_resident(ks, decode::decode_kernel<MC, false>, dp.G, decode::kThreads, decode::Layout<MC>::kAlloc, s,
                         o, tw, dp);
}

}  // namespace biloco
