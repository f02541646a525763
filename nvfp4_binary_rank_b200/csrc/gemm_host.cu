// Host side of the fused GEMM: shape decomposition, scratch, tensor maps and the
// choice of kernel instance.
#include <algorithm>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/biloco.h"
#include "decode_launch.h"
#include "fused_launch.h"
#include "fused_params.h"
#include "internal.h"

namespace biloco {

namespace {

constexpr int kTileRows = 128;
constexpr int kUnitK = 256;
constexpr int kSfBytes = 2048;
constexpr int kRB = 16;
constexpr int kSubK = 256;
constexpr int kXWords = 8;
constexpr int kVStageRanks = 64;
constexpr int kInKernelQuantMaxM = 8;


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

// 2-D tensor without swizzle: [rows][inner elements of elem_bytes], box [box_rows][box_inner].
bool make_tmap_plain(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t elem_bytes,
                     uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


int pick_bn(int M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

cudaError_t launch_for(int M, const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& txs,
                       const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, const LaunchOpts& o) {
  if (M <= 1) return launch_fused<16, 5, 1>(tw, tx, txs, tv, fp, s, o);
  if (M <= 2) return launch_fused<16, 5, 2>(tw, tx, txs, tv, fp, s, o);
  if (M <= 4) return launch_fused<16, 5, 4>(tw, tx, txs, tv, fp, s, o);
  if (M <= 8) return launch_fused<16, 5, 8>(tw, tx, txs, tv, fp, s, o);
  if (M <= 16) return launch_fused<16, 5, 16>(tw, tx, txs, tv, fp, s, o);
  if (M <= 32) return launch_fused<32, 3, 32>(tw, tx, txs, tv, fp, s, o);
  if (M <= 64) return launch_fused<64, 4, 32>(tw, tx, txs, tv, fp, s, o);
  return launch_fused<128, 3, 32>(tw, tx, txs, tv, fp, s, o);
}

// A launch error as a library status: a grid that cannot be resident at once is
// reported as such, anything else as a CUDA failure.
int launch_status(cudaError_t e) {
  if (e == cudaSuccess) return BILOCO_OK;
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    cudaGetLastError();
    return BILOCO_ERR_RESIDENCY;
  }
  return BILOCO_ERR_CUDA;
}

}  // namespace

// AUTO: the shared-z schedule.  Timed on a B200 over N = 5120, K in {5120, 13824},
// M in {1, 2, 4, 8, 16, 32, 64, 128}, r in {32, 128, 512, 1024} (CUDA-graph replay,
// weight copies past L2), it was the faster one at every point, by 1.3x (M = 128,
// r = 32) to 15x (M = 1, r = 512): computing z once and exchanging it costs less
// than every CTA recomputing the ranks its tiles need over the whole of K.
int resolve_mode(int M, int N, int K, int r, int requested) {
  (void)M; (void)N; (void)K; (void)r;
  if (requested == BILOCO_MODE_SHARED_Z || requested == BILOCO_MODE_LOCAL_Z) return requested;
  return BILOCO_MODE_SHARED_Z;
}

// AUTO: the signed-sum table of z for 1-2 rows (the decode kernel's CUDA-core U
// side; every other shape ignores the setting).  Timed on a B200 at N = K = 5120,
// M = 1 (CUDA-graph replay, weight copies past L2) it was faster at r = 512 (12.62
// vs 13.14 us per call) and r = 1024 (19.69 vs 21.06), and equal at r = 128.
int resolve_arith(int M, int N, int K, int r, int requested) {
  (void)N; (void)K; (void)r;
  if (requested == BILOCO_CORR_SIGNS || requested == BILOCO_CORR_LUT) return requested;
  return M <= 2 ? BILOCO_CORR_LUT : BILOCO_CORR_SIGNS;
}

int gemm_kernel_count_for(const GemmArgs& a) {
  const GemmPlan p = plan_gemm(a);
  return (p.decode || p.inq) ? 1 : 2;
}

GemmPlan plan_gemm(const GemmArgs& a) {
  const int M = a.M, N = a.N, K = a.K, r = a.r;
  GemmPlan p;
  p.KC = (K + kUnitK - 1) / kUnitK;
  p.T = N / kTileRows;
  p.U = p.T * p.KC;
  p.G = std::min(num_sms(), p.U);
  p.KW = K / 32;
  p.rpad = std::max((r + kRB - 1) / kRB, 1) * kRB;
  p.BN = pick_bn(M);
  p.bxr = p.BN <= 16 ? 16 : 32;
  p.inq = M <= kInKernelQuantMaxM;
  p.zdirect = (M <= 2) || (M * p.KC <= 64);
  p.shared_z = r > 0 && a.mode == BILOCO_MODE_SHARED_Z;
  p.unit_alu = p.inq || p.shared_z;
  const int ranks_per_tile = (r + p.T - 1) / p.T;
  p.fast = p.unit_alu && p.BN <= 32 && K % 128 == 0 && (!p.shared_z || ranks_per_tile <= kVStageRanks);

  // batches up to 128 rows take the decode kernel when a CTA's units fit its class
  // (ceil(U / G) units: the operand cache up to 16 rows, 64 units when streamed)
  p.decode = M <= kDecodeMaxRows && (r == 0 || p.shared_z) && (p.U + p.G - 1) / p.G <= decode_max_units(M);
  // The 128-row class takes at most about 2.5 CTAs per weight tile: its split-K
  // partials are 64 KB per contributor, and fewer contributors per tile shorten the
  // final sums more than the lost SMs slow the weight stream.  Timed on a B200
  // (N, K, r; us per call, 148 -> capped grid): 5120, 5120, 512: 61.0 -> 48.1;
  // 5120, 5120, 0: 36.8 -> 32.3; 5120, 13824, 512: 68.7 -> 60.1; M = 96, 5120,
  // 5120, 256: 50.1 -> 38.4; 5120, 5120, 1024: 74.0 -> 75.5.  With many tiles
  // (N = 13824) the cap does not apply; a fixed 100 CTAs there was slower.
  if (p.decode && decode_class(M) == 128) {
    const int g = std::max(1, 5 * p.T / 2);
    if (g < p.G && (p.U + g - 1) / g <= decode_max_units(M)) p.G = g;
  }

  ScratchNeed& need = p.need;
  if (p.decode) {
    const size_t bn = static_cast<size_t>(decode_bn(M));
    need.act_fp4 = static_cast<size_t>(p.KC) * decode_img_bytes(M);   // the activation image (8+ rows)
    need.act_sf = 16;
    // the decode kernel's z tiles, then the V-side partial sums: one bn x 128 block
    // per piece, max(G, rank blocks) pieces at most
    const size_t vpieces = static_cast<size_t>(std::max(p.G, (r + kTileRows - 1) / kTileRows));
    need.zpart = static_cast<size_t>(decode_ztile_bytes(M)) + vpieces * bn * kTileRows * 4;
    need.zfin = r ? static_cast<size_t>(M) * p.rpad * 4 : 16;
    need.slots = static_cast<size_t>(2 * p.G) * bn * kTileRows * 4;
    need.counter_words = 4 + static_cast<size_t>(p.T);   // z, done, tickets, q and v counters
    return p;
  }
  need.act_fp4 = p.inq ? 16 : static_cast<size_t>(M) * K / 2;
  need.act_sf = p.inq ? 16 : static_cast<size_t>(p.KC) * kSfBytes;
  need.zpart = r ? static_cast<size_t>(p.KC) * M * p.rpad * 4 : 16;
  need.zfin = r ? static_cast<size_t>(M) * p.rpad * 4 : 16;
  need.slots = static_cast<size_t>(2 * p.G) * p.BN * kTileRows * 4;
  need.counter_words = 2 + 2 * static_cast<size_t>(p.T);
  return p;
}

int run_gemm(const GemmArgs& a, cudaStream_t s) {
  const GemmPlan p = plan_gemm(a);
  Scratch* sc = get_scratch(s, p.need);
  if (!sc) return BILOCO_ERR_NOMEM;
  return launch_gemm(a, p, *sc, s);
}

int launch_gemm(const GemmArgs& a, const GemmPlan& p, const Scratch& scr, cudaStream_t s) {
  const int M = a.M, N = a.N, K = a.K, r = a.r;
  const int KC = p.KC, T = p.T, U = p.U, G = p.G, KW = p.KW, rpad = p.rpad, BN = p.BN;
  const bool inq = p.inq, zdirect = p.zdirect, shared_z = p.shared_z, unit_alu = p.unit_alu;
  const bool fast = p.fast;
  const Scratch* sc = &scr;

  cudaError_t e = cudaSuccess;
  if (p.decode) {
    CUtensorMap tw;
    if (!make_tmap(&tw, a.W_fp4, static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(N), kTileRows))
      return BILOCO_ERR_CUDA;
    DecodeParams dp = {};
    dp.w_sf = a.W_sf;
    dp.gscale = a.gscale;
    dp.Ubits = a.Ubits;
    dp.Vbits = a.Vbits;
    dp.alpha = a.alpha;
    dp.x = a.x;
    dp.y = a.y;
    dp.z = sc->zfin;
    dp.ztiles = reinterpret_cast<uint8_t*>(sc->zpart);
    dp.vpart = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sc->zpart) + decode_ztile_bytes(M));
    dp.slots = sc->slots;
    dp.z_ready = sc->counters;
    dp.done = sc->counters + 1;
    dp.tickets = sc->counters + 2;
    dp.q_ready = sc->counters + 2 + T;
    dp.v_ready = sc->counters + 3 + T;
    dp.xq = sc->act_fp4;
    dp.status = sc->status;
    dp.M = M; dp.N = N; dp.K = K; dp.r = r;
    dp.KC = KC; dp.T = T; dp.U = U; dp.G = G; dp.KW = KW;
    dp.RW = (r + 31) / 32;
    dp.rpad = rpad;
    dp.drop = a.drop;
    dp.lut = (a.arith == BILOCO_CORR_LUT) ? 1 : 0;
    const LaunchOpts o = current_launch_opts();
    if (M <= 1) e = launch_decode<1>(tw, dp, s, o);
    else if (M <= 2) e = launch_decode<2>(tw, dp, s, o);
    else if (M <= 4) e = launch_decode<4>(tw, dp, s, o);
    else if (M <= 8) e = launch_decode<8>(tw, dp, s, o);
    else if (M <= 16) e = launch_decode<16>(tw, dp, s, o);
    else if (M <= 32) e = launch_decode<32>(tw, dp, s, o);
    else if (M <= 64) e = launch_decode<64>(tw, dp, s, o);
    else e = launch_decode<128>(tw, dp, s, o);
    return launch_status(e);
  }
  if (!inq) {
    e = launch_prep_act(a.x, M, K, sc->act_fp4, sc->act_sf, s);
    if (e != cudaSuccess) return BILOCO_ERR_CUDA;
  }

  CUtensorMap tw, tx, txs, tv;
  if (!make_tmap(&tw, a.W_fp4, static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(N), kTileRows))
    return BILOCO_ERR_CUDA;
  if (inq) {
    tx = tw;                                           // not read when quantising in-kernel
  } else if (!make_tmap(&tx, sc->act_fp4, static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(M), BN)) {
    return BILOCO_ERR_CUDA;
  }
  const int bxr = p.bxr;
  txs = tw;
  tv = tw;
  if (fast) {
    if (!make_tmap_plain(&txs, a.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, static_cast<uint64_t>(K),
                         static_cast<uint64_t>(M), kSubK, static_cast<uint32_t>(bxr)))
      return BILOCO_ERR_CUDA;
    if (shared_z && !make_tmap_plain(&tv, a.Vbits, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4,
                                     static_cast<uint64_t>(KW), static_cast<uint64_t>(r), kXWords,
                                     kVStageRanks))
      return BILOCO_ERR_CUDA;
  }

  FusedParams fp = {};
  fp.w_sf = a.W_sf;
  fp.x_sf = sc->act_sf;
  fp.gscale = a.gscale;
  fp.Ubits = a.Ubits;
  fp.Vbits = a.Vbits;
  fp.alpha = a.alpha;
  fp.x = a.x;
  fp.y = a.y;
  fp.zpart = sc->zpart;
  fp.zfin = sc->zfin;
  fp.slots = sc->slots;
  fp.z_ready = sc->counters;
  fp.z_seen = sc->counters + 1;
  fp.tickets = sc->counters + 2;
  fp.vtick = sc->counters + 2 + T;
  fp.status = sc->status;
  fp.M = M; fp.N = N; fp.K = K; fp.r = r;
  fp.KC = KC; fp.T = T; fp.U = U; fp.G = G; fp.KW = KW;
  fp.rpad = rpad;
  fp.RW = (r + 31) / 32;
  fp.mode = a.mode;
  fp.inq = inq ? 1 : 0;
  fp.zdirect = zdirect ? 1 : 0;
  fp.fast = fast ? 1 : 0;
  fp.unit_alu = unit_alu ? 1 : 0;
  fp.bxr = bxr;

  // launched for programmatic overlap with the kernel before it (the activation
  // quantiser, or the previous call)
  fp.drop = a.drop;
  e = launch_for(M, tw, tx, txs, tv, fp, s, current_launch_opts());
  return launch_status(e);
}

}  // namespace biloco
