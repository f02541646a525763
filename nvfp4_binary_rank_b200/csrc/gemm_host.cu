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
                       const CUtensorMap& tv, const FusedParams& fp, cudaStream_t s, bool pdl) {
  if (M <= 1) return launch_fused_16_1(tw, tx, txs, tv, fp, s, pdl);
  if (M <= 2) return launch_fused_16_2(tw, tx, txs, tv, fp, s, pdl);
  if (M <= 4) return launch_fused_16_4(tw, tx, txs, tv, fp, s, pdl);
  if (M <= 8) return launch_fused_16_8(tw, tx, txs, tv, fp, s, pdl);
  if (M <= 16) return launch_fused_16_16(tw, tx, txs, tv, fp, s, pdl);
  if (M <= 32) return launch_fused_32_32(tw, tx, txs, tv, fp, s, pdl);
  if (M <= 64) return launch_fused_64_32(tw, tx, txs, tv, fp, s, pdl);
  return launch_fused_128_32(tw, tx, txs, tv, fp, s, pdl);
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

  // decode batches take the decode kernel when its operand cache holds every
  // unit of a CTA (ceil(U / G) units)
  p.decode = M <= kDecodeMaxRows && (r == 0 || p.shared_z) && (p.U + p.G - 1) / p.G <= kDecodeMaxUnits;

  ScratchNeed& need = p.need;
  if (p.decode) {
    need.act_fp4 = static_cast<size_t>(p.KC) * kDecodeQImgBytes;   // the activation image (8+ rows)
    need.act_sf = 16;
    // the decode kernel's z tiles, then the V-side partial sums: one 16 x 128 block
    // per piece, max(G, rank blocks) pieces at most
    const size_t vpieces = static_cast<size_t>(std::max(p.G, (r + kTileRows - 1) / kTileRows));
    need.zpart = 16 * 32 * 128 + vpieces * kDecodeMaxRows * kTileRows * 4;
    need.zfin = r ? static_cast<size_t>(M) * p.rpad * 4 : 16;
    need.slots = static_cast<size_t>(2 * p.G) * kDecodeMaxRows * kTileRows * 4;
    need.counter_words = 4 + 2 * static_cast<size_t>(p.T);   // z, tickets, q counters
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
    dp.vpart = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sc->zpart) + 16 * 32 * 128);
    dp.slots = sc->slots;
    dp.z_ready = sc->counters;
    dp.z_seen = sc->counters + 1;
    dp.tickets = sc->counters + 2;
    dp.q_ready = sc->counters + 2 + T;
    dp.q_seen = sc->counters + 3 + T;
    dp.xq = sc->act_fp4;
    dp.status = sc->status;
    dp.M = M; dp.N = N; dp.K = K; dp.r = r;
    dp.KC = KC; dp.T = T; dp.U = U; dp.G = G; dp.KW = KW;
    dp.RW = (r + 31) / 32;
    dp.rpad = rpad;
    if (M <= 1) e = launch_decode_1(tw, dp, s);
    else if (M <= 2) e = launch_decode_2(tw, dp, s);
    else if (M <= 4) e = launch_decode_4(tw, dp, s);
    else if (M <= 8) e = launch_decode_8(tw, dp, s);
    else e = launch_decode_16(tw, dp, s);
    return e == cudaSuccess ? BILOCO_OK : BILOCO_ERR_CUDA;
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

  // always launched for programmatic overlap with the kernel before it (the
  // activation quantiser, or the previous call)
  e = launch_for(M, tw, tx, txs, tv, fp, s, true);
  return e == cudaSuccess ? BILOCO_OK : BILOCO_ERR_CUDA;
}

}  // namespace biloco
