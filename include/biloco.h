/*
 * biloco.h - C ABI of libbiloco.so: the fused NVFP4 GEMM with a binary-sign
 * low-rank correction on one B200 (sm_100a).
 *
 * The operation (BiLoCo README, github jindavid/BiLoCo, sections "Decomposition"
 * and "Kernel"): a weight is split as W ~= U diag(alpha) V^T + R with sign
 * factors U in {+-1}^{N x r}, V in {+-1}^{K x r} and an NVFP4 residual R, and the
 * layer output is
 *
 *     y = FP4(x) FP4(R)^T + sum_i alpha_i (x . v_i) u_i            (BF16 out)
 *
 * computed in one fused launch: the FP4 product on the tensor cores, the sign
 * correction on the CUDA cores.
 *
 * Conventions for every call
 *   - Pointers are DEVICE pointers owned by the caller unless stated otherwise;
 *     the library never frees them.  Calls are asynchronous and ordered on
 *     `stream` (NULL = the legacy default stream).
 *   - Return value: BILOCO_OK (0) or a negative BILOCO_ERR_* code.  Argument,
 *     shape and alignment errors are detected on the host before anything is
 *     launched.  Errors raised inside a kernel (a bounded wait that expired)
 *     are reported by biloco_last_error().
 *   - Row-major everywhere.  "x_bf16" and "y_bf16" point to IEEE bfloat16 data.
 *   - The library keeps scratch memory per (device, stream), allocated on first
 *     use and grown when a larger shape arrives; biloco_shutdown() frees it.
 *     Calls on one stream must not run concurrently with each other from
 *     several host threads.
 *
 * NVFP4 format used throughout (E2M1 elements, one E4M3 scale per 16 elements
 * along K):
 *   - element codes: 4-bit E2M1, grid {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6};
 *     element 2j of a row in the low nibble of byte j; a zero is always code 0.
 *   - scale s = E4M3(amax_block / 6) for activations (no tensor scale), and
 *     s = E4M3(amax_block / (6 g)) for the weight with g = amax(|R|) / 2688
 *     (g = 1 if R == 0); E4M3 rounding is nearest-even with saturation at 448.
 *   - code = E2M1(v / S), S = s (activation) or S = s * g (weight), FP32
 *     division rounded to nearest, E2M1 nearest with ties to the even code,
 *     |v/S| > 6 saturates; if S == 0 the block's codes are 0.
 *
 * Sign packing: bit 1 = -1, bit 0 = +1 (a zero counts as +1), least significant
 * bit first in little-endian uint32 words; unused tail bits are 0.
 */
#ifndef BILOCO_H
#define BILOCO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st *biloco_stream_t;

enum {
  BILOCO_OK = 0,
  BILOCO_ERR_ARG = -1,     /* NULL pointer where one is required, negative size  */
  BILOCO_ERR_SHAPE = -2,   /* shape outside the supported limits                  */
  BILOCO_ERR_ALIGN = -3,   /* pointer not 16-byte aligned                         */
  BILOCO_ERR_CUDA = -4,    /* a CUDA runtime call or a kernel launch failed       */
  BILOCO_ERR_TIMEOUT = -5, /* a bounded device-side wait expired (see last_error) */
  BILOCO_ERR_NOMEM = -6,   /* library scratch could not be allocated              */
  BILOCO_ERR_DEVICE = -7,  /* the current device is not an sm_100 GPU             */
  BILOCO_ERR_RESIDENCY = -8 /* the GEMM grid cannot be resident on the GPU at once  */
};

/* Size limits of biloco_gemm.  The weight is cut into (N/128) * ceil(K/256) units
 * of 128 rows x 256 elements; at most BILOCO_MAX_UNITS of them (16.7 M units is
 * 275 GB of codes, more than any single GPU holds). */
#define BILOCO_MAX_M 128
#define BILOCO_MAX_R 1024
#define BILOCO_MAX_N (1 << 24)
#define BILOCO_MAX_UNITS (1 << 24)

/* z schedules of biloco_gemm (BiLoCo README, section "Kernel", mode table):
 *   BILOCO_MODE_AUTO       pick per (M, r, K) from a measured table
 *   BILOCO_MODE_SHARED_Z   every CTA computes one slice of z = alpha . (V^T x) at
 *                          entry and publishes it to scratch behind an arrival
 *                          counter; the GEMM tiles read z in their epilogue
 *                          (the "side CTAs + arrival flag" schedule)
 *   BILOCO_MODE_LOCAL_Z    every CTA computes, at entry, the part of z that its own
 *                          tiles need; no cross-CTA exchange (the "every CTA computes
 *                          the correction at kernel entry" schedule) */
enum { BILOCO_MODE_AUTO = 0, BILOCO_MODE_SHARED_Z = 1, BILOCO_MODE_LOCAL_Z = 2 };

/*
 * biloco_quant_act - BF16 activation -> NVFP4 codes and E4M3 block scales.
 * (BiLoCo README, section "Kernel": the activation enters the FP4 product as
 * NVFP4 codes A plus block scales A_sf; no tensor scale is passed.)
 *
 *   x_bf16  [M][K] bfloat16, 16-byte aligned
 *   M, K    M >= 1, K >= 16, K % 16 == 0
 *   x_fp4   out [M][K/2] bytes (two codes per byte)
 *   x_sf    out [M][K/16] E4M3 bytes
 * Bit-exact with the rules in the header comment.
 */
int biloco_quant_act(const void *x_bf16, int M, int K, uint8_t *x_fp4, uint8_t *x_sf,
                     biloco_stream_t stream);

/*
 * biloco_pack_signs - +-1 matrix -> packed sign words.
 * (BiLoCo README, section "Kernel": pack_signs(V.T), pack_signs(U.T).)
 *
 *   S     [rows][cols] float; bit = 1 where S < 0
 *   bits  out [rows][ceil(cols/32)] uint32, bit j of word w <-> column 32w + j
 * For the GEMM: Vbits = pack_signs(V^T) with rows = r, cols = K, and
 * Ubits = pack_signs(U) with rows = N, cols = r.
 */
int biloco_pack_signs(const float *S, int rows, int cols, uint32_t *bits,
                      biloco_stream_t stream);

/*
 * biloco_pack_weight - FP32 residual R -> NVFP4 codes, block scales in the
 * GEMM's tile layout, and the FP32 tensor scale.
 * (BiLoCo README, section "Decomposition": R is quantised to NVFP4; section
 * "Kernel": W_fp4, W_sf, w_global_scale.)
 *
 *   R       [N][K] float, 16-byte aligned; N % 128 == 0, K % 64 == 0
 *   W_fp4   out [N][K/2] bytes, 16-byte aligned
 *   W_sf    out biloco_weight_sf_bytes(N, K) bytes, 16-byte aligned, tile layout:
 *           the scale of weight row n and 16-element block b (k = 16b .. 16b+15)
 *           sits at byte
 *              ((((n/128) * KC + b/16) * 4 + (b%16)/4) * 512)
 *              + (n%32) * 16 + ((n%128)/32) * 4 + (b%4)
 *           with KC = ceil(K/256); bytes past K are zero.
 *   gscale  out device float, the tensor scale g
 * Runs three kernels; needs no host synchronisation.
 */
int biloco_pack_weight(const float *R, int N, int K, uint8_t *W_fp4, uint8_t *W_sf,
                       float *gscale, biloco_stream_t stream);

/* Bytes of the weight scale array: N * ceil(K/256) * 16. */
size_t biloco_weight_sf_bytes(int N, int K);

/*
 * biloco_decompose - W ~= U diag(alpha) V^T + R with binary sign factors.
 * (BiLoCo README, section "Decomposition": each rank-one term starts from random
 * signs and alternates u = sign(R v), v = sign(R^T u) for T steps, takes the
 * Frobenius-optimal coefficient and deflates the residual; after all r terms the
 * coefficients are refit jointly by least squares for the fixed signs.)
 *
 *   W          [N][K] float, 4-byte aligned, not modified (R_out may alias it)
 *   r, T       0 <= r <= 1024 terms, T >= 1 alternations per term
 *   v0bits     [r][ceil(K/32)] uint32: the start signs of each term's v, packed
 *              like pack_signs (bit 1 = -1); the caller draws them (the README
 *              seeds a generator); may be NULL when r == 0
 *   Ubits      out [N][ceil(r/32)] uint32 = pack_signs(U)    (biloco_gemm's Ubits)
 *   Vbits      out [r][ceil(K/32)] uint32 = pack_signs(V^T)  (biloco_gemm's Vbits)
 *   alpha      out [r] float, the refit coefficients
 *   R_out      out [N][K] float, W - U diag(alpha) V^T (feed it to
 *              biloco_pack_weight for the NVFP4 residual)
 *   workspace  device memory of at least biloco_decompose_workspace_bytes(N, K, r)
 *              bytes, 256-byte aligned, owned by the caller (it holds the FP64
 *              residual: about 8 N K bytes)
 * Every sign is decided on an FP64 sum, with sign(0) = +1; alpha_i = u^T R v /
 * (N K) for the current residual; the refit solves the normal equations
 * (u_i . u_j)(v_i . v_j) alpha = u_i^T W v_i by conjugate gradients (the
 * minimum-norm solution if terms repeat).  Asynchronous on `stream`; about
 * r (3 T + 2) kernel launches.  Errors: BILOCO_ERR_ARG (NULL pointer, workspace
 * too small), _SHAPE (N, K < 1, r out of range, T < 1, N K > 2^31), _ALIGN,
 * _DEVICE, _CUDA.
 */
size_t biloco_decompose_workspace_bytes(int N, int K, int r);
int biloco_decompose(const float *W, int N, int K, int r, int T, const uint32_t *v0bits,
                     uint32_t *Ubits, uint32_t *Vbits, float *alpha, float *R_out,
                     void *workspace, size_t workspace_bytes, biloco_stream_t stream);

/*
 * biloco_gemm - y = FP4(x) FP4(R)^T + sum_i alpha_i (x . v_i) u_i, in BF16.
 * (BiLoCo README, section "Kernel": one launch for decode batches; the FP4 GEMM
 * on tensor cores, z = alpha . (V x) on CUDA cores from bit-packed V, U z expanded
 * in the GEMM epilogue before the BF16 store.)
 *
 *   x_bf16  [M][K] bfloat16 activation; quantised inside the call exactly like
 *           biloco_quant_act, and used unquantised (BF16) for the correction
 *   W_fp4, W_sf, gscale   as written by biloco_pack_weight
 *   Ubits   [N][ceil(r/32)] uint32 = pack_signs(U)      (may be NULL when r == 0)
 *   Vbits   [r][K/32] uint32 = pack_signs(V^T)           (may be NULL when r == 0)
 *   alpha   [r] float                                    (may be NULL when r == 0)
 *   y_bf16  out [M][N] bfloat16, rounded to nearest-even from FP32
 *   limits  1 <= M <= 128, N % 128 == 0, N <= 2^24, K % 64 == 0, 0 <= r <= 1024,
 *           (N/128) * ceil(K/256) <= 2^24
 * Accumulation is FP32 in an unspecified order; results are deterministic for a
 * fixed shape, mode and GPU.  Under the shared-z schedule, batches of up to 128
 * rows run one kernel that quantises the activation itself when each CTA's share
 * of the weight fits the batch class (ceil(units / G) <= 16 units of 128 x 256
 * up to 16 rows, <= 64 above); otherwise an activation quantiser runs first for
 * M > 8 (biloco_gemm_kernel_count).
 * The fused kernel is launched with programmatic dependent launch: it may start
 * while the kernel before it on the stream finishes, and it reads W_fp4 and
 * W_sf before waiting for that kernel (everything else after).  So the weight
 * operand must not be written by a preceding kernel that triggers early launch
 * of its dependents (griddepcontrol.launch_dependents); kernels without that
 * trigger, biloco_pack_weight's included, are fully ordered before the call.
 *
 * Residency: the GEMM kernel runs one CTA per SM on G <= min(#SMs, units) CTAs
 * that exchange data behind grid-wide arrival counters, so all G CTAs must be
 * resident together.  The host checks that one CTA per SM fits
 * (BILOCO_ERR_RESIDENCY otherwise).  With the default launch form
 * (BILOCO_LAUNCH_PDL) the GPU must also not be shared with long-running kernels
 * on other streams, or with another biloco_gemm call running concurrently on
 * another stream: CTAs that cannot start leave the others waiting, and after
 * their bounded wait (about 1 s) they give up and biloco_last_error reports
 * BILOCO_ERR_TIMEOUT (y is then not valid).  Where the GPU is shared, select
 * BILOCO_LAUNCH_COOPERATIVE (biloco_set_launch): the driver then starts the
 * grid only once all of its CTAs can be resident.
 */
int biloco_gemm(const void *x_bf16, const uint8_t *W_fp4, const uint8_t *W_sf,
                const float *gscale, const uint32_t *Ubits, const uint32_t *Vbits,
                const float *alpha, void *y_bf16, int M, int N, int K, int r,
                biloco_stream_t stream);

/*
 * biloco_gemm_noalloc - biloco_gemm with no device allocation.
 * The BiLoCo pages have no counterpart of this call: it exists for callers that
 * cannot let the library allocate, e.g. an engine that has reserved nearly all of
 * HBM for its own pools, or a decode loop that cannot have its stream stalled
 * while biloco_gemm grows its per-stream scratch (synchronise, free, cudaMalloc).
 *
 * Same arguments, limits, results and error codes as biloco_gemm; the results
 * equal biloco_gemm's for the same shape and mode.  Its scratch is one static
 * device array of BILOCO_NOALLOC_SCRATCH_BYTES per device, part of the library's
 * device code; the call never calls cudaMalloc or cudaFree.  Extra limits,
 * checked on the host before anything is launched (BILOCO_ERR_SHAPE otherwise):
 *   N <= BILOCO_NOALLOC_MAX_N, and the call's scratch fits the array.  That
 *   scratch is 16 896 bytes of status and counters plus, each rounded up to 256,
 *   with KC = ceil(K/256), G = min(#SMs, (N/128)*KC) (for 65..128 rows on the
 *   decode-batch kernel at most 5*(N/128)/2 where that keeps <= 64 units per
 *   CTA) and rpad = 16*ceil(r/16):
 *   decode-batch kernel (M <= 128, shared-z schedule, ceil(units/G) <= 16 for
 *   M <= 16 or <= 64 above; BN = 16 for M <= 16, else the batch class 32, 64
 *   or 128 that holds M):
 *     KC * (M <= 16 ? 2304 : BN * 128 + 2048)  (quantised activation image)
 *     ztile + max(G, ceil(r/128)) * BN * 512   (z tiles, V-side partial sums;
 *                                               ztile = 65536 for M <= 16,
 *                                               else 4096 * BN)
 *     M * rpad * 4                             (z)
 *     2 * G * BN * 512                         (split-K partials)
 *   general kernel (every other shape; BN = 16, 32, 64, 128 for M <= 16, 32,
 *   64, 128):
 *     M > 8:  M*K/2 + KC*2048                  (quantised activation)
 *     r > 0:  (KC + 1) * M * rpad * 4          (z partials and z)
 *     always: 2 * G * BN * 512                 (split-K partials)
 *   On a 148-SM B200 every M <= 64 shape with K <= 13824 and r <= 1024 fits;
 *   M > 64 fits only small weights (few units, so a small G).
 * Caveats:
 *   - There is one array per device, shared by all streams and host threads:
 *     calls that overlap in time (on different streams, or from several threads
 *     without ordering) race on it and give wrong results.  Order the calls.
 *   - The first call on a device looks up the array's address
 *     (cudaGetSymbolAddress) and clears its status and counters with an
 *     asynchronous memset; make it before any stream capture begins.
 *   - Device-side errors (an expired bounded wait) are reported by
 *     biloco_last_error(stream), which also clears the array's counters.
 */
#define BILOCO_NOALLOC_SCRATCH_BYTES (16u << 20)
#define BILOCO_NOALLOC_MAX_N (1 << 18)
int biloco_gemm_noalloc(const void *x_bf16, const uint8_t *W_fp4, const uint8_t *W_sf,
                        const float *gscale, const uint32_t *Ubits, const uint32_t *Vbits,
                        const float *alpha, void *y_bf16, int M, int N, int K, int r,
                        biloco_stream_t stream);

/*
 * Launch form of the GEMM kernels for later biloco_gemm / biloco_gemm_noalloc
 * calls (process-wide), a combination of:
 *   BILOCO_LAUNCH_PDL          programmatic dependent launch: the kernel may start
 *                              while the kernel before it on the stream finishes
 *                              (its weight stream overlaps that kernel's tail)
 *   BILOCO_LAUNCH_COOPERATIVE  cooperative launch: every CTA of the grid is
 *                              resident together, whatever else runs on the GPU
 * Default BILOCO_LAUNCH_PDL.  With both flags the grid is launched with both
 * attributes where the driver accepts the pair, else cooperative only.  Not part
 * of the BiLoCo pages.  BILOCO_ERR_ARG for unknown flags.
 */
enum { BILOCO_LAUNCH_PDL = 1, BILOCO_LAUNCH_COOPERATIVE = 2 };
int biloco_set_launch(int flags);
int biloco_get_launch(void);

/*
 * Arithmetic of the correction's U side on the CUDA cores (the decode-batch
 * kernel at 1-2 rows; every other shape ignores it), for later calls
 * (process-wide):
 *   BILOCO_CORR_SIGNS  sign-adds: every rank's z added or subtracted per weight row
 *   BILOCO_CORR_LUT    table lookups: each CTA that completes a tile builds, from
 *                      z, the 16 signed sums of every group of four ranks
 *                      (FluxBin, "LUT-based Multiplication"; the BiLoCo README's
 *                      LUT branch), and a weight row adds one entry per four ranks
 *   BILOCO_CORR_AUTO   the measured choice per shape
 * Both give y within the stated tolerance of the oracle (different FP32 summation
 * orders).  BILOCO_ERR_ARG for an unknown value.  Not part of the BiLoCo pages'
 * API.
 */
enum { BILOCO_CORR_AUTO = 0, BILOCO_CORR_SIGNS = 1, BILOCO_CORR_LUT = 2 };
int biloco_set_correction(int arith);
/* The arithmetic biloco_gemm would use for this shape under the current setting. */
int biloco_resolve_correction(int M, int N, int K, int r);

/* Select the z schedule for later biloco_gemm calls (process-wide). */
int biloco_set_mode(int mode);
/* The schedule biloco_gemm would use for this shape under the current setting. */
int biloco_resolve_mode(int M, int N, int K, int r);

/*
 * biloco_last_error - synchronise `stream`, return and clear the first error a
 * kernel on it recorded (BILOCO_ERR_TIMEOUT when a bounded wait expired), or
 * BILOCO_OK.  After an error the stream's scratch counters are reset.  Once
 * biloco_gemm_noalloc has run on the current device, its static scratch is
 * checked and reset the same way; because that array serves every stream, the
 * call then synchronises the whole device first (cudaDeviceSynchronize), so that
 * a no-allocation call still running on another stream is neither missed nor
 * cleared while it runs.
 */
int biloco_last_error(biloco_stream_t stream);

/*
 * biloco_selftest_wait_timeout - exercise the failure path on the GPU without a
 * fault.  Launches one warp that waits, through the same bounded mbarrier wait
 * the GEMM kernels use, on a phase nothing completes.  After the wait's
 * wall-clock limit (about 1 s) the kernel records BILOCO_ERR_TIMEOUT in
 * `stream`'s status word and returns, leaving the context usable; a following
 * biloco_last_error(stream) reports it.  The BiLoCo pages have no counterpart
 * of this call.
 */
int biloco_selftest_wait_timeout(biloco_stream_t stream);

/*
 * biloco_selftest_drop_arrivals - exercise the GEMM's own failure path on the GPU
 * without a fault.  The next biloco_gemm or biloco_gemm_noalloc call that runs
 * the decode-batch kernel (M <= 128, shared-z schedule) leaves out the grid-wide
 * arrivals selected by `mask` (1: the z slices, 2: the activation image, which
 * batches of 8 rows and more share, 3: both); every other call, and every call
 * after that one, is unaffected.  The
 * CTAs waiting on those arrivals give up after their bounded wait (about 1 s),
 * leave together, drain their copies and tensor-core work, free their tensor
 * memory and record BILOCO_ERR_TIMEOUT; y of that call is not valid.  A following
 * biloco_last_error(stream) reports the timeout and resets the counters, after
 * which calls on the stream are correct again.  BILOCO_ERR_ARG for a mask outside
 * 0..3.  The BiLoCo pages have no counterpart of this call.
 */
int biloco_selftest_drop_arrivals(int mask);

/* Human-readable name of a status code (static storage). */
const char *biloco_status_string(int status);

/* Number of kernels biloco_gemm would launch per call for this shape under the
 * current schedule setting: 1 when the GEMM kernel quantises the activation
 * itself (the decode-batch kernel, M <= 128, or the general kernel at M <= 8),
 * else 2 (quantiser + GEMM).  BILOCO_ERR_SHAPE for shapes biloco_gemm rejects.
 * Uses the device's SM count (the current device must be set). */
int biloco_gemm_kernel_count(int M, int N, int K, int r);

/* Free every stream's scratch.  Safe to call more than once. */
void biloco_shutdown(void);

#ifdef __cplusplus
}
#endif
#endif /* BILOCO_H */
