// Binary low-rank decomposition W ~= U diag(alpha) V^T + R on the GPU
// (BiLoCo README, section "Decomposition": each rank-one term starts from random
// signs and alternates u = sign(R v), v = sign(R^T u) for T steps, takes the
// Frobenius-optimal coefficient and deflates the residual; after all r terms the
// coefficients are refit jointly by least squares for the fixed signs).
//
// The residual is kept explicitly, in FP64, in the caller's workspace, so that
// every sign decision is taken on an FP64 sum (sign(0) = +1).  Each alternation
// is two passes over it, both bound by memory bandwidth (CUDA cores, coalesced
// FP64 loads):
//   * rows:    u_n = sign(sum_k R[n][k] v_k), one warp per row, four rows per
//              warp interleaved, a fixed-order shuffle reduction;
//   * columns: (R^T u)_k in S row slices (one thread per column, consecutive
//              threads on consecutive columns), then the slices added in order;
//              v_k = sign of the sum.  The last alternation's column pass also
//              gives u^T R v = sum_k |(R^T u)_k|, so alpha = that / (N K).
// Deflation R -= alpha u v^T is one more read-write pass.
//
// The refit solves G alpha = b with G_ij = (u_i . u_j)(v_i . v_j) (exact integer
// dot products of sign words by popcount) and b_i = u_i^T W v_i, which follows
// from the greedy coefficients: b_i = alpha_i N K + sum_{j<i} alpha_j G_ij.  G is
// symmetric positive semidefinite and b lies in its range, so conjugate gradients
// from zero converge to the minimum-norm solution (the least-squares one when
// terms repeat).  The returned residual W - U diag(alpha) V^T is an FP64 rank-r
// update, stored as FP32.
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/biloco.h"
#include "internal.h"

namespace biloco {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t bit_of(const uint32_t* words, int i) {
  return (__ldg(words + (i >> 5)) >> (i & 31)) & 1u;
}

// u = sign(R v): CTA of 8 warps covers 32 rows, each warp 4 of them.  Also keeps
// the rank-major copy of the word it writes.
__global__ void __launch_bounds__(kThreads)
rows_sign_kernel(const double* __restrict__ R, int N, int K, const uint32_t* __restrict__ vbits,
                 uint32_t* __restrict__ ubits) {
  __shared__ uint32_t neg[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * 32 + warp * 4;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int kb = 0; kb < K; kb += 32) {
    const int k = kb + lane;
    if (k < K) {
      const bool vneg = ((__ldg(vbits + (kb >> 5)) >> lane) & 1u) != 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = row0 + j;
        if (n < N) {
          const double x = __ldg(R + static_cast<size_t>(n) * K + k);
          acc[j] += vneg ? -x : x;
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    if (lane == 0) neg[warp * 4 + j] = (row0 + j < N && acc[j] < 0.0) ? 1u : 0u;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const uint32_t w = __ballot_sync(0xffffffffu, neg[threadIdx.x] != 0);
    if (threadIdx.x == 0) ubits[blockIdx.x] = w;
  }
}

// Partial sums of (R^T u)_k over row slice s: part[s][k].
__global__ void __launch_bounds__(kThreads)
cols_partial_kernel(const double* __restrict__ R, int N, int K, const uint32_t* __restrict__ ubits,
                    int rows_per_slice, double* __restrict__ part) {
  const int k = blockIdx.x * kThreads + threadIdx.x;
  const int s = blockIdx.y;
  const int n0 = s * rows_per_slice, n1 = min(N, n0 + rows_per_slice);
  if (k >= K) return;
  double acc0 = 0.0, acc1 = 0.0;
  int n = n0;
  for (; n + 1 < n1; n += 2) {
    const double a = __ldg(R + static_cast<size_t>(n) * K + k);
    const double b = __ldg(R + static_cast<size_t>(n + 1) * K + k);
    acc0 += bit_of(ubits, n) ? -a : a;
    acc1 += bit_of(ubits, n + 1) ? -b : b;
  }
  if (n < n1) {
    const double a = __ldg(R + static_cast<size_t>(n) * K + k);
    acc0 += bit_of(ubits, n) ? -a : a;
  }
  part[static_cast<size_t>(s) * K + k] = acc0 + acc1;
}

// v = sign(sum_s part[s][k]) and, per CTA, the partial sum of |(R^T u)_k|.
__global__ void __launch_bounds__(kThreads)
cols_finish_kernel(const double* __restrict__ part, int S, int K, uint32_t* __restrict__ vbits,
                   double* __restrict__ absdot) {
  __shared__ double red[kThreads / 32];
  const int k = blockIdx.x * kThreads + threadIdx.x;
  double sum = 0.0;
  if (k < K)
    for (int s = 0; s < S; ++s) sum += part[static_cast<size_t>(s) * K + k];
  const uint32_t w = __ballot_sync(0xffffffffu, k < K && sum < 0.0);
  if ((threadIdx.x & 31) == 0 && k < K) vbits[k >> 5] = w;
  double a = fabs(sum);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int j = 0; j < kThreads / 32; ++j) t += red[j];
    absdot[blockIdx.x] = t;
  }
}

// alpha_i = sum of the CTA partials of u^T R v, in order, / (N K).
__global__ void alpha_kernel(const double* __restrict__ absdot, int nparts, double nk,
                             double* __restrict__ alpha_i) {
  double t = 0.0;
  for (int j = 0; j < nparts; ++j) t += absdot[j];
  *alpha_i = t / nk;
}

// R -= alpha u v^T.
__global__ void __launch_bounds__(kThreads)
deflate_kernel(double* __restrict__ R, int N, int K, const uint32_t* __restrict__ ubits,
               const uint32_t* __restrict__ vbits, const double* __restrict__ alpha_i) {
  const double a = *alpha_i;
  const size_t total = static_cast<size_t>(N) * K;
  for (size_t idx = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x; idx < total;
       idx += static_cast<size_t>(gridDim.x) * kThreads) {
    const int n = static_cast<int>(idx / K), k = static_cast<int>(idx - static_cast<size_t>(n) * K);
    const bool neg = (bit_of(ubits, n) ^ bit_of(vbits, k)) != 0;
    R[idx] -= neg ? -a : a;
  }
}

__global__ void __launch_bounds__(kThreads)
widen_kernel(const float* __restrict__ W, size_t total, double* __restrict__ R) {
  for (size_t idx = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x; idx < total;
       idx += static_cast<size_t>(gridDim.x) * kThreads)
    R[idx] = static_cast<double>(__ldg(W + idx));
}

// G_ij = (u_i . u_j)(v_i . v_j) from rank-major sign words, and
// b_i = alpha_i N K + sum_{j<i} alpha_j G_ij.  One thread per (i, j).
__global__ void __launch_bounds__(kThreads)
gram_kernel(const uint32_t* __restrict__ ut, int NW, int N, const uint32_t* __restrict__ vt, int KW, int K,
            int r, double* __restrict__ G) {
  const int idx = blockIdx.x * kThreads + threadIdx.x;
  if (idx >= r * r) return;
  const int i = idx / r, j = idx - i * r;
  int du = 0, dv = 0;
  for (int w = 0; w < NW; ++w) du += __popc(__ldg(ut + static_cast<size_t>(i) * NW + w) ^ __ldg(ut + static_cast<size_t>(j) * NW + w));
  for (int w = 0; w < KW; ++w) dv += __popc(__ldg(vt + static_cast<size_t>(i) * KW + w) ^ __ldg(vt + static_cast<size_t>(j) * KW + w));
  G[idx] = static_cast<double>(N - 2 * du) * static_cast<double>(K - 2 * dv);
}

// Conjugate gradients on G alpha = b (b from the greedy coefficients), one CTA.
// Stops when ||residual|| <= 1e-15 ||b|| or after max_it steps.
__global__ void __launch_bounds__(1024)
refit_cg_kernel(const double* __restrict__ G, const double* __restrict__ ag, int r, double nk, int max_it,
                double* __restrict__ work, float* __restrict__ alpha_out, double* __restrict__ alpha_fit) {
  __shared__ double red[32];
  __shared__ double scal;
  double* x = work;
  double* res = work + r;
  double* p = work + 2 * r;
  double* q = work + 3 * r;
  double* b = work + 4 * r;
  const int tid = threadIdx.x;
  auto block_sum = [&](double v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((tid & 31) == 0) red[tid >> 5] = v;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int j = 0; j < (blockDim.x + 31) / 32; ++j) t += red[j];
      scal = t;
    }
    __syncthreads();
    const double out = scal;
    __syncthreads();
    return out;
  };
  for (int i = tid; i < r; i += blockDim.x) {
    double bi = ag[i] * nk;
    for (int j = 0; j < i; ++j) bi += ag[j] * G[static_cast<size_t>(i) * r + j];
    b[i] = bi;
    x[i] = 0.0;
    res[i] = bi;
    p[i] = bi;
  }
  __syncthreads();
  double rr = 0.0;
  for (int i = tid; i < r; i += blockDim.x) rr += res[i] * res[i];
  rr = block_sum(rr);
  const double stop = 1e-30 * rr;                // (1e-15 ||b||)^2
  for (int it = 0; it < max_it && rr > stop; ++it) {
    double pq = 0.0;
    for (int i = tid; i < r; i += blockDim.x) {
      double s = 0.0;
      for (int j = 0; j < r; ++j) s += G[static_cast<size_t>(i) * r + j] * p[j];
      q[i] = s;
      pq += p[i] * s;
    }
    pq = block_sum(pq);
    if (pq <= 0.0) break;
    const double a = rr / pq;
    double rr2 = 0.0;
    for (int i = tid; i < r; i += blockDim.x) {
      x[i] += a * p[i];
      res[i] -= a * q[i];
      rr2 += res[i] * res[i];
    }
    rr2 = block_sum(rr2);
    const double beta = rr2 / rr;
    for (int i = tid; i < r; i += blockDim.x) p[i] = res[i] + beta * p[i];
    rr = rr2;
    __syncthreads();
  }
  for (int i = tid; i < r; i += blockDim.x) {
    alpha_fit[i] = x[i];
    alpha_out[i] = static_cast<float>(x[i]);
  }
}

// R_out = W - U diag(alpha) V^T (FP64 sum, FP32 out).  A CTA owns 16 rows x 256
// columns; each thread one column of 16 rows.  The rank loop reads one sign word
// per 32 ranks.
__global__ void __launch_bounds__(kThreads)
residual_kernel(const float* __restrict__ W, int N, int K, const uint32_t* __restrict__ ubits, int RW,
                const uint32_t* __restrict__ vt, int KW, const double* __restrict__ alpha, int r,
                float* __restrict__ Rout) {
  __shared__ uint32_t us[16][32];                  // this CTA's rows: their rank words (r <= 1024)
  __shared__ double as[1024];
  const int k = blockIdx.x * kThreads + threadIdx.x;
  const int n0 = blockIdx.y * 16;
  for (int idx = threadIdx.x; idx < 16 * RW; idx += kThreads) {
    const int j = idx / RW, w = idx - j * RW;
    us[j][w] = (n0 + j < N) ? __ldg(ubits + static_cast<size_t>(n0 + j) * RW + w) : 0u;
  }
  for (int i = threadIdx.x; i < r; i += kThreads) as[i] = alpha[i];
  __syncthreads();
  if (k >= K) return;
  double acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.0;
  for (int i = 0; i < r; ++i) {
    const uint32_t vneg = bit_of(vt + static_cast<size_t>(i) * KW, k);
    const double a = as[i];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t uneg = (us[j][i >> 5] >> (i & 31)) & 1u;
      acc[j] += (uneg ^ vneg) ? -a : a;
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int n = n0 + j;
    if (n < N) {
      const size_t o = static_cast<size_t>(n) * K + k;
      Rout[o] = static_cast<float>(static_cast<double>(__ldg(W + o)) - acc[j]);
    }
  }
}

// Rank-major U words [r][NW] -> row-major Ubits [N][RW] (bit i of word i / 32).
__global__ void __launch_bounds__(kThreads)
transpose_u_kernel(const uint32_t* __restrict__ ut, int NW, int N, int r, int RW, uint32_t* __restrict__ ubits) {
  const int idx = blockIdx.x * kThreads + threadIdx.x;
  if (idx >= N * RW) return;
  const int n = idx / RW, w = idx - n * RW;
  uint32_t word = 0u;
  for (int b = 0; b < 32; ++b) {
    const int i = w * 32 + b;
    if (i < r) word |= ((__ldg(ut + static_cast<size_t>(i) * NW + (n >> 5)) >> (n & 31)) & 1u) << b;
  }
  ubits[idx] = word;
}

unsigned blocks_for(size_t threads) { return static_cast<unsigned>((threads + kThreads - 1) / kThreads); }

struct Work {
  double* R;         // [N][K]
  double* part;      // [S][K]
  double* absdot;    // [ceil(K/256)]
  double* ag;        // [r] greedy coefficients
  double* afit;      // [r] refit coefficients
  double* G;         // [r][r]
  double* cg;        // [5 r]
  uint32_t* ut;      // [r][NW] rank-major U words
  size_t bytes;
};

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

Work carve(void* base, int N, int K, int r, int S) {
  Work w{};
  uint8_t* b = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = b ? b + off : nullptr;
    off = align256(off + bytes);
    return p;
  };
  const int NW = (N + 31) / 32;
  w.R = reinterpret_cast<double*>(take(static_cast<size_t>(N) * K * 8));
  w.part = reinterpret_cast<double*>(take(static_cast<size_t>(S) * K * 8));
  w.absdot = reinterpret_cast<double*>(take(static_cast<size_t>((K + kThreads - 1) / kThreads) * 8));
  w.ag = reinterpret_cast<double*>(take(static_cast<size_t>(r) * 8 + 8));
  w.afit = reinterpret_cast<double*>(take(static_cast<size_t>(r) * 8 + 8));
  w.G = reinterpret_cast<double*>(take(static_cast<size_t>(r) * r * 8 + 8));
  w.cg = reinterpret_cast<double*>(take(static_cast<size_t>(5 * r) * 8 + 8));
  w.ut = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(r) * NW * 4 + 4));
  w.bytes = off;
  return w;
}

// Row slices of the column pass: enough CTAs for two per SM, at least 32 rows each.
int column_slices(int N, int K) {
  const int cblocks = (K + kThreads - 1) / kThreads;
  int S = (2 * num_sms() + cblocks - 1) / cblocks;
  S = std::max(1, std::min(S, (N + 31) / 32));
  return S;
}

}  // namespace

}  // namespace biloco

using namespace biloco;

extern "C" size_t biloco_decompose_workspace_bytes(int N, int K, int r) {
  if (N < 1 || K < 1 || r < 0 || r > BILOCO_MAX_R) return 0;
  return carve(nullptr, N, K, r, column_slices(N, K)).bytes;
}

extern "C" int biloco_decompose(const float* W, int N, int K, int r, int T, const uint32_t* v0bits,
                                uint32_t* Ubits, uint32_t* Vbits, float* alpha, float* R_out,
                                void* workspace, size_t workspace_bytes, biloco_stream_t stream) {
  if (!W || !R_out || !workspace || (r > 0 && (!v0bits || !Ubits || !Vbits || !alpha))) return BILOCO_ERR_ARG;
  if (N < 1 || K < 1 || r < 0 || r > BILOCO_MAX_R || T < 1 || static_cast<long long>(N) * K > (1ll << 31))
    return BILOCO_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) || (reinterpret_cast<uintptr_t>(W) & 3u) ||
      (reinterpret_cast<uintptr_t>(R_out) & 3u))
    return BILOCO_ERR_ALIGN;
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return BILOCO_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess) return BILOCO_ERR_CUDA;
  if (major != 10) return BILOCO_ERR_DEVICE;
  const int S = column_slices(N, K);
  const Work w = carve(workspace, N, K, r, S);
  if (workspace_bytes < w.bytes) return BILOCO_ERR_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int NW = (N + 31) / 32, KW = (K + 31) / 32, RW = (r + 31) / 32;
  const size_t total = static_cast<size_t>(N) * K;
  const unsigned fill = static_cast<unsigned>(num_sms()) * 8u;
  const int cblocks = (K + kThreads - 1) / kThreads;
  const int rows_per_slice = (N + S - 1) / S;
  const double nk = static_cast<double>(N) * static_cast<double>(K);

  widen_kernel<<<fill, kThreads, 0, s>>>(W, total, w.R);
  for (int i = 0; i < r; ++i) {
    uint32_t* u = w.ut + static_cast<size_t>(i) * NW;
    uint32_t* v = Vbits + static_cast<size_t>(i) * KW;
    const uint32_t* vcur = v0bits + static_cast<size_t>(i) * KW;
    for (int t = 0; t < T; ++t) {
      rows_sign_kernel<<<NW, kThreads, 0, s>>>(w.R, N, K, vcur, u);
      cols_partial_kernel<<<dim3(cblocks, S), kThreads, 0, s>>>(w.R, N, K, u, rows_per_slice, w.part);
      cols_finish_kernel<<<cblocks, kThreads, 0, s>>>(w.part, S, K, v, w.absdot);
      vcur = v;
    }
    alpha_kernel<<<1, 1, 0, s>>>(w.absdot, cblocks, nk, w.ag + i);
    deflate_kernel<<<fill, kThreads, 0, s>>>(w.R, N, K, u, v, w.ag + i);
  }
  if (r > 0) {
    gram_kernel<<<blocks_for(static_cast<size_t>(r) * r), kThreads, 0, s>>>(w.ut, NW, N, Vbits, KW, K, r, w.G);
    refit_cg_kernel<<<1, 1024, 0, s>>>(w.G, w.ag, r, nk, std::min(r, 256), w.cg, alpha, w.afit);
    transpose_u_kernel<<<blocks_for(static_cast<size_t>(N) * RW), kThreads, 0, s>>>(w.ut, NW, N, r, RW, Ubits);
    residual_kernel<<<dim3(cblocks, (N + 15) / 16), kThreads, 0, s>>>(W, N, K, Ubits, RW, Vbits, KW, w.afit, r,
                                                                       R_out);
  } else {
    cudaMemcpyAsync(R_out, W, total * sizeof(float), cudaMemcpyDeviceToDevice, s);
  }
  return cudaGetLastError() == cudaSuccess ? BILOCO_OK : BILOCO_ERR_CUDA;
}
