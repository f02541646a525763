// C ABI of libbiloco.so: argument checking, per-(device, stream) scratch and the
// device status word.  The compute lives in quant.cu, gemm_host.cu and the
// fused_*.cu kernel instances; noalloc.cu holds the static-scratch variant.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/biloco.h"
#include "internal.h"

namespace biloco {

namespace {

std::mutex g_mu;
std::atomic<int> g_mode{BILOCO_MODE_AUTO};
std::atomic<int> g_launch{BILOCO_LAUNCH_PDL};
std::atomic<int> g_arith{BILOCO_CORR_AUTO};
std::atomic<int> g_drop{0};   // failure-path self test, consumed by the next GEMM call

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BILOCO_ERR_CUDA;
  static std::mutex mu;
  static std::vector<int> ok_devices, bad_devices;
  std::lock_guard<std::mutex> lk(mu);
  if (std::find(ok_devices.begin(), ok_devices.end(), dev) != ok_devices.end()) return BILOCO_OK;
  if (std::find(bad_devices.begin(), bad_devices.end(), dev) != bad_devices.end())
    return BILOCO_ERR_DEVICE;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return BILOCO_ERR_CUDA;
  if (major != 10) {
    bad_devices.push_back(dev);
    return BILOCO_ERR_DEVICE;
  }
  ok_devices.push_back(dev);
  return BILOCO_OK;
}

// Region offsets of one scratch block, every region 256-byte aligned.
struct Carve {
  size_t status, counters, act_fp4, act_sf, zpart, zfin, slots, total;
};

Carve carve(const ScratchNeed& n) {
  Carve c{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + std::max<size_t>(bytes, 1), 256);
    return at;
  };
  c.status = take(16);
  c.counters = take(n.counter_words * 4);
  c.act_fp4 = take(n.act_fp4);
  c.act_sf = take(n.act_sf);
  c.zpart = take(n.zpart);
  c.zfin = take(n.zfin);
  c.slots = take(n.slots);
  c.total = off;
  return c;
}

ScratchNeed max_need(const ScratchNeed& a, const ScratchNeed& b) {
  ScratchNeed m;
  m.act_fp4 = std::max(a.act_fp4, b.act_fp4);
  m.act_sf = std::max(a.act_sf, b.act_sf);
  m.zpart = std::max(a.zpart, b.zpart);
  m.zfin = std::max(a.zfin, b.zfin);
  m.slots = std::max(a.slots, b.slots);
  m.counter_words = std::max(a.counter_words, b.counter_words);
  return m;
}

struct ScratchEntry {
  Scratch s;
  ScratchNeed have{};
};

std::vector<ScratchEntry*> g_entries;

void apply_carve(Scratch& s, const Carve& c, const ScratchNeed& n) {
  uint8_t* b = static_cast<uint8_t*>(s.base);
  s.status = reinterpret_cast<int*>(b + c.status);
  s.counters = reinterpret_cast<uint32_t*>(b + c.counters);
  s.counter_words = n.counter_words;
  s.act_fp4 = b + c.act_fp4;
  s.act_sf = b + c.act_sf;
  s.zpart = reinterpret_cast<float*>(b + c.zpart);
  s.zfin = reinterpret_cast<float*>(b + c.zfin);
  s.slots = reinterpret_cast<float*>(b + c.slots);
}

}  // namespace

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

Scratch* get_scratch(cudaStream_t stream, const ScratchNeed& need) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  ScratchEntry* e = nullptr;
  for (ScratchEntry* x : g_entries)
    if (x->s.device == dev && x->s.stream == stream) e = x;
  if (e) {
    const ScratchNeed& h = e->have;
    if (need.act_fp4 <= h.act_fp4 && need.act_sf <= h.act_sf && need.zpart <= h.zpart &&
        need.zfin <= h.zfin && need.slots <= h.slots && need.counter_words <= h.counter_words)
      return &e->s;
  }
  ScratchNeed want = e ? max_need(e->have, need) : need;
  const Carve c = carve(want);
  if (e) {
    // grow: the old block may still be in use by queued work on this stream
    if (cudaStreamSynchronize(stream) != cudaSuccess) return nullptr;
    cudaFree(e->s.base);
    e->s.base = nullptr;
  } else {
    e = new ScratchEntry();
    e->s.device = dev;
    e->s.stream = stream;
    g_entries.push_back(e);
  }
  void* base = nullptr;
  if (cudaMalloc(&base, c.total) != cudaSuccess) {
    e->have = ScratchNeed{};
    return nullptr;
  }
  // zero everything: counters and status start at 0, scale atoms start finite
  if (cudaMemsetAsync(base, 0, c.total, stream) != cudaSuccess) return nullptr;
  e->s.base = base;
  e->s.bytes = c.total;
  e->have = want;
  apply_carve(e->s, c, want);
  return &e->s;
}

int check_gemm_args(const void* x_bf16, const uint8_t* W_fp4, const uint8_t* W_sf, const float* gscale,
                    const uint32_t* Ubits, const uint32_t* Vbits, const float* alpha, void* y_bf16,
                    int M, int N, int K, int r, GemmArgs* a) {
  if (!x_bf16 || !W_fp4 || !W_sf || !gscale || !y_bf16) return BILOCO_ERR_ARG;
  if (r > 0 && (!Ubits || !Vbits || !alpha)) return BILOCO_ERR_ARG;
  if (M < 1 || M > BILOCO_MAX_M || N < 128 || N % 128 || K < 64 || K % 64 || r < 0 ||
      r > BILOCO_MAX_R || N > BILOCO_MAX_N ||
      static_cast<long long>(N / 128) * ((K + 255) / 256) > BILOCO_MAX_UNITS)
    return BILOCO_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(W_fp4) || !aligned16(W_sf) || !aligned16(y_bf16) ||
      (reinterpret_cast<uintptr_t>(gscale) & 3u) || (r > 0 && (!aligned16(Ubits) || !aligned16(Vbits) ||
                                                               (reinterpret_cast<uintptr_t>(alpha) & 3u))))
    return BILOCO_ERR_ALIGN;
  int d = check_device();
  if (d) return d;
  a->x = static_cast<const uint16_t*>(x_bf16);
  a->W_fp4 = W_fp4;
  a->W_sf = W_sf;
  a->gscale = gscale;
  a->Ubits = Ubits;
  a->Vbits = Vbits;
  a->alpha = alpha;
  a->y = static_cast<uint16_t*>(y_bf16);
  a->M = M;
  a->N = N;
  a->K = K;
  a->r = r;
  a->mode = resolve_mode(M, N, K, r, g_mode.load());
  a->arith = resolve_arith(M, N, K, r, g_arith.load());
  a->drop = g_drop.exchange(0);
  return BILOCO_OK;
}

LaunchOpts current_launch_opts() {
  LaunchOpts o;
  const int f = g_launch.load();
  o.pdl = (f & BILOCO_LAUNCH_PDL) != 0;
  o.cooperative = (f & BILOCO_LAUNCH_COOPERATIVE) != 0;
  return o;
}

}  // namespace biloco

using namespace biloco;

extern "C" {

int biloco_quant_act(const void* x_bf16, int M, int K, uint8_t* x_fp4, uint8_t* x_sf,
                     biloco_stream_t stream) {
  if (!x_bf16 || !x_fp4 || !x_sf) return BILOCO_ERR_ARG;
  if (M < 1 || K < 16 || K % 16) return BILOCO_ERR_SHAPE;
  if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(x_fp4) & 7u)) return BILOCO_ERR_ALIGN;
  int d = check_device();
  if (d) return d;
  return launch_quant_act_rowmajor(static_cast<const uint16_t*>(x_bf16), M, K, x_fp4, x_sf,
                                   reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? BILOCO_OK
             : BILOCO_ERR_CUDA;
}

int biloco_pack_signs(const float* S, int rows, int cols, uint32_t* bits, biloco_stream_t stream) {
  if (!S || !bits) return BILOCO_ERR_ARG;
  if (rows < 1 || cols < 1) return BILOCO_ERR_SHAPE;
  int d = check_device();
  if (d) return d;
  return launch_pack_signs(S, rows, cols, bits, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? BILOCO_OK
             : BILOCO_ERR_CUDA;
}

size_t biloco_weight_sf_bytes(int N, int K) {
  if (N < 0 || K < 0) return 0;
  return static_cast<size_t>(N) * ((K + 255) / 256) * 16;
}

int biloco_pack_weight(const float* R, int N, int K, uint8_t* W_fp4, uint8_t* W_sf, float* gscale,
                       biloco_stream_t stream) {
  if (!R || !W_fp4 || !W_sf || !gscale) return BILOCO_ERR_ARG;
  if (N < 128 || N % 128 || K < 64 || K % 64) return BILOCO_ERR_SHAPE;
  if (!aligned16(R) || !aligned16(W_fp4) || !aligned16(W_sf) ||
      (reinterpret_cast<uintptr_t>(gscale) & 3u))
    return BILOCO_ERR_ALIGN;
  int d = check_device();
  if (d) return d;
  return launch_pack_weight(R, N, K, W_fp4, W_sf, gscale, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? BILOCO_OK
             : BILOCO_ERR_CUDA;
}

int biloco_gemm(const void* x_bf16, const uint8_t* W_fp4, const uint8_t* W_sf, const float* gscale,
                const uint32_t* Ubits, const uint32_t* Vbits, const float* alpha, void* y_bf16, int M,
                int N, int K, int r, biloco_stream_t stream) {
  GemmArgs a;
  const int st = check_gemm_args(x_bf16, W_fp4, W_sf, gscale, Ubits, Vbits, alpha, y_bf16, M, N, K, r, &a);
  if (st) return st;
  return run_gemm(a, reinterpret_cast<cudaStream_t>(stream));
}

int biloco_selftest_wait_timeout(biloco_stream_t stream) {
  int d = check_device();
  if (d) return d;
  ScratchNeed need = {16, 16, 16, 16, 16, 2};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Scratch* sc = get_scratch(s, need);
  if (!sc) return BILOCO_ERR_NOMEM;
  return launch_wait_timeout(sc->status, s) == cudaSuccess ? BILOCO_OK : BILOCO_ERR_CUDA;
}

int biloco_selftest_drop_arrivals(int mask) {
  if (mask < 0 || mask > 3) return BILOCO_ERR_ARG;
  g_drop.store(mask);
  return BILOCO_OK;
}

int biloco_set_launch(int flags) {
  if (flags < 0 || flags > (BILOCO_LAUNCH_PDL | BILOCO_LAUNCH_COOPERATIVE)) return BILOCO_ERR_ARG;
  g_launch.store(flags);
  return BILOCO_OK;
}

int biloco_get_launch(void) { return g_launch.load(); }

int biloco_set_correction(int arith) {
  if (arith != BILOCO_CORR_AUTO && arith != BILOCO_CORR_SIGNS && arith != BILOCO_CORR_LUT) return BILOCO_ERR_ARG;
  g_arith.store(arith);
  return BILOCO_OK;
}

int biloco_resolve_correction(int M, int N, int K, int r) { return resolve_arith(M, N, K, r, g_arith.load()); }

int biloco_set_mode(int mode) {
  if (mode != BILOCO_MODE_AUTO && mode != BILOCO_MODE_SHARED_Z && mode != BILOCO_MODE_LOCAL_Z)
    return BILOCO_ERR_ARG;
  g_mode.store(mode);
  return BILOCO_OK;
}

int biloco_resolve_mode(int M, int N, int K, int r) { return resolve_mode(M, N, K, r, g_mode.load()); }

int biloco_last_error(biloco_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BILOCO_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BILOCO_ERR_CUDA;
  Scratch* sc = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (ScratchEntry* e : g_entries)
      if (e->s.device == dev && e->s.stream == s && e->s.base) sc = &e->s;
  }
  int status = 0;
  if (sc) {
    if (cudaMemcpy(&status, sc->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
      return BILOCO_ERR_CUDA;
    if (status != 0) {
      // a kernel gave up part-way: clear the status and every cross-CTA counter
      cudaMemset(sc->status, 0, sizeof(int));
      cudaMemset(sc->counters, 0, sc->counter_words * 4);
      cudaDeviceSynchronize();
    }
  }
  const int static_status = noalloc_take_status();
  return status != 0 ? status : static_status;
}

const char* biloco_status_string(int status) {
  switch (status) {
    case BILOCO_OK: return "ok";
    case BILOCO_ERR_ARG: return "invalid argument";
    case BILOCO_ERR_SHAPE: return "unsupported shape";
    case BILOCO_ERR_ALIGN: return "pointer not 16-byte aligned";
    case BILOCO_ERR_CUDA: return "CUDA call failed";
    case BILOCO_ERR_TIMEOUT: return "device-side wait timed out";
    case BILOCO_ERR_NOMEM: return "scratch allocation failed";
    case BILOCO_ERR_DEVICE: return "device is not sm_100";
    case BILOCO_ERR_RESIDENCY: return "grid cannot be resident on the GPU at once";
    default: return "unknown status";
  }
}

int biloco_gemm_kernel_count(int M, int N, int K, int r) {
  if (M < 1 || M > BILOCO_MAX_M || N < 128 || N % 128 || K < 64 || K % 64 || r < 0 || r > BILOCO_MAX_R)
    return BILOCO_ERR_SHAPE;
  GemmArgs a = {};
  a.M = M;
  a.N = N;
  a.K = K;
  a.r = r;
  a.mode = resolve_mode(M, N, K, r, g_mode.load());
  return gemm_kernel_count_for(a);
}

void biloco_shutdown(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (ScratchEntry* e : g_entries) {
    if (e->s.base) {
      int cur = 0;
      cudaGetDevice(&cur);
      cudaSetDevice(e->s.device);
      cudaDeviceSynchronize();
      cudaFree(e->s.base);
      cudaSetDevice(cur);
    }
    delete e;
  }
  g_entries.clear();
}

}  // extern "C"
