// biloco_gemm_noalloc: the fused GEMM with all of its scratch in one static
// device array of the library, so that the call allocates no device memory.
//
// biloco_gemm keeps scratch per (device, stream): it calls cudaMalloc on the
// first call and, when a larger shape arrives, synchronises the stream, frees
// the block and allocates a bigger one.  Some callers cannot have that.  A
// serving engine that reserves nearly all of HBM for its own pools at start-up
// may have no memory left for a hidden cudaMalloc, and one that runs a
// fixed-latency decode loop cannot have the library stall its stream for a
// re-allocation in the middle of a run.  This entry point serves them: its
// scratch is a module-scope __device__ array created with the library's device
// code, it never allocates or frees, and a shape that does not fit is refused
// on the host.
//
// Layout of the array: the status word (256 bytes), the cross-CTA counters for
// up to BILOCO_NOALLOC_MAX_N / 128 weight tiles (a fixed region, so that no
// other region ever overlaps them and they stay zero between calls: every
// kernel returns the counters it used to zero when it ends without error),
// then the shape-dependent regions of the call, carved anew for each shape.
#include <algorithm>
#include <cstdint>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/biloco.h"
#include "internal.h"

namespace biloco {

namespace {

constexpr size_t kCap = BILOCO_NOALLOC_SCRATCH_BYTES;
constexpr size_t kStatusOff = 0;
constexpr size_t kCounterOff = 256;
constexpr size_t kCounterWordsMax = 4 + 2 * static_cast<size_t>(BILOCO_NOALLOC_MAX_N / 128);
constexpr size_t kDataOff = (kCounterOff + kCounterWordsMax * 4 + 255) / 256 * 256;

__device__ __align__(256) uint8_t g_noalloc_scratch[kCap];

struct DeviceScratch {
  int device;
  uint8_t* base;
  bool zeroed;       // status word and counters cleared on some stream
};

std::mutex g_mu;
std::vector<DeviceScratch> g_devices;

size_t round256(size_t v) { return (std::max<size_t>(v, 1) + 255) / 256 * 256; }

// The array's address on the current device, looked up once per device.
DeviceScratch* device_scratch(int dev) {
  for (DeviceScratch& d : g_devices)
    if (d.device == dev) return &d;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return nullptr;
  }
  g_devices.push_back(DeviceScratch{dev, static_cast<uint8_t*>(p), false});
  return &g_devices.back();
}

}  // namespace

int noalloc_take_status() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BILOCO_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceScratch* d = nullptr;
  for (DeviceScratch& x : g_devices)
    if (x.device == dev && x.zeroed) d = &x;
  if (!d) return BILOCO_OK;
  // The array is shared by every stream of the device, and a call on any of them
  // (non-blocking ones included) may still be running: wait for all of them
  // before reading the status, so that no error is missed or cleared early.
  if (cudaDeviceSynchronize() != cudaSuccess) return BILOCO_ERR_CUDA;
  int status = 0;
  if (cudaMemcpy(&status, d->base + kStatusOff, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return BILOCO_ERR_CUDA;
  if (status != 0) {
    // a kernel gave up part-way: its counters may be left non-zero
    if (cudaMemset(d->base, 0, kDataOff) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
      return BILOCO_ERR_CUDA;
  }
  return status;
}

}  // namespace biloco

using namespace biloco;

extern "C" int biloco_gemm_noalloc(const void* x_bf16, const uint8_t* W_fp4, const uint8_t* W_sf,
                                   const float* gscale, const uint32_t* Ubits, const uint32_t* Vbits,
                                   const float* alpha, void* y_bf16, int M, int N, int K, int r,
                                   biloco_stream_t stream) {
  GemmArgs a;
  const int st = check_gemm_args(x_bf16, W_fp4, W_sf, gscale, Ubits, Vbits, alpha, y_bf16, M, N, K, r, &a);
  if (st) return st;
  if (N > BILOCO_NOALLOC_MAX_N) return BILOCO_ERR_SHAPE;
  const GemmPlan p = plan_gemm(a);
  if (p.need.counter_words > kCounterWordsMax) return BILOCO_ERR_SHAPE;

  // carve the shape-dependent regions behind the fixed header
  size_t off = kDataOff;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += round256(bytes);
    return at;
  };
  const size_t o_fp4 = take(p.need.act_fp4);
  const size_t o_sf = take(p.need.act_sf);
  const size_t o_zpart = take(p.need.zpart);
  const size_t o_zfin = take(p.need.zfin);
  const size_t o_slots = take(p.need.slots);
  if (off > kCap) return BILOCO_ERR_SHAPE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BILOCO_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceScratch* d = device_scratch(dev);
    if (!d) return BILOCO_ERR_CUDA;
    if (!d->zeroed) {
      // first call on this device: the status word and the counters start at zero
      if (cudaMemsetAsync(d->base, 0, kDataOff, s) != cudaSuccess) return BILOCO_ERR_CUDA;
      d->zeroed = true;
    }
    base = d->base;
  }

  Scratch sc;
  sc.device = dev;
  sc.stream = s;
  sc.base = base;
  sc.bytes = off;
  sc.status = reinterpret_cast<int*>(base + kStatusOff);
  sc.counters = reinterpret_cast<uint32_t*>(base + kCounterOff);
  sc.counter_words = p.need.counter_words;
  sc.act_fp4 = base + o_fp4;
  sc.act_sf = base + o_sf;
  sc.zpart = reinterpret_cast<float*>(base + o_zpart);
  sc.zfin = reinterpret_cast<float*>(base + o_zfin);
  sc.slots = reinterpret_cast<float*>(base + o_slots);
  return launch_gemm(a, p, sc, s);
}
