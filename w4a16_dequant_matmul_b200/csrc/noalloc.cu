// Per-tensor INT4 quantization without any device allocation by the caller or the library.
//
// Who needs this: code that must not call cudaMalloc on the hot path. Examples are a
// plugin inside an inference engine that owns all device memory and hands plugins only
// their inputs and outputs, a framework whose caching allocator would be bypassed (and
// its pool fragmented) by a raw cudaMalloc, or a latency-critical loop where cudaMalloc's
// implicit device-wide synchronization is not acceptable. The regular per-tensor entry
// point needs a caller-provided workspace for its grid-wide min/max; this variant keeps
// that workspace in a fixed array in the library's own device memory instead.
//
// The scratch array g_noalloc_ranges lives for as long as the library is loaded, once on
// every GPU that loads it (32 KB each). Host code cannot use the array's name as a device
// address, so the address is looked up with cudaGetSymbolAddress once per device, with
// that device current, on the first call there; make that first call before any stream
// capture. Every call on a device shares the one array: calls that overlap on the GPU
// (for example on two streams at once) race on it and give wrong results. Nothing in it
// has to start at zero: the range pass writes every slot that the encode pass reads.
#include <mutex>

#include "../../include/wq.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int kNoAllocMaxRanges = 4096;  // (min, max) pairs: 32 KB
static __device__ __align__(256) float2 g_noalloc_ranges[kNoAllocMaxRanges];

constexpr int kMaxDevices = 64;
struct NoAllocDevice {
  float2* ranges = nullptr;  // device address of g_noalloc_ranges on this device, once known
};
NoAllocDevice g_na[kMaxDevices];
std::mutex g_na_mu;

// Device address of the scratch array on the current device (nullptr on failure). Only a
// successful lookup is kept, so a failed one (for example inside a stream capture) is
// retried by the next call instead of failing every later call on that device.
float2* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_na_mu);
  NoAllocDevice& d = g_na[dev];
  if (!d.ranges) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_ranges) == cudaSuccess && p != nullptr)
      d.ranges = static_cast<float2*>(p);
    else
      cudaGetLastError();  // clear the error of the failed lookup
  }
  return d.ranges;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" wq_status wq_quantize_rtn_per_tensor_noalloc(const void* W, wq_dtype w_dtype,
                                                        int64_t N, int64_t K, int64_t ldw,
                                                        uint8_t* packed, uint16_t* S,
                                                        uint16_t* Z, void* stream) {
  if (N < 0 || K < 0) return WQ_ERR_SHAPE;
  if (w_dtype != WQ_F32 && w_dtype != WQ_BF16) return WQ_ERR_DTYPE;
  if (N == 0 || K == 0) return WQ_OK;
  if (!W || !packed || !S || !Z) return WQ_ERR_NULL;
  if (N > 0x7fffffffLL || K > 0x7fffffffLL || K % 32 != 0 || ldw < K) return WQ_ERR_SHAPE;
  const size_t es = w_dtype == WQ_F32 ? 4 : 2;
  if (!aligned(W, 16) || (ldw * es) % 16 != 0 || !aligned(packed, 16) || !aligned(S, 2) ||
      !aligned(Z, 2))
    return WQ_ERR_ALIGN;
  int sms = 0;
  unsigned* status = nullptr;
  if (!wq::current_device(&sms, &status)) return WQ_ERR_NODEVICE;
  if (!wq::pointers_on_current_device({W, packed, S, Z})) return WQ_ERR_DEVICE;
  // The range pass uses one (min, max) slot per CTA, 8 CTAs per SM.
  const int nparts = wq::per_tensor_parts(sms);
  if (nparts > kNoAllocMaxRanges) return WQ_ERR_UNSUPPORTED;
  float2* ranges = scratch_address();
  if (!ranges) return WQ_ERR_CUDA;
  const cudaError_t e = wq::launch_quant_per_tensor(
      W, w_dtype == WQ_BF16, ldw, (int)N, (int)K, packed, S, Z, ranges, nparts, status,
      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}
