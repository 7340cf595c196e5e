// C ABI of libwq (declared in include/wq.h): argument validation, kernel choice by shape,
// the device status word. No device memory is allocated here.
#include <initializer_list>
#include <mutex>

#include "../../include/wq.h"
#include "common.cuh"
#include "kernels.h"
#include "tc_gemm.h"

namespace {

__device__ unsigned g_wq_status;  // per-device status word (bits wq::kSt*)

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool ok = false;             // set once the queries below have succeeded
  int sms = 0;
  unsigned* status = nullptr;  // device address of g_wq_status on that device
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Current device's cached info (SM count, status-word address); nullptr if unusable. Only
// a successful set of queries is kept: a failure (no device, not sm_100, a lookup refused
// during a stream capture) is returned as is and retried by the next call.
const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ok) {
    int major = 0, minor = 0, sms = 0;
    void* addr = nullptr;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        major == 10 && minor == 0 && cudaGetSymbolAddress(&addr, g_wq_status) == cudaSuccess) {
      d.sms = sms;
      d.status = static_cast<unsigned*>(addr);
      d.ok = true;
    } else {
      cudaGetLastError();
    }
  }
  return d.ok ? &d : nullptr;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Every non-null pointer is device memory of the current device, or managed memory.
bool on_current_device(std::initializer_list<const void*> ptrs) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  for (const void* p : ptrs) {
    if (!p) continue;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    if (at.type == cudaMemoryTypeManaged) continue;
    if (at.type != cudaMemoryTypeDevice || at.device != dev) return false;
  }
  return true;
}

wq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA; }

bool fits_int(int64_t v) { return v >= 0 && v <= 0x7fffffffLL; }

}  // namespace

namespace wq {
bool pointers_on_current_device(std::initializer_list<const void*> ptrs) {
  return on_current_device(ptrs);
}

bool current_device(int* sms, unsigned** status) {
  const DeviceInfo* d = device_info();
  if (!d) return false;
  *sms = d->sms;
  *status = d->status;
  return true;
}
}  // namespace wq

extern "C" {

int32_t wq_version(void) { return WQ_VERSION; }

const char* wq_status_string(wq_status s) {
  switch (s) {
    case WQ_OK: return "ok";
    case WQ_ERR_NULL: return "a required pointer is NULL";
    case WQ_ERR_SHAPE: return "invalid sizes (N, K, M, group, leading dimension) or alpha";
    case WQ_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
    case WQ_ERR_DTYPE: return "dtype not supported by this call";
    case WQ_ERR_UNSUPPORTED: return "parameter combination not supported";
    case WQ_ERR_CUDA: return "CUDA runtime error";
    case WQ_ERR_NONFINITE: return "non-finite weight or scale overflow";
    case WQ_ERR_TIMEOUT: return "device wait timed out";
    case WQ_ERR_RANGE: return "code above 15, or a scale factor not finite and positive";
    case WQ_ERR_NODEVICE: return "no usable sm_100 CUDA device";
    case WQ_ERR_DEVICE: return "a pointer is not memory of the current device";
  }
  return "unknown status";
}

wq_status wq_quantize_rtn_g128(const void* W, wq_dtype w_dtype, int64_t N, int64_t K,
                               int64_t ldw, const wq_qparams* params, uint8_t* packed,
                               uint16_t* S, uint16_t* Z, void* stream) {
  const wq_qparams p = params ? *params : wq_qparams{4, 128, 1};
  if (N < 0 || K < 0) return WQ_ERR_SHAPE;
  if (w_dtype != WQ_F32 && w_dtype != WQ_BF16) return WQ_ERR_DTYPE;
  const bool int4 = p.w_bit == 4 && (p.zero_point == 1 || p.zero_point == 0);
  const bool int8 = p.w_bit == 8 && p.zero_point == 0;
  if (!int4 && !int8) return WQ_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return WQ_OK;
  if (!W || !packed || !S || (int4 && !Z)) return WQ_ERR_NULL;
  if (int8 && Z) return WQ_ERR_UNSUPPORTED;
  if (!fits_int(N) || !fits_int(K) || K % 32 != 0 || ldw < K) return WQ_ERR_SHAPE;
  if (int4 && (p.group < 32 || p.group % 32 != 0 || K % p.group != 0)) return WQ_ERR_SHAPE;
  if (int8 && p.group != K) return WQ_ERR_UNSUPPORTED;
  const size_t es = w_dtype == WQ_F32 ? 4 : 2;
  if (!aligned(W, 16) || (ldw * es) % 16 != 0 || !aligned(packed, 16) || !aligned(S, 2) ||
      (Z && !aligned(Z, 2)))
    return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({W, packed, S, Z})) return WQ_ERR_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf16 = w_dtype == WQ_BF16;
  if (int4)
    return from_cuda(wq::launch_quant_asym(W, bf16, ldw, (int)N, (int)K, p.group, packed, S, Z,
                                           p.zero_point == 0, d->status, d->sms, st));
  return from_cuda(wq::launch_quant_sym_int8(W, bf16, ldw, (int)N, (int)K,
                                             reinterpret_cast<int8_t*>(packed), S, d->status,
                                             d->sms, st));
}

size_t wq_quantize_per_tensor_workspace_bytes(int64_t N, int64_t K) {
  (void)N;
  (void)K;
  const DeviceInfo* d = device_info();
  const int sms = d ? d->sms : 148;
  return static_cast<size_t>(wq::per_tensor_parts(sms)) * sizeof(float2);
}

wq_status wq_quantize_rtn_per_tensor(const void* W, wq_dtype w_dtype, int64_t N, int64_t K,
                                     int64_t ldw, uint8_t* packed, uint16_t* S, uint16_t* Z,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  if (N < 0 || K < 0) return WQ_ERR_SHAPE;
  if (w_dtype != WQ_F32 && w_dtype != WQ_BF16) return WQ_ERR_DTYPE;
  if (N == 0 || K == 0) return WQ_OK;
  if (!W || !packed || !S || !Z || !workspace) return WQ_ERR_NULL;
  if (!fits_int(N) || !fits_int(K) || K % 32 != 0 || ldw < K) return WQ_ERR_SHAPE;
  const size_t es = w_dtype == WQ_F32 ? 4 : 2;
  if (!aligned(W, 16) || (ldw * es) % 16 != 0 || !aligned(packed, 16) || !aligned(S, 2) ||
      !aligned(Z, 2) || !aligned(workspace, 16))
    return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({W, packed, S, Z, workspace})) return WQ_ERR_DEVICE;
  const int nparts = wq::per_tensor_parts(d->sms);
  if (workspace_bytes < static_cast<size_t>(nparts) * sizeof(float2)) return WQ_ERR_SHAPE;
  return from_cuda(wq::launch_quant_per_tensor(
      W, w_dtype == WQ_BF16, ldw, (int)N, (int)K, packed, S, Z, static_cast<float2*>(workspace),
      nparts, d->status, static_cast<cudaStream_t>(stream)));
}

wq_status wq_pack_int4(const uint8_t* codes, int64_t N, int64_t K, uint8_t* packed,
                       void* stream) {
  if (N < 0 || K < 0) return WQ_ERR_SHAPE;
  if (N == 0 || K == 0) return WQ_OK;
  if (!codes || !packed) return WQ_ERR_NULL;
  if (K % 32 != 0) return WQ_ERR_SHAPE;
  if (!aligned(codes, 16) || !aligned(packed, 16)) return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({codes, packed})) return WQ_ERR_DEVICE;
  return from_cuda(wq::launch_pack_int4(codes, N, K, packed, d->status, d->sms,
                                        static_cast<cudaStream_t>(stream)));
}

wq_status wq_dequant(const uint8_t* packed, const uint16_t* S, const uint16_t* Z, int64_t N,
                     int64_t K, int32_t group, void* out, wq_dtype out_dtype, void* stream) {
  if (N < 0 || K < 0) return WQ_ERR_SHAPE;
  if (out_dtype != WQ_F32 && out_dtype != WQ_BF16) return WQ_ERR_DTYPE;
  if (N == 0 || K == 0) return WQ_OK;
  if (!packed || !S || !Z || !out) return WQ_ERR_NULL;
  if (!fits_int(K) || K % 32 != 0) return WQ_ERR_SHAPE;
  if (group != 0 && (group < 32 || group % 32 != 0 || K % group != 0)) return WQ_ERR_SHAPE;
  if (!aligned(packed, 16) || !aligned(out, 16) || !aligned(S, 2) || !aligned(Z, 2))
    return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({packed, S, Z, out})) return WQ_ERR_DEVICE;
  const int g = group ? group : (int)K;
  const int sz_row = group ? (int)(K / group) : 0;
  return from_cuda(wq::launch_dequant(packed, S, Z, N, (int)K, g, sz_row, out,
                                      out_dtype == WQ_BF16, d->sms,
                                      static_cast<cudaStream_t>(stream)));
}

// Token counts up to which the decode kernels (in passes of at most 8 tokens, at most
// kMaxPasses of them) beat the tensor-core GEMM, whose tiles are too few for small M.
constexpr int64_t kSkinnyMaxM = 32;
// From this many tokens on (to 64, g = 128) the skinny tensor-core kernel takes the call;
// below it only where the decode kernels would pass over the weights more than once.
constexpr int64_t kTcSkinnyMinM = 9;
constexpr int64_t kMaxPasses = 8;

wq_status wq_w4a16_gemm(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* packed,
                        const uint16_t* S, const uint16_t* Z, int64_t N, int64_t K,
                        int32_t group, uint16_t* Y, int64_t ldy, void* stream) {
  if (M < 0 || N < 0 || K <= 0) return WQ_ERR_SHAPE;
  if (M == 0 || N == 0) return WQ_OK;
  if (!X || !packed || !S || !Z || !Y) return WQ_ERR_NULL;
  if (!fits_int(M) || !fits_int(N) || !fits_int(K) || K % 32 != 0 || ldx < K || ldy < N)
    return WQ_ERR_SHAPE;
  if (group != 0 && (group < 32 || group % 32 != 0 || K % group != 0)) return WQ_ERR_SHAPE;
  if (!aligned(X, 16) || ldx % 8 != 0 || !aligned(packed, 16) || !aligned(S, 2) ||
      !aligned(Z, 2) || !aligned(Y, 2))
    return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({X, packed, S, Z, Y})) return WQ_ERR_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int g = group ? group : (int)K;
  const int sz_row = group ? (int)(K / group) : 0;
  wq::GemvArgs a{X, ldx, packed, S, Z, (int)(M < 8 ? M : 8), (int)N, (int)K, g, sz_row, Y,
                 ldy, d->status};
  // 3..64 tokens, g = 128: one pass over the weights on the tensor core, from
  // kTcSkinnyMinM tokens on, or wherever the decode kernels would need more than one pass
  // over blocks of tokens (long rows at small M)
  if (M >= 3 && M <= wq::kSkinnyMaxTokens) {
    wq::GemvArgs t = a;
    t.M = static_cast<int>(M);
    if (wq::tc_skinny_ok(t) && (M >= kTcSkinnyMinM || wq::gemv_fast_block(a) < M)) {
      const cudaError_t e = wq::launch_tc_skinny(t, d->sms, st);
      if (e != cudaErrorInvalidValue) return from_cuda(e);
    }
  }
  // M = 1 beyond the register-loaded kernels' K only where the streaming kernel takes it
  if (M <= kSkinnyMaxM &&
      (M > 1 || K <= wq::gemv_max_k() || wq::gemv_imma_bulk_ok(a) || wq::gemv_tma_ok(a) ||
       (wq::gemv_stream_ok(a) && wq::gemv_stream_fits(a)))) {
    // Small M: the decode kernels, in passes over blocks of tokens when the whole of M has
    // no fast kernel (the weights come from HBM once; later passes find them in L2).
    const int b = wq::gemv_fast_block(a);
    if (b > 0 && (M + b - 1) / b <= kMaxPasses) {
      for (int64_t m0 = 0; m0 < M; m0 += b) {
        wq::GemvArgs p = a;
        p.X = X + m0 * ldx;
        p.Y = Y + m0 * ldy;
        p.M = static_cast<int>(M - m0 < b ? M - m0 : b);
        const wq_status e = from_cuda(wq::launch_gemv_w4a16(p, d->sms, st));
        if (e != WQ_OK) return e;
      }
      return WQ_OK;
    }
    if (M <= 8) {
      a.M = (int)M;
      return from_cuda(wq::launch_gemv_w4a16(a, d->sms, st));
    }
  }
  wq::TcGemmArgs t{X, ldx, packed, S, Z, nullptr, (int)M, (int)N, (int)K, g, sz_row, Y, ldy};
  return wq::launch_tc_gemm(t, d->sms, d->status, st);
}

wq_status wq_w8a16_gemm(const uint16_t* X, int64_t M, int64_t ldx, const int8_t* codes,
                        const uint16_t* S, int64_t N, int64_t K, uint16_t* Y, int64_t ldy,
                        void* stream) {
  if (M < 0 || N < 0 || K <= 0) return WQ_ERR_SHAPE;
  if (M == 0 || N == 0) return WQ_OK;
  if (!X || !codes || !S || !Y) return WQ_ERR_NULL;
  if (!fits_int(M) || !fits_int(N) || !fits_int(K) || K % 32 != 0 || ldx < K || ldy < N)
    return WQ_ERR_SHAPE;
  if (!aligned(X, 16) || ldx % 8 != 0 || !aligned(codes, 16) || !aligned(S, 2) ||
      !aligned(Y, 2))
    return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({X, codes, S, Y})) return WQ_ERR_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // 3 to 64 tokens: the skinny tensor-core kernel on the s8 codes as they are (one or two
  // tokens stream faster through the row kernel below: 7B step at M = 1 37 us against 49)
  if (M >= 3 && M <= wq::kSkinnyMaxTokens) {
    wq::GemvArgs t{X, ldx, reinterpret_cast<const uint8_t*>(codes), S, nullptr, (int)M, (int)N,
                   (int)K, (int)K, 1, Y, ldy, d->status};
    if (wq::tc_skinny8_ok(t)) {
      const cudaError_t e = wq::launch_tc_skinny8(t, d->sms, st);
      if (e != cudaErrorInvalidValue) return from_cuda(e);
    }
  }
  if (M <= 8) {
    wq::Gemv8Args a{X, ldx, codes, S, (int)M, (int)N, (int)K, Y, ldy};
    return from_cuda(wq::launch_gemv_w8a16(a, st));
  }
  wq::TcGemmArgs a{X, ldx, nullptr, S, nullptr, codes, (int)M, (int)N, (int)K, (int)K, 1, Y, ldy};
  return wq::launch_tc_gemm(a, d->sms, d->status, st);
}

wq_status wq_channel_stat(const void* A, wq_dtype dtype, int64_t rows, int64_t cols,
                          int64_t lda, int32_t stat, float* out, void* stream) {
  if (rows < 0 || cols < 0) return WQ_ERR_SHAPE;
  if (dtype != WQ_F32 && dtype != WQ_BF16) return WQ_ERR_DTYPE;
  if (stat != WQ_STAT_ABSMAX && stat != WQ_STAT_ABSMEAN) return WQ_ERR_UNSUPPORTED;
  if (cols == 0) return WQ_OK;
  if (rows == 0) return WQ_ERR_SHAPE;  // a statistic over no rows
  if (!A || !out) return WQ_ERR_NULL;
  if (!fits_int(cols) || cols % 8 != 0 || lda < cols) return WQ_ERR_SHAPE;
  const size_t es = dtype == WQ_F32 ? 4 : 2;
  if (!aligned(A, 16) || (lda * es) % 16 != 0 || !aligned(out, 4)) return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({A, out})) return WQ_ERR_DEVICE;
  return from_cuda(wq::launch_channel_stat(A, dtype == WQ_BF16, lda, rows, (int)cols,
                                           stat == WQ_STAT_ABSMEAN, out, d->sms,
                                           static_cast<cudaStream_t>(stream)));
}

// alpha in [0, 1] (the migration strength / the AWQ exponent).
static bool alpha_ok(float alpha) { return alpha >= 0.0f && alpha <= 1.0f; }

wq_status wq_smooth_scales(const float* xmax, const float* wmax, int64_t K, float alpha,
                           float* s, void* stream) {
  if (K < 0 || !alpha_ok(alpha)) return WQ_ERR_SHAPE;
  if (K == 0) return WQ_OK;
  if (!xmax || !wmax || !s) return WQ_ERR_NULL;
  if (!fits_int(K)) return WQ_ERR_SHAPE;
  if (!aligned(xmax, 4) || !aligned(wmax, 4) || !aligned(s, 4)) return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({xmax, wmax, s})) return WQ_ERR_DEVICE;
  return from_cuda(wq::launch_smooth_scales(xmax, wmax, (int)K, alpha, s, d->sms,
                                            static_cast<cudaStream_t>(stream)));
}

wq_status wq_awq_scales(const float* a_mag, int64_t K, float alpha, float* s, void* stream) {
  if (K < 0 || !alpha_ok(alpha)) return WQ_ERR_SHAPE;
  if (K == 0) return WQ_OK;
  if (!a_mag || !s) return WQ_ERR_NULL;
  if (!fits_int(K)) return WQ_ERR_SHAPE;
  if (!aligned(a_mag, 4) || !aligned(s, 4)) return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({a_mag, s})) return WQ_ERR_DEVICE;
  return from_cuda(wq::launch_awq_scales(a_mag, (int)K, alpha, s,
                                         static_cast<cudaStream_t>(stream)));
}

wq_status wq_quantize_rtn_scaled(const void* W, wq_dtype w_dtype, int64_t N, int64_t K,
                                 int64_t ldw, const float* s, const wq_qparams* params,
                                 uint8_t* packed, uint16_t* S, uint16_t* Z, void* stream) {
  const wq_qparams p = params ? *params : wq_qparams{4, 128, 1};
  if (N < 0 || K < 0) return WQ_ERR_SHAPE;
  if (w_dtype != WQ_F32 && w_dtype != WQ_BF16) return WQ_ERR_DTYPE;
  if (p.w_bit != 4 || (p.zero_point != 0 && p.zero_point != 1)) return WQ_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return WQ_OK;
  if (!W || !s || !packed || !S || !Z) return WQ_ERR_NULL;
  if (!fits_int(N) || !fits_int(K) || K % 32 != 0 || ldw < K) return WQ_ERR_SHAPE;
  if (p.group < 32 || p.group % 32 != 0 || K % p.group != 0) return WQ_ERR_SHAPE;
  const size_t es = w_dtype == WQ_F32 ? 4 : 2;
  if (!aligned(W, 16) || (ldw * es) % 16 != 0 || !aligned(s, 16) || !aligned(packed, 16) ||
      !aligned(S, 2) || !aligned(Z, 2))
    return WQ_ERR_ALIGN;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({W, s, packed, S, Z})) return WQ_ERR_DEVICE;
  return from_cuda(wq::launch_quant_scaled(W, w_dtype == WQ_BF16, ldw, (int)N, (int)K, p.group,
                                           s, packed, S, Z, p.zero_point == 0, d->status,
                                           d->sms, static_cast<cudaStream_t>(stream)));
}

wq_status wq_scale_activations(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                               const float* s, uint16_t* Xs, int64_t ldxs, void* stream) {
  if (M < 0 || K < 0) return WQ_ERR_SHAPE;
  if (M == 0 || K == 0) return WQ_OK;
  if (!X || !s || !Xs) return WQ_ERR_NULL;
  if (!fits_int(M) || !fits_int(K) || K % 8 != 0 || ldx < K || ldxs < K) return WQ_ERR_SHAPE;
  if (!aligned(X, 16) || !aligned(Xs, 16) || !aligned(s, 16) || ldx % 8 != 0 || ldxs % 8 != 0)
    return WQ_ERR_ALIGN;
  if (X == Xs && ldx != ldxs) return WQ_ERR_UNSUPPORTED;  // in place only row for row
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({X, s, Xs})) return WQ_ERR_DEVICE;
  return from_cuda(wq::launch_scale_activations(X, ldx, (int)M, (int)K, s, Xs, ldxs, d->sms,
                                                static_cast<cudaStream_t>(stream)));
}

size_t wq_gptq_workspace_bytes(int64_t N, int64_t K) {
  (void)N;
  return K > 0 ? wq::gptq_workspace_bytes(K) : 0;
}

wq_status wq_quantize_gptq(const void* W, wq_dtype w_dtype, int64_t N, int64_t K, int64_t ldw,
                           const uint16_t* X, int64_t T, int64_t ldx, double damp,
                           const wq_qparams* params, uint8_t* packed, uint16_t* S, uint16_t* Z,
                           void* workspace, size_t workspace_bytes, void* stream) {
  const wq_qparams p = params ? *params : wq_qparams{4, 128, 1};
  if (N < 0 || K < 0 || T < 0) return WQ_ERR_SHAPE;
  if (w_dtype != WQ_F32 && w_dtype != WQ_BF16) return WQ_ERR_DTYPE;
  if (p.w_bit != 4 || (p.zero_point != 0 && p.zero_point != 1)) return WQ_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return WQ_OK;
  if (!W || !X || !packed || !S || !Z || !workspace) return WQ_ERR_NULL;
  if (!fits_int(N) || !fits_int(K) || !fits_int(T) || T == 0 || K % 64 != 0 || ldw < K ||
      ldx < K || !(damp >= 0.0 && damp <= 1e6))
    return WQ_ERR_SHAPE;
  if (p.group < 32 || p.group % 32 != 0 || K % p.group != 0) return WQ_ERR_SHAPE;
  if (K > wq::gptq_max_k()) return WQ_ERR_UNSUPPORTED;
  const size_t es = w_dtype == WQ_F32 ? 4 : 2;
  if (!aligned(W, 16) || (ldw * es) % 16 != 0 || !aligned(packed, 16) || !aligned(S, 2) ||
      !aligned(Z, 2) || !aligned(X, 2) || !aligned(workspace, 16))
    return WQ_ERR_ALIGN;
  if (workspace_bytes < wq::gptq_workspace_bytes(K)) return WQ_ERR_SHAPE;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  if (!on_current_device({W, X, packed, S, Z, workspace})) return WQ_ERR_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf16 = w_dtype == WQ_BF16;
  // the grid: round-to-nearest S' and Z of the original weights (its codes are replaced)
  cudaError_t e = wq::launch_quant_asym(W, bf16, ldw, (int)N, (int)K, p.group, packed, S, Z,
                                        p.zero_point == 0, d->status, d->sms, st);
  if (e != cudaSuccess) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_gptq(W, bf16, ldw, (int)N, (int)K, p.group, X, ldx, (int)T, damp,
                                   packed, S, Z, workspace, d->status, d->sms, st));
}

wq_status wq_selftest_bounded_wait(uint64_t limit_ns, int32_t spin, void* stream) {
  if (limit_ns < 1000u || limit_ns > 1000000000u) return WQ_ERR_SHAPE;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  return from_cuda(wq::launch_bounded_wait_selftest(limit_ns, spin != 0, d->status,
                                                    static_cast<cudaStream_t>(stream)));
}

wq_status wq_get_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WQ_ERR_CUDA;
  const DeviceInfo* d = device_info();
  if (!d) return WQ_ERR_NODEVICE;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_wq_status, sizeof(v)) != cudaSuccess) return WQ_ERR_CUDA;
  if (v != 0) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_wq_status, &zero, sizeof(zero)) != cudaSuccess) return WQ_ERR_CUDA;
  }
  if (v & wq::kStNonFinite) return WQ_ERR_NONFINITE;
  if (v & wq::kStRange) return WQ_ERR_RANGE;
  if (v & wq::kStTimeout) return WQ_ERR_TIMEOUT;
  return WQ_OK;
}

}  // extern "C"
