// Round-to-nearest quantizer kernels ("DL S067 - Quantization", sections 1-2;
// "Model Quantization", section 1).
//
//  * quant_asym_group<T, L>: groups of g = 8L consecutive weights (g in 32..256), L lanes
//    per group, 8 weights per lane in registers: one 16-B (bf16) or two 16-B (fp32)
//    coalesced loads, NaN-propagating min/max, an xor-shuffle reduction over the L lanes,
//    S'/Z computed exactly by every lane, codes packed 8 per 32-bit word and stored
//    coalesced (a warp writes 128 contiguous bytes).
//  * quant_asym_wide<T>: g > 256 (e.g. g = K, one scale per output channel): one warp per
//    group, two passes over the group (range, then codes; the second pass hits L2).
//  * quant_sym_int8_row<T>: symmetric INT8 with one scale per output row.
//  * per-tensor: a grid-wide min/max into the caller's workspace, then codes.
#include "common.cuh"
#include "kernels.h"

namespace wq {
namespace {

// Load 8 consecutive weights starting at p (16-byte aligned) as floats.
__device__ __forceinline__ void load8(const uint16_t* p, float v[8]) {
  uint4 u = ld_stream_u4(p);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
  v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
  v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}
__device__ __forceinline__ void load8(const float* p, float v[8]) {
  uint4 a = ld_stream_u4(p);
  uint4 b = ld_stream_u4(p + 4);
  v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
  v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
  v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
  v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
}

__device__ __forceinline__ void range8(const float v[8], float& mn, float& mx) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mn = fmin_nan(mn, v[i]);
    mx = fmax_nan(mx, v[i]);
  }
}

// Eight codes q = clip(RNE(w/S') + Z, 0, 15), nibble i of the result = code of v[i].
__device__ __forceinline__ uint32_t encode8(const float v[8], const AsymScale& sz) {
  uint32_t word = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float q = rne_quotient(v[i], sz.s, sz.inv_s) + sz.z;
    q = fminf(fmaxf(q, 0.0f), 15.0f);
    word |= static_cast<uint32_t>(__float2int_rz(q)) << (4 * i);
  }
  return word;
}

template <typename T, int L>
__global__ void __launch_bounds__(256)
quant_asym_group(const T* __restrict__ W, int64_t ldw, int N, int K,
                 uint8_t* __restrict__ packed, uint16_t* __restrict__ S,
                 uint16_t* __restrict__ Z, unsigned* status) {
  constexpr int kGroup = 8 * L;
  constexpr int kGroupsPerWarp = 32 / L;
  const int G = K / kGroup;
  const int64_t total = static_cast<int64_t>(N) * G;
  const int lane = threadIdx.x & 31;
  const int sub = lane % L;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;

  // Each lane walks groups t = t0, t0 + stride, ... with its (row n, group g) updated
  // incrementally (no 64-bit division in the loop).
  const int64_t stride = nwarps * kGroupsPerWarp;
  const int64_t stride_n = stride / G;
  const int stride_g = static_cast<int>(stride - stride_n * G);
  int64_t t = warp * kGroupsPerWarp + lane / L;
  int64_t n = t / G;
  int g = static_cast<int>(t - n * G);
  for (int64_t base = warp * kGroupsPerWarp; base < total; base += stride) {
    const bool active = t < total;
    float v[8];
    if (active) {
      load8(W + n * ldw + static_cast<int64_t>(g) * kGroup + sub * 8, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    }
    float mn = 0.0f, mx = 0.0f;  // the range always includes zero
    range8(v, mn, mx);
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) {
      mn = fmin_nan(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const AsymScale sz = asym_scale_zero(mn, mx);
    if (active) {
      const uint32_t word = encode8(v, sz);
      *reinterpret_cast<uint32_t*>(packed + n * (K / 2) + static_cast<int64_t>(g) * (kGroup / 2) +
                                   sub * 4) = word;
      if (sub == 0) {
        S[t] = static_cast<uint16_t>(sz.sbits);
        Z[t] = static_cast<uint16_t>(f32_to_f16_bits(sz.z));
        if (sz.bad) set_status(status, kStNonFinite);
      }
    }
    t += stride;
    n += stride_n;
    g += stride_g;
    if (g >= G) {
      g -= G;
      ++n;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
quant_asym_wide(const T* __restrict__ W, int64_t ldw, int N, int K, int group,
                uint8_t* __restrict__ packed, uint16_t* __restrict__ S,
                uint16_t* __restrict__ Z, unsigned* status) {
  const int G = K / group;
  const int64_t total = static_cast<int64_t>(N) * G;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t t = warp; t < total; t += nwarps) {
    const int64_t n = t / G;
    const int g = static_cast<int>(t - n * G);
    const T* src = W + n * ldw + static_cast<int64_t>(g) * group;
    float mn = 0.0f, mx = 0.0f;
    for (int k = lane * 8; k < group; k += 256) {
      float v[8];
      load8(src + k, v);
      range8(v, mn, mx);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fmin_nan(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const AsymScale sz = asym_scale_zero(mn, mx);
    uint8_t* dst = packed + n * (K / 2) + static_cast<int64_t>(g) * (group / 2);
    for (int k = lane * 8; k < group; k += 256) {
      float v[8];
      load8(src + k, v);
      *reinterpret_cast<uint32_t*>(dst + k / 2) = encode8(v, sz);
    }
    if (lane == 0) {
      S[t] = static_cast<uint16_t>(sz.sbits);
      Z[t] = static_cast<uint16_t>(f32_to_f16_bits(sz.z));
      if (sz.bad) set_status(status, kStNonFinite);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
quant_sym_int8_row(const T* __restrict__ W, int64_t ldw, int N, int K,
                   int8_t* __restrict__ codes, uint16_t* __restrict__ S, unsigned* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t n = warp; n < N; n += nwarps) {
    const T* src = W + n * ldw;
    float amax = 0.0f;
    for (int k = lane * 8; k < K; k += 256) {
      float v[8];
      load8(src + k, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmax_nan(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmax_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const AsymScale sc = sym_scale(amax, 127.0f);
    int8_t* dst = codes + n * K;
    for (int k = lane * 8; k < K; k += 256) {
      float v[8];
      load8(src + k, v);
      uint32_t w0 = 0, w1 = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float q = rne_quotient(v[i], sc.s, sc.inv_s);
        q = fminf(fmaxf(q, -127.0f), 127.0f);
        uint32_t b = static_cast<uint32_t>(__float2int_rz(q)) & 0xFFu;
        if (i < 4) w0 |= b << (8 * i); else w1 |= b << (8 * (i - 4));
      }
      *reinterpret_cast<uint2*>(dst + k) = make_uint2(w0, w1);
    }
    if (lane == 0) {
      S[n] = static_cast<uint16_t>(sc.sbits);
      if (sc.bad) set_status(status, kStNonFinite);
    }
  }
}

// ---- per-tensor: pass 1 (grid-wide range), pass 2 (codes)

template <typename T>
__global__ void __launch_bounds__(256)
range_partials(const T* __restrict__ W, int64_t ldw, int N, int K, float2* __restrict__ part) {
  const int64_t chunks_per_row = K / 8;
  const int64_t total = static_cast<int64_t>(N) * chunks_per_row;
  float mn = 0.0f, mx = 0.0f;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < total;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = c / chunks_per_row;
    const int64_t k = (c - n * chunks_per_row) * 8;
    float v[8];
    load8(W + n * ldw + k, v);
    range8(v, mn, mx);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fmin_nan(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  __shared__ float2 red[8];
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = make_float2(mn, mx);
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (blockDim.x >> 5); ++w) {
      mn = fmin_nan(mn, red[w].x);
      mx = fmax_nan(mx, red[w].y);
    }
    part[blockIdx.x] = make_float2(mn, mx);
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
encode_per_tensor(const T* __restrict__ W, int64_t ldw, int N, int K,
                  const float2* __restrict__ part, int nparts, uint8_t* __restrict__ packed,
                  uint16_t* __restrict__ S, uint16_t* __restrict__ Z, unsigned* status) {
  __shared__ AsymScale sh;
  if (threadIdx.x < 32) {
    float mn = 0.0f, mx = 0.0f;
    for (int i = threadIdx.x; i < nparts; i += 32) {
      float2 p = part[i];
      mn = fmin_nan(mn, p.x);
      mx = fmax_nan(mx, p.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fmin_nan(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (threadIdx.x == 0) {
      sh = asym_scale_zero(mn, mx);
      if (blockIdx.x == 0) {
        S[0] = static_cast<uint16_t>(sh.sbits);
        Z[0] = static_cast<uint16_t>(f32_to_f16_bits(sh.z));
        if (sh.bad) set_status(status, kStNonFinite);
      }
    }
  }
  __syncthreads();
  const AsymScale sz = sh;
  const int64_t chunks_per_row = K / 8;
  const int64_t total = static_cast<int64_t>(N) * chunks_per_row;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < total;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = c / chunks_per_row;
    const int64_t k = (c - n * chunks_per_row) * 8;
    float v[8];
    load8(W + n * ldw + k, v);
    *reinterpret_cast<uint32_t*>(packed + n * (K / 2) + k / 2) = encode8(v, sz);
  }
}

int grid_for(int64_t work_items, int per_block, int sms) {
  int64_t blocks = (work_items + per_block - 1) / per_block;
  int64_t cap = static_cast<int64_t>(sms) * 8;
  if (blocks > cap) blocks = cap;
  return static_cast<int>(blocks < 1 ? 1 : blocks);
}

template <typename T>
cudaError_t launch_quant_asym_t(const T* W, int64_t ldw, int N, int K, int group,
                                uint8_t* packed, uint16_t* S, uint16_t* Z, unsigned* status,
                                int sms, cudaStream_t st) {
  const int64_t groups = static_cast<int64_t>(N) * (K / group);
  switch (group) {
    case 32: quant_asym_group<T, 4><<<grid_for(groups, 64, sms), 256, 0, st>>>(W, ldw, N, K, packed, S, Z, status); break;
    case 64: quant_asym_group<T, 8><<<grid_for(groups, 32, sms), 256, 0, st>>>(W, ldw, N, K, packed, S, Z, status); break;
    case 128: quant_asym_group<T, 16><<<grid_for(groups, 16, sms), 256, 0, st>>>(W, ldw, N, K, packed, S, Z, status); break;
    case 256: quant_asym_group<T, 32><<<grid_for(groups, 8, sms), 256, 0, st>>>(W, ldw, N, K, packed, S, Z, status); break;
    default: quant_asym_wide<T><<<grid_for(groups, 8, sms), 256, 0, st>>>(W, ldw, N, K, group, packed, S, Z, status); break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_asym(const void* W, bool bf16, int64_t ldw, int N, int K, int group,
                              uint8_t* packed, uint16_t* S, uint16_t* Z, unsigned* status,
                              int sms, cudaStream_t st) {
  if (bf16)
    return launch_quant_asym_t(static_cast<const uint16_t*>(W), ldw, N, K, group, packed, S, Z,
                               status, sms, st);
  return launch_quant_asym_t(static_cast<const float*>(W), ldw, N, K, group, packed, S, Z,
                             status, sms, st);
}

cudaError_t launch_quant_sym_int8(const void* W, bool bf16, int64_t ldw, int N, int K,
                                  int8_t* codes, uint16_t* S, unsigned* status, int sms,
                                  cudaStream_t st) {
  const int grid = grid_for(N, 8, sms);
  if (bf16)
    quant_sym_int8_row<uint16_t><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(W), ldw, N,
                                                       K, codes, S, status);
  else
    quant_sym_int8_row<float><<<grid, 256, 0, st>>>(static_cast<const float*>(W), ldw, N, K,
                                                    codes, S, status);
  return cudaGetLastError();
}

int per_tensor_parts(int sms) { return sms * 8; }

cudaError_t launch_quant_per_tensor(const void* W, bool bf16, int64_t ldw, int N, int K,
                                    uint8_t* packed, uint16_t* S, uint16_t* Z, float2* part,
                                    int nparts, unsigned* status, cudaStream_t st) {
  if (bf16) {
    const uint16_t* w = static_cast<const uint16_t*>(W);
    range_partials<uint16_t><<<nparts, 256, 0, st>>>(w, ldw, N, K, part);
    encode_per_tensor<uint16_t><<<nparts, 256, 0, st>>>(w, ldw, N, K, part, nparts, packed, S, Z,
                                                        status);
  } else {
    const float* w = static_cast<const float*>(W);
    range_partials<float><<<nparts, 256, 0, st>>>(w, ldw, N, K, part);
    encode_per_tensor<float><<<nparts, 256, 0, st>>>(w, ldw, N, K, part, nparts, packed, S, Z,
                                                     status);
  }
  return cudaGetLastError();
}

}  // namespace wq
