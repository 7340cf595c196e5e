// Packing of 4-bit codes two per byte and dequantization W_hat = S'(q - Z)
// ("Model Quantization", sections 1 and 4: INT4 weights with FP16 scales/zero-points).
// Both are HBM-streaming kernels: one thread per 32 codes, 16-byte loads and stores.
#include "common.cuh"
#include "kernels.h"

namespace wq {
namespace {

// codes [N, K] uint8 -> packed [N, K/2]; byte j = c[2j] | c[2j+1] << 4.
__global__ void __launch_bounds__(256)
pack_int4_kernel(const uint8_t* __restrict__ codes, int64_t total32,
                 uint8_t* __restrict__ packed, unsigned* status) {
  bool bad = false;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total32;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 a = ld_stream_u4(codes + i * 32);
    const uint4 b = ld_stream_u4(codes + i * 32 + 16);
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t u = in[2 * j], v = in[2 * j + 1];
      bad |= ((u | v) & 0xF0F0F0F0u) != 0u;
      // bytes c0..c3 of u and c4..c7 of v -> nibbles 0..7 of the result
      const uint32_t lo = (u & 0x0000000Fu) | ((u >> 4) & 0x000000F0u) |
                          ((u >> 8) & 0x00000F00u) | ((u >> 12) & 0x0000F000u);
      const uint32_t hi = (v & 0x0000000Fu) | ((v >> 4) & 0x000000F0u) |
                          ((v >> 8) & 0x00000F00u) | ((v >> 12) & 0x0000F000u);
      out[j] = (lo & 0xFFFFu) | (hi << 16);
    }
    *reinterpret_cast<uint4*>(packed + i * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (bad) set_status(status, kStRange);
}

// One thread per 32 codes (one 16-byte load); g is a multiple of 32 so the 32 codes
// share one (S', Z). sz_row = scales per row (0 for per-tensor), gshift = log2(g) or -1.
template <bool kBf16Out>
__global__ void __launch_bounds__(256)
dequant_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ S,
               const uint16_t* __restrict__ Z, int64_t N, int K, int group, int sz_row,
               void* __restrict__ out) {
  const int64_t per_row = K / 32;
  const int64_t total = N * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / per_row;
    const int k = static_cast<int>(i - n * per_row) * 32;
    const int64_t gi = n * sz_row + (sz_row ? k / group : 0);
    const float s = f16_bits_to_f32(ld_nc_u16(S + gi));
    const float z = f16_bits_to_f32(ld_nc_u16(Z + gi));
    const uint4 p = ld_stream_u4(packed + n * (K / 2) + k / 2);
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
    float w[32];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e)
        w[8 * j + e] = s * (static_cast<float>((words[j] >> (4 * e)) & 0xFu) - z);  // exact
    if (kBf16Out) {
      uint16_t* o = static_cast<uint16_t*>(out) + n * K + k;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 r;
        r.x = pack_bf16x2(w[8 * v + 0], w[8 * v + 1]);
        r.y = pack_bf16x2(w[8 * v + 2], w[8 * v + 3]);
        r.z = pack_bf16x2(w[8 * v + 4], w[8 * v + 5]);
        r.w = pack_bf16x2(w[8 * v + 6], w[8 * v + 7]);
        reinterpret_cast<uint4*>(o)[v] = r;
      }
    } else {
      float* o = static_cast<float*>(out) + n * K + k;
#pragma unroll
      for (int v = 0; v < 8; ++v)
        reinterpret_cast<float4*>(o)[v] =
            make_float4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
  }
}

int grid_cap(int64_t items, int sms) {
  int64_t b = (items + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  if (b > cap) b = cap;
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_pack_int4(const uint8_t* codes, int64_t N, int64_t K, uint8_t* packed,
                             unsigned* status, int sms, cudaStream_t st) {
  const int64_t total32 = N * K / 32;
  pack_int4_kernel<<<grid_cap(total32, sms), 256, 0, st>>>(codes, total32, packed, status);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* packed, const uint16_t* S, const uint16_t* Z,
                           int64_t N, int K, int group, int sz_row, void* out, bool bf16_out,
                           int sms, cudaStream_t st) {
  const int64_t items = N * (K / 32);
  if (bf16_out)
    dequant_kernel<true><<<grid_cap(items, sms), 256, 0, st>>>(packed, S, Z, N, K, group, sz_row,
                                                               out);
  else
    dequant_kernel<false><<<grid_cap(items, sms), 256, 0, st>>>(packed, S, Z, N, K, group, sz_row,
                                                                out);
  return cudaGetLastError();
}

}  // namespace wq
