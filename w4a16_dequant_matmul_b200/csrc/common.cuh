// Device helpers shared by the libwq kernels: exact roundings used by the quantizer,
// bit-level conversions, streaming loads, and the device status word bits.
//
// Numerics (see "DL S067 - Quantization", section 1 "The core math"): the stored scale
// is the binary16 round-half-even of the EXACT (beta - alpha)/15, and codes are the
// round-half-even of the EXACT quotient w/S'. Both are decided here with exact sign
// tests (FMA residuals, float64 differences), so that they agree bit for bit with any
// correct implementation of the definition, whatever the reciprocal's accuracy.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

// Let kernel `kern` use `bytes` of dynamic shared memory, with all of the SM's unified L1 /
// shared memory configured as shared memory. Every large-shared-memory kernel of the library
// asks for the same split, so consecutive launches of different kernels on a stream do not
// make an SM change its split between them (which needs the SM to drain first).
template <typename F>
inline cudaError_t set_smem_attrs(F* kern, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  return e;
}

// Bits of the device status word (see wq_get_status).
enum : unsigned { kStNonFinite = 1u, kStRange = 2u, kStTimeout = 4u };

__device__ __forceinline__ void set_status(unsigned* st, unsigned bit) {
  atomicOr(st, bit);
}

__device__ __forceinline__ float f16_bits_to_f32(unsigned b) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
}

__device__ __forceinline__ unsigned f32_to_f16_bits(float v) {
  return __half_as_ushort(__float2half_rn(v));
}

// NaN-propagating min / max (a NaN weight must not vanish in the range reduction).
__device__ __forceinline__ float fmin_nan(float a, float b) {
  float d;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// 16-byte read-only streaming load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// 16-byte read-only load through L1 (for small operands reused by many warps).
__device__ __forceinline__ uint4 ld_nc_u4(const void* p) {
  uint4 r;
  asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ unsigned short ld_nc_u16(const void* p) {
  unsigned short r;
  asm("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

// Value of a binary16 bit pattern in [0, 0x7C00]; 0x7C00 stands for 2^16 (the value the
// rounding would produce one step above the largest finite 65504).
__device__ __forceinline__ float f16_grid_value(unsigned b) {
  return b >= 0x7C00u ? 65536.0f : f16_bits_to_f32(b);
}

// Sign of (hi + lo) - div*m, exactly: div*m is exact in float64 (m has <= 12 significant
// bits, div <= 127); hi - div*m is exact in float64 whenever the two are within a factor
// 2^29 of each other, and otherwise its sign is not in doubt; adding lo keeps the sign.
__device__ __forceinline__ double exact_diff(float hi, float lo, float div, float m) {
  return ((double)hi - (double)div * (double)m) + (double)lo;
}

// binary16 bit pattern of round-half-even((hi + lo) / div), where hi >= 0 is finite and lo
// is the exact rounding error of hi (hi + lo is the exact value); rdiv = 1/div rounded to
// float. 0x7C00 means overflow.
static __device__ __noinline__ unsigned rne_f16_of_quotient(float hi, float lo, float div,
                                                            float rdiv) {
  // Candidate: hi * rdiv is within 2^-23 relative of the quotient, so its binary16
  // rounding is within one binary16 step of the answer; the two midpoint tests fix it.
  unsigned b = __half_as_ushort(__float2half_rn(__fmul_rn(hi, rdiv)));
  if (b < 0x7C00u) {
    float m = 0.5f * (f16_grid_value(b) + f16_grid_value(b + 1));
    double d = exact_diff(hi, lo, div, m);
    if (d > 0.0 || (d == 0.0 && ((b + 1u) & 1u) == 0u)) return b + 1u;
  }
  if (b > 0u) {
    float m = 0.5f * (f16_grid_value(b - 1) + f16_grid_value(b));
    double d = exact_diff(hi, lo, div, m);
    if (d < 0.0 || (d == 0.0 && ((b - 1u) & 1u) == 0u)) return b - 1u;
  }
  return b;
}

// round-half-even of the exact quotient w/s for a binary16-valued s > 0 and |w/s| < 2^20.
// k = rint(w * (1/s)) is off by at most one near a half-integer; the two FMA residuals
// w - (k +- 1/2)s are exact in sign (the product is exact and the sum is rounded once),
// so they decide the true rounding, ties to even.
__device__ __forceinline__ float rne_quotient(float w, float s, float inv_s) {
  float k = rintf(w * inv_s);
  float rh = fmaf(-(k + 0.5f), s, w);
  float rl = fmaf(-(k - 0.5f), s, w);
  bool odd = (__float2int_rz(k) & 1) != 0;
  if (rh > 0.0f || (rh == 0.0f && odd)) {
    k += 1.0f;
  } else if (rl < 0.0f || (rl == 0.0f && odd)) {
    k -= 1.0f;
  }
  return k;
}

struct AsymScale {
  float s;        // S' as float
  float inv_s;    // 1/S' (only a hint for rne_quotient)
  float z;        // Z as float, integral in [0, 15]
  unsigned sbits; // S' binary16 bits
  bool bad;       // non-finite range or binary16 overflow
};

// S' = binary16 RNE((beta - alpha)/15) with S' = 0 -> 1; Z = clip(RNE(-alpha/S'), 0, 15).
// mn = min(0, min w) <= 0 <= mx = max(0, max w) (NaN if a weight was NaN).
__device__ __forceinline__ AsymScale asym_scale_zero(float mn, float mx) {
  AsymScale r;
  float a = mx, b = -mn;
  float hi = a + b;  // exact split of a + b into hi + lo (Fast2Sum, larger operand first)
  float lo = (a >= b) ? (b - (hi - a)) : (a - (hi - b));
  r.bad = !isfinite(hi);
  unsigned sb = r.bad ? 0x3C00u : rne_f16_of_quotient(hi, lo, 15.0f, 1.0f / 15.0f);
  if (sb >= 0x7C00u) {
    r.bad = true;
    sb = 0x3C00u;
  }
  if (sb == 0u) sb = 0x3C00u;  // range below half the smallest subnormal: S' = 1
  r.sbits = sb;
  r.s = f16_bits_to_f32(sb);
  r.inv_s = __frcp_rn(r.s);
  float z = r.bad ? 0.0f : rne_quotient(b, r.s, r.inv_s);
  r.z = fminf(fmaxf(z, 0.0f), 15.0f);
  return r;
}

// Symmetric scale s' = binary16 RNE(amax / qmax), 0 -> 1. Sets bad on overflow / NaN.
__device__ __forceinline__ AsymScale sym_scale(float amax, float qmax) {
  AsymScale r;
  r.bad = !isfinite(amax);
  unsigned sb = r.bad ? 0x3C00u : rne_f16_of_quotient(amax, 0.0f, qmax, 1.0f / qmax);
  if (sb >= 0x7C00u) {
    r.bad = true;
    sb = 0x3C00u;
  }
  if (sb == 0u) sb = 0x3C00u;
  r.sbits = sb;
  r.s = f16_bits_to_f32(sb);
  r.inv_s = __frcp_rn(r.s);
  r.z = 0.0f;
  return r;
}

// Symmetric INT4 per group in the asymmetric storage ("DL S067 - Quantization", section 2,
// quantize_per_group): s' = binary16 RNE(max|w| / 7) (0 -> 1) and Z = 8, so that the
// asymmetric encode clip(RNE(w/s') + 8, 0, 15) stores clip(RNE(w/s'), -8, 7) + 8 and every
// dequant s'(code - Z) is s'q. mn = min(0, min w), mx = max(0, max w) (NaN if a weight was).
__device__ __forceinline__ AsymScale sym4_scale_zero(float mn, float mx) {
  AsymScale r = sym_scale(fmax_nan(-mn, mx), 7.0f);
  r.z = 8.0f;
  return r;
}

// bf16 pair (one 32-bit word) -> two floats.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two floats -> bf16 pair, round-half-even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace wq
