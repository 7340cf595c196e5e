// Round-to-nearest quantizer kernels ("DL S067 - Quantization", sections 1-2;
// "Model Quantization", section 1).
//
//  * quant_asym_lanegroup<T, g>: g in {32, 64, 128, 256}, one lane per group; a warp
//    stages its 32 groups in shared memory with coalesced loads, then each lane takes the
//    range, S'/Z and the codes of its own group (fast FMA path for bf16, exact fallback).
//  * quant_asym_wide<T>: g > 256 (e.g. g = K, one scale per output channel): one warp per
//    group, two passes over the group (range, then codes; the second pass hits L2).
//  * quant_sym_int8_row<T>: symmetric INT8 with one scale per output row.
//  * per-tensor: a grid-wide min/max into the caller's workspace, then codes.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

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

// NaN-propagating packed bf16 min / max (two weights per instruction).
__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Codes of 8 bf16 weights (4 pairs) without a per-weight exact test.
//
// Why it is exact: write w = M_w 2^a and S' = M_s 2^b with M_w, M_s odd integers, M_w < 2^8
// (bf16) and M_s < 2^11 (binary16). Then w/S' - (k + 1/2) has denominator 2 M_s (when
// a >= b - 1) and is either 0 or at least 1/4094 in magnitude; when a < b - 1 and w/S' is
// near a half-integer at all, the same gap is at least 1/510. So the exact quotient is
// either a half-integer or at least 2^-12 away from every half-integer. The product with
// the fp32 reciprocal inv_s = RN(1/S') is within |w/S'| 2^-24 < 2^-19 of the quotient (the
// caller guarantees |w/S'| < 32). One FMA, RN(w inv_s + 1536), snaps it to the 2^-13 grid
// (the spacing of floats in [1024, 2048)): a half-integer quotient lands on itself exactly,
// any other stays strictly on its own side of the nearest half-integer. Adding
// 1.5 2^23 - 1536 + Ze then rounds the snapped value to an integer with ties to even
// (spacing 1 in [2^23, 2^24)); Ze = Z rounded up to even keeps the parity of k, so ties go
// to even k as RNE(w/S') requires. The low byte of the sum is k + Ze = code + (Z & 1); the
// caller's `zfix` = (Z & 1) * 0x11111111 removes that bias from the packed word (mod 2^32,
// where every byte sum fits). kClamp clips the codes to [0, 15] in the float domain.
template <bool kClamp>
__device__ __forceinline__ uint32_t encode8_snap(const uint32_t w[4], float inv_s, float cz,
                                                 float tlo, float thi, uint32_t zfix) {
  const float2 inv2 = make_float2(inv_s, inv_s);
  const float2 g2 = make_float2(1536.0f, 1536.0f), c2 = make_float2(cz, cz);
  uint32_t tb[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 v = make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
    const float2 snapped = __ffma2_rn(v, inv2, g2);
    float2 t = __fadd2_rn(snapped, c2);
    if constexpr (kClamp) {
      t.x = fminf(fmaxf(t.x, tlo), thi);
      t.y = fminf(fmaxf(t.y, tlo), thi);
    }
    tb[2 * j] = __float_as_uint(t.x);
    tb[2 * j + 1] = __float_as_uint(t.y);
  }
  const uint32_t ev = __byte_perm(__byte_perm(tb[0], tb[2], 0x0040), __byte_perm(tb[4], tb[6], 0x0040), 0x5410);
  const uint32_t od = __byte_perm(__byte_perm(tb[1], tb[3], 0x0040), __byte_perm(tb[5], tb[7], 0x0040), 0x5410);
  return ev + (od << 4) - zfix;
}

// Codes of one group of GS weights held at shared-memory address row_s, written to dst
// (16-byte aligned): the bf16 snap path above.
template <int GS, bool kClamp>
__device__ __forceinline__ void encode_group_snap(uint32_t row_s, uint8_t* dst, const AsymScale& sz) {
  const int z1 = static_cast<int>(sz.z) & 1;
  const float cz = 12581376.0f + (sz.z + static_cast<float>(z1));  // 1.5 2^23 - 1536 + Ze
  const float tlo = 12582912.0f + static_cast<float>(z1);
  const float thi = tlo + 15.0f;
  const uint32_t zfix = static_cast<uint32_t>(z1) * 0x11111111u;
#pragma unroll 2
  for (int k = 0; k < GS; k += 32) {  // 32 weights -> 16 bytes of codes
    uint32_t words[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 u = lds128(row_s + (k + 8 * j) * 2);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
      words[j] = encode8_snap<kClamp>(wv, sz.inv_s, cz, tlo, thi, zfix);
    }
    *reinterpret_cast<uint4*>(dst + k / 2) = make_uint4(words[0], words[1], words[2], words[3]);
  }
}

// Codes of one group by the exact per-weight decision (fp32 input, or a group whose range
// is not finite); kept out of line so that the common path stays small in the
// instruction cache.
template <typename T, int GS>
__device__ __noinline__ void encode_group_exact(uint32_t row_s, uint8_t* dst, AsymScale sz) {
  for (int k = 0; k < GS; k += 8) {
    float v[8];
    if constexpr (sizeof(T) == 2) {
      const uint4 u = lds128(row_s + k * 2);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = bf16_lo(wv[e]);
        v[2 * e + 1] = bf16_hi(wv[e]);
      }
    } else {
      const uint4 a0 = lds128(row_s + k * 4), a1 = lds128(row_s + k * 4 + 16);
      v[0] = __uint_as_float(a0.x); v[1] = __uint_as_float(a0.y);
      v[2] = __uint_as_float(a0.z); v[3] = __uint_as_float(a0.w);
      v[4] = __uint_as_float(a1.x); v[5] = __uint_as_float(a1.y);
      v[6] = __uint_as_float(a1.z); v[7] = __uint_as_float(a1.w);
    }
    *reinterpret_cast<uint32_t*>(dst + k / 2) = encode8(v, sz);
  }
}

// 16-byte streaming load that stays where it is written (volatile): used to issue the next
// step's loads before the current step's arithmetic, so that the two overlap.
__device__ __forceinline__ uint4 ld_stream_u4_early(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <typename T, int GS>
struct LaneGroupCfg {
  static constexpr int kRowBytes = GS * static_cast<int>(sizeof(T));  // bytes per group
  static constexpr int kChunks = kRowBytes / 16;                       // 16-byte chunks per group
  // groups per warp step: 32 (one per lane) while a step is at most 16 chunks per lane
  static constexpr int kStepGroups = kChunks <= 16 ? 32 : 512 / kChunks;
  static constexpr int kPre = kStepGroups * kChunks / 32;  // chunks each lane prefetches
  static constexpr int kStride = kRowBytes + 16;           // padded shared-memory row
  static constexpr int kWarps = 4;
};

// Groups of g <= 256 weights, one lane per group. A warp takes kStepGroups consecutive
// groups per step. Each step's weights are first loaded cooperatively (every load
// instruction of the warp reads 512 contiguous bytes) into registers, one step ahead, and
// then written to the warp's shared-memory buffer, whose rows are padded by 16 bytes so
// that lane l's reads of group l do not conflict. Every lane then reduces its group
// (pass 1), computes S' and Z once, and encodes it (pass 2), both passes reading shared
// memory while the next step's loads are in flight. For bf16 input the range uses packed
// bf16 min/max and the codes the fast path above; a group whose end codes fall outside
// [0, 15] (possible only through the binary16 rounding of S or a double tie) or a near-tie
// takes the exact path.
template <typename T, int GS>
__global__ void __launch_bounds__(128, 4)
quant_asym_lanegroup(const T* __restrict__ W, int64_t ldw, int N, int K,
                     uint8_t* __restrict__ packed, uint16_t* __restrict__ S,
                     uint16_t* __restrict__ Z, bool sym, unsigned* status) {
  using Cfg = LaneGroupCfg<T, GS>;
  constexpr bool kBf16 = sizeof(T) == 2;
  constexpr int kChunks = Cfg::kChunks;
  constexpr int kStepGroups = Cfg::kStepGroups;
  constexpr int kPre = Cfg::kPre;
  constexpr int kStride = Cfg::kStride;
  __shared__ __align__(16) uint8_t buf[Cfg::kWarps][kStepGroups * kStride];
  const int G = K / GS;
  const int64_t total = static_cast<int64_t>(N) * G;
  const int lane = threadIdx.x & 31;
  const uint32_t mybuf_s = smem_u32(buf[threadIdx.x >> 5]);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * Cfg::kWarps + (threadIdx.x >> 5);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * Cfg::kWarps * kStepGroups;
  // The group of lane l in a step is base + (l mod kStepGroups); its row n and index g are
  // advanced incrementally (no 64-bit division inside the loop).
  const int myg = lane % kStepGroups;
  int64_t t = warp * kStepGroups + myg;
  int64_t n = t / G;
  int g = static_cast<int>(t - n * G);
  const int64_t stride_n = stride / G;
  const int stride_g = static_cast<int>(stride - stride_n * G);
  auto advance = [&]() {
    t += stride;
    n += stride_n;
    g += stride_g;
    if (g >= G) {
      g -= G;
      ++n;
    }
  };
  // Chunk i of this lane: group (lane + 32 i) / kChunks of the step, 16-byte chunk
  // (lane + 32 i) mod kChunks of that group. Rows stored back to back (ldw == K) make a
  // full step one contiguous range, read at constant offsets from one address; otherwise
  // (and for the last, partial step) each chunk takes its group's address from the lane
  // that owns the group, and chunks past the end read W's first bytes instead (loaded,
  // never used), so that no loaded value goes through a select.
  const bool contiguous = ldw == K;
  uint4 pre[kPre];
  auto prefetch = [&](int64_t base) {
    if (contiguous && base + kStepGroups <= total) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>(W) + base * Cfg::kRowBytes + 16 * lane;
#pragma unroll
      for (int i = 0; i < kPre; ++i) pre[i] = ld_stream_u4_early(src + 512 * i);
    } else {
      const uint8_t* mine =
          reinterpret_cast<const uint8_t*>(W + n * ldw + static_cast<int64_t>(g) * GS);
#pragma unroll
      for (int i = 0; i < kPre; ++i) {
        const int ci = lane + 32 * i;
        const int gl = ci / kChunks, ch = ci % kChunks;
        const uint8_t* src = reinterpret_cast<const uint8_t*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(mine), gl));
        src = base + gl < total ? src + 16 * ch : reinterpret_cast<const uint8_t*>(W);
        pre[i] = ld_stream_u4_early(src);
      }
    }
  };
  int64_t base = warp * kStepGroups;
  if (base < total) prefetch(base);
  for (; base < total; base += stride) {
    __syncwarp();
#pragma unroll
    for (int i = 0; i < kPre; ++i) {
      const int ci = lane + 32 * i;
      sts128(mybuf_s + (ci / kChunks) * kStride + 16 * (ci % kChunks), pre[i]);
    }
    __syncwarp();
    const int64_t tc = t, nc = n;
    const int gc = g;
    advance();
    if (base + stride < total) prefetch(base + stride);
    const bool active = lane < kStepGroups && tc < total;
    const uint32_t row_s = mybuf_s + myg * kStride;
    float mn = 0.0f, mx = 0.0f;
    if constexpr (kBf16) {
      uint32_t lo2 = 0u, hi2 = 0u;  // bf16x2 (0, 0): the range includes zero
#pragma unroll 4
      for (int ch = 0; ch < kChunks; ++ch) {
        const uint4 u = lds128(row_s + 16 * ch);
        lo2 = bmin2(bmin2(lo2, u.x), bmin2(u.y, bmin2(u.z, u.w)));
        hi2 = bmax2(bmax2(hi2, u.x), bmax2(u.y, bmax2(u.z, u.w)));
      }
      mn = fmin_nan(bf16_lo(lo2), bf16_hi(lo2));
      mx = fmax_nan(bf16_lo(hi2), bf16_hi(hi2));
    } else {
#pragma unroll 4
      for (int ch = 0; ch < kChunks; ++ch) {
        const uint4 u = lds128(row_s + 16 * ch);
        const float v[4] = {__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z),
                            __uint_as_float(u.w)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          mn = fmin_nan(mn, v[e]);
          mx = fmax_nan(mx, v[e]);
        }
      }
    }
    const AsymScale sz = sym ? sym4_scale_zero(mn, mx) : asym_scale_zero(mn, mx);
    // The snap path needs bf16 weights and a finite range (then |w/S'| < 32). Codes of the
    // range ends decide whether any code needs the clip; the whole warp then takes the
    // clipping variant, so that the warp does not split.
    const bool exact = !kBf16 || sz.bad;
    bool clip = false;
    if (active && !exact) {
      const float c_lo = rne_quotient(mn, sz.s, sz.inv_s) + sz.z;
      const float c_hi = rne_quotient(mx, sz.s, sz.inv_s) + sz.z;
      clip = c_lo < 0.0f || c_hi > 15.0f;
    }
    const bool any_clip = __any_sync(0xffffffffu, clip);
    if (active) {
      uint8_t* dst = packed + nc * (K / 2) + static_cast<int64_t>(gc) * (GS / 2);
      if constexpr (kBf16) {
        if (exact) {
          encode_group_exact<T, GS>(row_s, dst, sz);
        } else if (any_clip) {
          encode_group_snap<GS, true>(row_s, dst, sz);
        } else {
          encode_group_snap<GS, false>(row_s, dst, sz);
        }
      } else {
        encode_group_exact<T, GS>(row_s, dst, sz);
      }
      S[tc] = static_cast<uint16_t>(sz.sbits);
      Z[tc] = static_cast<uint16_t>(f32_to_f16_bits(sz.z));
      if (sz.bad) set_status(status, kStNonFinite);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
quant_asym_wide(const T* __restrict__ W, int64_t ldw, int N, int K, int group,
                uint8_t* __restrict__ packed, uint16_t* __restrict__ S,
                uint16_t* __restrict__ Z, bool sym, unsigned* status) {
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
    const AsymScale sz = sym ? sym4_scale_zero(mn, mx) : asym_scale_zero(mn, mx);
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

// One block per kWarps * kStepGroups groups, at most one resident wave of blocks (the
// blocks loop over the rest), so that no block starts after the others have finished.
template <typename T, int GS>
void launch_lanegroup(const T* W, int64_t ldw, int N, int K, uint8_t* packed, uint16_t* S,
                      uint16_t* Z, bool sym, unsigned* status, int64_t groups, int sms,
                      cudaStream_t st) {
  using Cfg = LaneGroupCfg<T, GS>;
  static int per_sm = 0;  // resident blocks per SM (the same on every sm_100 device)
  if (per_sm == 0) {
    int v = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, quant_asym_lanegroup<T, GS>,
                                                      32 * Cfg::kWarps, 0) != cudaSuccess || v < 1)
      v = 1;
    per_sm = v;
  }
  constexpr int kPerBlock = Cfg::kWarps * Cfg::kStepGroups;
  int64_t blocks = (groups + kPerBlock - 1) / kPerBlock;
  const int64_t cap = static_cast<int64_t>(sms) * per_sm;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quant_asym_lanegroup<T, GS><<<static_cast<int>(blocks), 32 * Cfg::kWarps, 0, st>>>(
      W, ldw, N, K, packed, S, Z, sym, status);
}

template <typename T>
cudaError_t launch_quant_asym_t(const T* W, int64_t ldw, int N, int K, int group,
                                uint8_t* packed, uint16_t* S, uint16_t* Z, bool sym,
                                unsigned* status, int sms, cudaStream_t st) {
  const int64_t groups = static_cast<int64_t>(N) * (K / group);
  switch (group) {
    case 32: launch_lanegroup<T, 32>(W, ldw, N, K, packed, S, Z, sym, status, groups, sms, st); break;
    case 64: launch_lanegroup<T, 64>(W, ldw, N, K, packed, S, Z, sym, status, groups, sms, st); break;
    case 128: launch_lanegroup<T, 128>(W, ldw, N, K, packed, S, Z, sym, status, groups, sms, st); break;
    case 256: launch_lanegroup<T, 256>(W, ldw, N, K, packed, S, Z, sym, status, groups, sms, st); break;
    default:
      quant_asym_wide<T><<<grid_for(groups, 8, sms), 256, 0, st>>>(W, ldw, N, K, group, packed,
                                                                   S, Z, sym, status);
      break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_asym(const void* W, bool bf16, int64_t ldw, int N, int K, int group,
                              uint8_t* packed, uint16_t* S, uint16_t* Z, bool sym,
                              unsigned* status, int sms, cudaStream_t st) {
  if (bf16)
    return launch_quant_asym_t(static_cast<const uint16_t*>(W), ldw, N, K, group, packed, S, Z,
                               sym, status, sms, st);
  return launch_quant_asym_t(static_cast<const float*>(W), ldw, N, K, group, packed, S, Z, sym,
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
