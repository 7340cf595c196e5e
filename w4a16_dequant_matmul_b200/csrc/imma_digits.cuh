// Integer warp-level MMA pieces of the small-M W4A16 kernels (gemv_imma.cu, gemv_tma.cu).
// ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
// "The vocabulary": 4-bit weights, 16-bit activations, the product accumulated in fp32.)
//
// For one group of 128 k and one output row,
//     sum_k x_k S'(q_k - Z) = S' (sum_k q_k x_k - Z sum_k x_k).
// The integer codes q are already what an integer MMA multiplies; the bf16 activations are
// written as integers too: per token and group, x_k 2^s is rounded to an integer x_int,k with
// |x_int| < 2^22 (s from the group's largest exponent). That is exact for every x_k within
// 2^14 of the group's largest magnitude (a bf16 value has 8 significant bits) and otherwise
// off by at most 2^-23 of that magnitude, below the rounding of an fp32 sum. x_int splits into
// three signed bytes, x_int = d0 + 2^8 d1 + 2^16 d2: the B operand of mma.sync m16n8k32
// (u8 codes x s8 digits -> s32), one column per (token, digit). Per group and row the MMA
// gives the exact integers D_i = sum_k q_k d_i,k; with the column sums X_i = sum_k d_i,k,
// (q - Z) enters exactly:
//     sum_k x_k (q_k - Z) = 2^-s sum_i 2^(8i) (D_i - Z X_i),
// the only roundings being the fp32 combination of the digits, the scaling and the
// accumulation over groups; no large offset is subtracted afterwards.
//
// k order. A lane (g, c) of an m16n8k32 fragment holds row g (and g + 8), MMA k slots
// 4c .. 4c + 3 (register a0 / a1) and 16 + 4c .. 16 + 4c + 3 (a2 / a3). It reads 16 bytes of
// a group's 64 packed bytes: bytes 16c .. 16c + 15, i.e. codes 32c .. 32c + 31, as four words;
// MMA w of the group takes word w, whose even codes (w & 0x0F0F0F0F) fill slots 4c .. 4c + 3
// and whose odd codes ((w >> 4) & 0x0F0F0F0F) fill 16 + 4c .. 16 + 4c + 3. prep_group lays
// the digits out in the same order, so each MMA multiplies matching k.
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"

namespace wq {

// 1.5 * 2^23: adding it to |v| < 2^22 rounds v to an integer held in the low mantissa bits.
constexpr float kImmaMagic = 12582912.0f;
constexpr int kImmaMagicBits = 0x4B400000;

// Digit columns per n-block of 8: token m uses columns 4m .. 4m + 2 (column 4m + 3 is zero),
// so a lane's two accumulator columns (2c, 2c + 1) always belong to one token.
template <int M> struct Cols {
  static constexpr int NB = (4 * M + 7) / 8;   // n-blocks of 8 columns
  static constexpr int FC = M == 1 ? 3 : 8;    // stored columns per n-block
  static constexpr uint32_t kFragBytes = NB * FC * 128;  // per group: [nb][h][col][c][16 B]
  static constexpr int MT = M == 1 ? 1 : 2 * NB;          // token slots with stored columns
};


__device__ __forceinline__ void imma_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                           uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// x * p2 + 1.5 * 2^23 in fp32 with a bf16 x and bf16 p2 (exact product, one rounding).
__device__ __forceinline__ float fma_bf16(uint32_t x_bits16, uint32_t p2_bits16, float c) {
  float d;
  asm("{\n\t.reg .b16 a, b;\n\tcvt.u16.u32 a, %1;\n\tcvt.u16.u32 b, %2;\n\t"
      "fma.rn.f32.bf16 %0, a, b, %3;\n\t}"
      : "=f"(d)
      : "r"(x_bits16), "r"(p2_bits16), "f"(c));
  return d;
}

// Signed byte digits (d0, d1, d2, 0) of round(x 2^s) for one bf16 x, given the group's
// scale 2^s as a bf16 (s <= 127) or, for groups below 2^-106, split into two fp32 factors.
__device__ __forceinline__ uint32_t digits_of(uint32_t xb, uint32_t p2b, bool split, float f1,
                                             float f2) {
  float t;
  if (!split) {
    t = fma_bf16(xb, p2b, kImmaMagic);
  } else {
    t = fmaf(__uint_as_float(xb << 16) * f1, f2, kImmaMagic);
  }
  // t = 1.5 * 2^23 + x_int exactly; + 0x808080 then ^ 0x808080 gives balanced signed bytes
  return (static_cast<uint32_t>(__float_as_int(t) - kImmaMagicBits) + 0x808080u) ^ 0x808080u;
}

// 2^e as a float for e in [-149, 127] (exact; subnormal below -126).
__device__ __forceinline__ float pow2i(int e) {
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23)
                   : __uint_as_float(1u << (e + 149));
}

// One group's X (xv: lane l holds k = 4l .. 4l + 3 of each token) -> its digit fragments,
// column sums and scales in shared memory. Called by one warp; only that warp reads them.
template <int M>
__device__ __forceinline__ void prep_group(uint8_t* fr, float* xs, float* xp,
                                           const uint2 (&xv)[M], int lane) {
  using C = Cols<M>;
  constexpr int FC = C::FC;
  const int c = lane >> 3, w = (lane >> 1) & 3, half = lane & 1;
#pragma unroll
  for (int m = 0; m < C::MT; ++m) {
    uint32_t z[4] = {0u, 0u, 0u, 0u};
    float p = 0.0f;
    if (m < M) {
      const uint2 xu = xv[m < M ? m : 0];
      const uint32_t xb[4] = {xu.x & 0xFFFFu, xu.x >> 16, xu.y & 0xFFFFu, xu.y >> 16};
      uint32_t e = 0;
#pragma unroll
      for (int v = 0; v < 4; ++v) e = max(e, (xb[v] >> 7) & 0xFFu);
      e = __reduce_max_sync(0xffffffffu, e);
      if (e == 0xFFu) {  // inf or NaN in the group: its products are not finite
        p = __uint_as_float(0x7FC00000u);
      } else {
        // s = 21 - (exponent of the largest |x|), so |x 2^s| < 2^22
        const int ex = static_cast<int>(e < 1u ? 1u : e) - 127;
        const int sc = 21 - ex;
        const bool split = sc > 127;
        const uint32_t p2b = split ? 0u : static_cast<uint32_t>(sc + 127) << 7;  // bf16 2^s
        const float f1 = split ? pow2i(100) : 0.0f;
        const float f2 = split ? pow2i(sc - 100) : 0.0f;
#pragma unroll
        for (int v = 0; v < 4; ++v) z[v] = digits_of(xb[v], p2b, split, f1, f2);
        p = pow2i(-sc);
      }
    }
    // lane (c, w, half) holds k = 32c + 8w + 4 half + {0..3}: its bytes go to the b0 / b1
    // halves (k even / k odd) of MMA w, column (token m, digit i), quad lane c
    const int nb = m >> 1, colbase = 4 * (m & 1);
    uint8_t* blk = fr + nb * FC * 128;
    uint32_t h0[3], h1[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      h0[i] = __byte_perm(z[0], z[2], static_cast<uint32_t>(i | ((4 + i) << 4)));
      h1[i] = __byte_perm(z[1], z[3], static_cast<uint32_t>(i | ((4 + i) << 4)));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int col = colbase + i;
      if (col < FC) {  // digit 3 is always zero: stored only where the layout has the column
        uint8_t* slot = blk + (w >> 1) * (FC * 64) + (col * 4 + c) * 16 + (w & 1) * 8 + 2 * half;
        sts16(smem_u32(slot), static_cast<uint16_t>(i < 3 ? h0[i < 3 ? i : 0] : 0u));
        sts16(smem_u32(slot + 4), static_cast<uint16_t>(i < 3 ? h1[i < 3 ? i : 0] : 0u));
      }
    }
    // column sums of the digits: (digit 0 + 2^16 digit 1) in one reduction, digit 2 in another
    const int s0 = __dp4a(static_cast<int>(h0[0]), 0x0101, __dp4a(static_cast<int>(h1[0]), 0x0101, 0));
    const int s1 = __dp4a(static_cast<int>(h0[1]), 0x0101, __dp4a(static_cast<int>(h1[1]), 0x0101, 0));
    const int s2 = __dp4a(static_cast<int>(h0[2]), 0x0101, __dp4a(static_cast<int>(h1[2]), 0x0101, 0));
    const int v01 = __reduce_add_sync(0xffffffffu, s0 + 65536 * s1);
    const int v2 = __reduce_add_sync(0xffffffffu, s2);
    if (lane == 0) {
      const int x0 = static_cast<int>(static_cast<int16_t>(v01 & 0xFFFF));  // |sum| < 2^15
      xs[nb * 8 + colbase] = static_cast<float>(x0);
      xs[nb * 8 + colbase + 1] = static_cast<float>((v01 - x0) >> 16);
      xs[nb * 8 + colbase + 2] = static_cast<float>(v2);
      xs[nb * 8 + colbase + 3] = 0.0f;
      if (m < M) xp[m] = p;
    }
  }
  if (M == 1 && lane < 4) xs[4 + lane] = 0.0f;  // columns 4..7 are unused with one token
}


}  // namespace wq
