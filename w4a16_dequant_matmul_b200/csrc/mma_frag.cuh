// Warp-level MMA pieces shared by the small-M W4A16 kernels: the m16n8k16 bf16 MMA, the
// decode of packed 4-bit codes into bf16 operands, and the X (B operand) fragments.
//
// k order. A lane of the A fragment holds, per 32-bit register, two weights of one row at
// "consecutive" k. Codes are read 32 at a time (16 bytes of a packed row: lane c of a quad
// reads codes 32c .. 32c + 31 of the group), and the k order inside each MMA is permuted so
// that a register pairs codes j and j + 4 of one packed word: MMA k slots (2c, 2c+1,
// 2c+8, 2c+9) of word w hold codes 8w + {0, 4, 1, 5} (first MMA of the word) or
// 8w + {2, 6, 3, 7} (second). build_x_fragment applies the same permutation to X, so the
// dot products are unchanged.
#pragma once

#include <stdint.h>

namespace wq {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// (a & b) | c in one 3-input logic op (both constants arrive in registers, so no second op).
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// (1 + q/16) bf16 pairs of a word's codes: out[i] = (code i, code i + 4) for i = 0..3. The
// code lands in the top four mantissa bits of a bf16 1.0. mask = 0x00780078,
// magic = 0x3F803F80 (passed in registers by the caller).
__device__ __forceinline__ void unpack_bf16_hi(uint32_t w, uint32_t mask, uint32_t magic,
                                               uint32_t (&out)[4]) {
  out[0] = and_or(w << 3, mask, magic);
  out[1] = and_or(w >> 1, mask, magic);
  out[2] = and_or(w >> 5, mask, magic);
  out[3] = and_or(w >> 9, mask, magic);
}

// B fragments of 32 consecutive bf16 values of X (xw[16] = the 32 values as 16 words, in
// order) for the four MMA pairs of a quad lane: out[4w + 0..1] feed the first MMA of
// packed word w, out[4w + 2..3] the second.
__device__ __forceinline__ void build_x_fragment(const uint32_t (&xw)[16], uint32_t (&out)[16]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int w = j >> 1, o = j & 1;
    const uint32_t lo = xw[4 * w + o];
    const uint32_t hi = xw[4 * w + 2 + o];
    out[2 * j] = __byte_perm(lo, hi, 0x5410);
    out[2 * j + 1] = __byte_perm(lo, hi, 0x7632);
  }
}

}  // namespace wq
