// W4A16 decode GEMV / small-M matmul on CUDA cores: Y[m, n] = sum_k X[m, k] S'(q - Z).
// ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
// "The vocabulary" and "Overview": decode reads every weight once, so it is bound by HBM.)
//
// gemv_slices<M, RB> (M = 1):
//   * The CTA has C = ceil(K/1024) warps; warp c owns the k-slice [1024c, 1024c + 1024)
//     for its whole life, lane l the 32 k starting at 1024c + 32l. Its slice of X (32M
//     floats) and the slice sums sum_k x (M floats) stay in registers.
//   * The CTA streams a block of RB output rows: per row, each lane issues one 16-byte
//     non-allocating load of packed nibbles plus S', Z (all RB rows' loads are issued
//     before any is used), so a warp keeps RB x 512 B in flight.
//   * Dequantization stays in registers and S' is factored out of each group:
//       sum_k x (S'(q - Z)) = S' (sum_k x q - Z sum_k x).
//     A nibble q becomes the float 0.5 + q/256 with one byte-permute (bits 0x3F00qq00),
//     so sum_k x q = 256 sum_k x f - 128 sum_k x; the products run as packed fp32x2 FMAs.
//     Accumulation is fp32 throughout (exact weights, fp32 rounding only).
//   * Per-lane partials go through shared memory once per CTA and are summed over the
//     C warps and 32 lanes in a fixed order (deterministic, no atomics).
//
// gemv_rows<M> (2 <= M <= 8): one warp per output row, X re-read through L1; a simple
//   path for small batches.
#include "common.cuh"
#include "kernels.h"

namespace wq {
namespace {

constexpr int kSlice = 1024;  // k per warp slice: 32 lanes x 32 weights (16 bytes)

// Four float2 = the floats (0.5 + q/256) of the 8 nibbles of `w`, ordered by k:
// out[j] = {f(k = 2j), f(k = 2j + 1)} for the byte j of w.
__device__ __forceinline__ void nibbles_to_f2(uint32_t w, float2 out[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu;
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t sel = 0x7044u | (static_cast<uint32_t>(j) << 8);
    out[j].x = __uint_as_float(__byte_perm(lo, 0x3F000000u, sel));
    out[j].y = __uint_as_float(__byte_perm(hi, 0x3F000000u, sel));
  }
}

template <int M, int RB>
__global__ void __launch_bounds__(1024)
gemv_slices(const uint16_t* __restrict__ X, int64_t ldx, const uint8_t* __restrict__ P,
            const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K,
            int group, int sz_row, uint16_t* __restrict__ Y, int64_t ldy) {
  extern __shared__ float red[];  // [C][RB*M][32]
  const int C = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int k0 = warp * kSlice + lane * 32;
  const bool kact = k0 < K;
  const int gi_k = sz_row ? k0 / group : 0;

  // x slice (fp32 pairs) and its sums, kept for the CTA's lifetime
  float2 x[M][16];
  float sx[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint4 u = kact ? ld_nc_u4(X + m * ldx + k0 + 8 * v) : make_uint4(0, 0, 0, 0);
      const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[m][4 * v + e] = make_float2(bf16_lo(ws[e]), bf16_hi(ws[e]));
        s2.x += x[m][4 * v + e].x;
        s2.y += x[m][4 * v + e].y;
      }
    }
    sx[m] = s2.x + s2.y;
  }

  float acc[RB][M];
  const int n0 = blockIdx.x * RB;
  uint4 p[RB];
  float s[RB], z[RB];
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    const int n = n0 + r;
    const bool ok = kact && n < N;
    p[r] = ok ? ld_stream_u4(P + static_cast<int64_t>(n) * (K / 2) + k0 / 2) : make_uint4(0, 0, 0, 0);
    const int64_t gi = static_cast<int64_t>(n) * sz_row + gi_k;
    s[r] = ok ? f16_bits_to_f32(ld_nc_u16(S + gi)) : 0.0f;
    z[r] = ok ? f16_bits_to_f32(ld_nc_u16(Zp + gi)) : 0.0f;
  }
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    float2 a[M];
#pragma unroll
    for (int m = 0; m < M; ++m) a[m] = make_float2(0.0f, 0.0f);
    const uint32_t ws[4] = {p[r].x, p[r].y, p[r].z, p[r].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f[4];
      nibbles_to_f2(ws[i], f);
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int m = 0; m < M; ++m) a[m] = __ffma2_rn(x[m][4 * i + j], f[j], a[m]);
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float t = fmaf(-(128.0f + z[r]), sx[m], 256.0f * (a[m].x + a[m].y));
      acc[r][m] = s[r] * t;
    }
  }

  // per-lane partials -> shared -> sum over (warps, lanes) in a fixed order
  constexpr int V = RB * M;
#pragma unroll
  for (int r = 0; r < RB; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m) red[(warp * V + r * M + m) * 32 + lane] = acc[r][m];
  __syncthreads();
  for (int v = warp; v < V; v += C) {
    float t = 0.0f;
    for (int c = 0; c < C; ++c) t += red[(c * V + v) * 32 + lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    const int r = v / M, m = v % M;
    const int n = n0 + r;
    if (lane == 0 && n < N) {
      __nv_bfloat16 h = __float2bfloat16_rn(t);
      Y[m * ldy + n] = *reinterpret_cast<uint16_t*>(&h);
    }
  }
}

template <int M>
__global__ void __launch_bounds__(256)
gemv_rows(const uint16_t* __restrict__ X, int64_t ldx, const uint8_t* __restrict__ P,
          const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K,
          int group, int sz_row, uint16_t* __restrict__ Y, int64_t ldy) {
  const int lane = threadIdx.x & 31;
  const int n = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (n >= N) return;
  float acc[M];
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = 0.0f;
  for (int k0 = lane * 32; k0 < K; k0 += kSlice) {
    const uint4 pk = ld_stream_u4(P + static_cast<int64_t>(n) * (K / 2) + k0 / 2);
    const int64_t gi = static_cast<int64_t>(n) * sz_row + (sz_row ? k0 / group : 0);
    const float s = f16_bits_to_f32(ld_nc_u16(S + gi));
    const float z = f16_bits_to_f32(ld_nc_u16(Zp + gi));
    const uint32_t ws[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float2 a = make_float2(0.0f, 0.0f), sxx = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 u = ld_nc_u4(X + m * ldx + k0 + 8 * i);
        const uint32_t xs[4] = {u.x, u.y, u.z, u.w};
        float2 f[4];
        nibbles_to_f2(ws[i], f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 xv = make_float2(bf16_lo(xs[j]), bf16_hi(xs[j]));
          a = __ffma2_rn(xv, f[j], a);
          sxx.x += xv.x;
          sxx.y += xv.y;
        }
      }
      const float t = fmaf(-(128.0f + z), sxx.x + sxx.y, 256.0f * (a.x + a.y));
      acc[m] = fmaf(s, t, acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float t = acc[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) {
      __nv_bfloat16 h = __float2bfloat16_rn(t);
      Y[m * ldy + n] = *reinterpret_cast<uint16_t*>(&h);
    }
  }
}

// W8A16, symmetric INT8 per output row: Y[m, n] = s'_n sum_k X[m, k] q[n, k]. One warp per
// row, 16 codes per lane per step; a code byte b becomes q via the float 2^23 + (b ^ 0x80)
// minus 2^23 + 128 (exact).
template <int M>
__global__ void __launch_bounds__(256)
gemv8_rows(const uint16_t* __restrict__ X, int64_t ldx, const int8_t* __restrict__ Q,
           const uint16_t* __restrict__ S, int N, int K, uint16_t* __restrict__ Y,
           int64_t ldy) {
  const int lane = threadIdx.x & 31;
  const int n = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (n >= N) return;
  float acc[M];
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = 0.0f;
  for (int k0 = lane * 16; k0 < K; k0 += 512) {
    const uint4 pk = ld_stream_u4(Q + static_cast<int64_t>(n) * K + k0);
    const uint32_t ws[4] = {pk.x ^ 0x80808080u, pk.y ^ 0x80808080u, pk.z ^ 0x80808080u,
                            pk.w ^ 0x80808080u};
    float q[16];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        q[4 * i + j] = __uint_as_float(__byte_perm(ws[i], 0x4B000000u, 0x7440u | j)) - 8388736.0f;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint4 u0 = ld_nc_u4(X + m * ldx + k0);
      const uint4 u1 = ld_nc_u4(X + m * ldx + k0 + 8);
      const uint32_t xs[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        a = __ffma2_rn(make_float2(bf16_lo(xs[e]), bf16_hi(xs[e])),
                       make_float2(q[2 * e], q[2 * e + 1]), a);
      acc[m] += a.x + a.y;
    }
  }
  const float s = f16_bits_to_f32(ld_nc_u16(S + n));
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float t = acc[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) {
      __nv_bfloat16 h = __float2bfloat16_rn(s * t);
      Y[m * ldy + n] = *reinterpret_cast<uint16_t*>(&h);
    }
  }
}

template <int M>
cudaError_t launch_rows8(const Gemv8Args& a, cudaStream_t st) {
  gemv8_rows<M><<<(a.N + 7) / 8, 256, 0, st>>>(a.X, a.ldx, a.Q, a.S, a.N, a.K, a.Y, a.ldy);
  return cudaGetLastError();
}

template <int M>
cudaError_t launch_rows(const GemvArgs& a, cudaStream_t st) {
  const int grid = (a.N + 7) / 8;
  gemv_rows<M><<<grid, 256, 0, st>>>(a.X, a.ldx, a.P, a.S, a.Z, a.N, a.K, a.group, a.sz_row,
                                     a.Y, a.ldy);
  return cudaGetLastError();
}

template <int M, int RB>
cudaError_t launch_slices(const GemvArgs& a, cudaStream_t st) {
  const int C = (a.K + kSlice - 1) / kSlice;
  const int threads = 32 * C;
  const size_t smem = static_cast<size_t>(C) * RB * M * 32 * sizeof(float);
  const int grid = (a.N + RB - 1) / RB;
  gemv_slices<M, RB><<<grid, threads, smem, st>>>(a.X, a.ldx, a.P, a.S, a.Z, a.N, a.K, a.group,
                                                  a.sz_row, a.Y, a.ldy);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv_w8a16(const Gemv8Args& a, cudaStream_t st) {
  switch (a.M) {
    case 1: return launch_rows8<1>(a, st);
    case 2: return launch_rows8<2>(a, st);
    case 3: return launch_rows8<3>(a, st);
    case 4: return launch_rows8<4>(a, st);
    case 5: return launch_rows8<5>(a, st);
    case 6: return launch_rows8<6>(a, st);
    case 7: return launch_rows8<7>(a, st);
    case 8: return launch_rows8<8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

int gemv_max_k() { return 32 * kSlice; }

cudaError_t launch_gemv_w4a16(const GemvArgs& a, cudaStream_t st) {
  switch (a.M) {
    case 1: return launch_slices<1, 8>(a, st);
    case 2: return launch_rows<2>(a, st);
    case 3: return launch_rows<3>(a, st);
    case 4: return launch_rows<4>(a, st);
    case 5: return launch_rows<5>(a, st);
    case 6: return launch_rows<6>(a, st);
    case 7: return launch_rows<7>(a, st);
    case 8: return launch_rows<8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wq
