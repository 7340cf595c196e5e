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
#include "ptx.cuh"

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

// Butterfly reduce-scatter of RB per-lane values (RB a power of two <= 32) over the 32
// lanes of a warp: afterwards lane l holds the warp-wide sum of value l / (32 / RB).
template <int RB>
__device__ __forceinline__ float warp_reduce_scatter(float v[RB], int lane) {
#pragma unroll
  for (int half = RB / 2, o = 16; half >= 1; half >>= 1, o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float keep = upper ? v[j + half] : v[j];
      const float send = upper ? v[j] : v[j + half];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float t = v[0];
#pragma unroll
  for (int o = 16 / RB; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

// M = 1 decode GEMV. Persistent CTAs of C warps; warp c owns the k-range
// [c*1024*SEGS, (c+1)*1024*SEGS): lane l handles segments s = 0..SEGS-1 of 32 weights at
// k = c*1024*SEGS + 1024 s + 32 l (each warp load instruction reads 512 contiguous bytes).
// Its x values and their sums stay in registers for the kernel's lifetime. The CTA walks
// row blocks of RB (blk = blockIdx.x, + gridDim.x, ...); each lane keeps the packed codes
// and S', Z of the next D rows in flight while it computes the current row.
template <int SEGS, int D, int RB>
__global__ void __launch_bounds__(512)
gemv_m1(const uint16_t* __restrict__ X, const uint8_t* __restrict__ P,
        const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K,
        int group, int sz_row, uint16_t* __restrict__ Y) {
  constexpr int NB = D + 1;  // ring of row buffers; RB % NB == 0
  static_assert(RB % NB == 0, "ring size must divide the row block");
  __shared__ float red[2][32][RB];
  const int C = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int kseg[SEGS];
  bool kact[SEGS];
  int gik[SEGS];
  float2 x[SEGS][16];
  float sx[SEGS];
#pragma unroll
  for (int s = 0; s < SEGS; ++s) {
    kseg[s] = warp * 1024 * SEGS + 1024 * s + 32 * lane;
    kact[s] = kseg[s] < K;
    gik[s] = sz_row ? kseg[s] / group : 0;
    float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = kact[s] ? ld_nc_u4(X + kseg[s] + 8 * v) : make_uint4(0, 0, 0, 0);
      const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[s][4 * v + e] = make_float2(bf16_lo(ws[e]), bf16_hi(ws[e]));
        s2.x += x[s][4 * v + e].x;
        s2.y += x[s][4 * v + e].y;
      }
    }
    sx[s] = s2.x + s2.y;
  }

  const int nblk = (N + RB - 1) / RB;
  const int64_t prow = K / 2;
  uint4 pb[NB][SEGS];
  float sb[NB][SEGS], zb[NB][SEGS];

  auto fetch = [&](int buf, int n) {
#pragma unroll
    for (int s = 0; s < SEGS; ++s) {
      const bool ok = kact[s] && n < N;
      pb[buf][s] = ok ? ld_stream_u4(P + n * prow + kseg[s] / 2) : make_uint4(0, 0, 0, 0);
      const int64_t gi = static_cast<int64_t>(n) * sz_row + gik[s];
      sb[buf][s] = ok ? f16_bits_to_f32(ld_nc_u16(S + gi)) : 0.0f;
      zb[buf][s] = ok ? f16_bits_to_f32(ld_nc_u16(Zp + gi)) : 0.0f;
    }
  };

  int blk = blockIdx.x;
#pragma unroll
  for (int j = 0; j < D; ++j) fetch(j, blk * RB + j);
  int parity = 0;
  while (blk < nblk) {
    const int nxt = blk + gridDim.x;
    float acc[RB];
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      {  // keep D rows in flight: row i + D of this block, or the start of the next one
        const int j = i + D;
        const int n = j < RB ? blk * RB + j : nxt * RB + (j - RB);
        if (j < RB || nxt < nblk) fetch(j % NB, n);
      }
      const int b = i % NB;
      float a = 0.0f;
#pragma unroll
      for (int s = 0; s < SEGS; ++s) {
        float2 a2 = make_float2(0.0f, 0.0f);
        const uint32_t ws[4] = {pb[b][s].x, pb[b][s].y, pb[b][s].z, pb[b][s].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          float2 f[4];
          nibbles_to_f2(ws[w], f);
#pragma unroll
          for (int q = 0; q < 4; ++q) a2 = __ffma2_rn(x[s][4 * w + q], f[q], a2);
        }
        const float t = fmaf(-(128.0f + zb[b][s]), sx[s], 256.0f * (a2.x + a2.y));
        a = fmaf(sb[b][s], t, a);
      }
      acc[i] = a;
    }
    const float tot = warp_reduce_scatter<RB>(acc, lane);
    if ((lane & (32 / RB - 1)) == 0) red[parity][warp][lane / (32 / RB)] = tot;
    __syncthreads();
    if (threadIdx.x < RB) {
      float t = 0.0f;
      for (int c = 0; c < C; ++c) t += red[parity][c][threadIdx.x];
      const int n = blk * RB + threadIdx.x;
      if (n < N) {
        __nv_bfloat16 h = __float2bfloat16_rn(t);
        Y[n] = *reinterpret_cast<uint16_t*>(&h);
      }
    }
    parity ^= 1;
    blk = nxt;
  }
}

// M = 1 decode GEMV fed by bulk asynchronous copies. A row block of RB = 8 rows is three
// contiguous byte ranges (packed rows, their S', their Z); one producer lane streams row
// blocks into a ring of shared-memory stages with cp.async.bulk, completing on an
// mbarrier per stage, so the bytes in flight are bounded by shared memory, not registers.
// Consumer warps are bound to k-slices as in gemv_m1 (x and its sums in registers); WR
// warps share a slice and split the block's rows. The per-block sums over slices go
// through shared memory behind an mbarrier. Every wait is bounded: on a timeout the
// kernel records kStTimeout, the producer waits (bounded) for its copies to land, and all
// warps return.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

template <int WR>
__global__ void __launch_bounds__(1024)
gemv_m1_bulk(const uint16_t* __restrict__ X, const uint8_t* __restrict__ P,
             const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K,
             int group, int G, int stages, uint16_t* __restrict__ Y, unsigned* status) {
  constexpr int RB = 8;
  constexpr int RW = RB / WR;  // rows per consumer warp
  extern __shared__ __align__(128) uint8_t smem[];
  const int C = (K + 1023) / 1024;
  const int ncons = C * WR;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t pbytes = RB * (K / 2);
  const uint32_t sbytes = RB * G * 2;
  const uint32_t stage_bytes = pbytes + 2 * sbytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(stages) * stage_bytes);
  uint64_t* empty = full + stages;
  uint64_t* redbar = empty + stages;  // [2]
  float* red = reinterpret_cast<float*>(redbar + 2);  // [2][C][RB]
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], ncons);
    }
    mbar_init(&redbar[0], ncons);
    mbar_init(&redbar[1], ncons);
    fence_barrier_init();
  }
  __syncthreads();
  const int nblk = N / RB;

  if (warp == ncons) {  // producer warp: one lane issues the copies
    if (lane == 0) {
      int i = 0;
      for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x, ++i) {
        const int st = i % stages;
        const uint32_t use = i / stages;
        if (use > 0 && !mbar_wait_bounded(&empty[st], (use - 1) & 1u, kWaitLimitNs)) {
          set_status(status, kStTimeout);
          break;
        }
        uint8_t* dst = smem + static_cast<size_t>(st) * stage_bytes;
        mbar_arrive_expect_tx(&full[st], stage_bytes);
        bulk_g2s(dst, P + static_cast<int64_t>(blk) * pbytes, pbytes, &full[st]);
        bulk_g2s(dst + pbytes, S + static_cast<int64_t>(blk) * RB * G, sbytes, &full[st]);
        bulk_g2s(dst + pbytes + sbytes, Zp + static_cast<int64_t>(blk) * RB * G, sbytes,
                 &full[st]);
      }
      // never leave the CTA with copies in flight: wait for the last fill of each stage
      for (int st = 0; st < stages && st < i; ++st) {
        const uint32_t last = (i - 1 - st) / stages;
        if (!mbar_wait_bounded(&full[st], last & 1u, kWaitLimitNs)) set_status(status, kStTimeout);
      }
    }
    return;
  }

  const int slice = warp / WR;
  const int wr = warp % WR;
  const int k0 = slice * 1024 + lane * 32;
  const bool kact = k0 < K;
  const int gik = kact ? k0 / group : 0;
  float2 x[16];
  float sx;
  {
    float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = kact ? ld_nc_u4(X + k0 + 8 * v) : make_uint4(0, 0, 0, 0);
      const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[4 * v + e] = make_float2(bf16_lo(ws[e]), bf16_hi(ws[e]));
        s2.x += x[4 * v + e].x;
        s2.y += x[4 * v + e].y;
      }
    }
    sx = s2.x + s2.y;
  }

  int i = 0;
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x, ++i) {
    const int st = i % stages;
    if (!mbar_wait_bounded(&full[st], (i / stages) & 1u, kWaitLimitNs)) {
      set_status(status, kStTimeout);
      return;
    }
    const uint32_t base = smem_u32(smem) + st * stage_bytes;
    const uint32_t sS = base + pbytes;
    const uint32_t sZ = sS + sbytes;
    float acc[RW];
#pragma unroll
    for (int rr = 0; rr < RW; ++rr) {
      const int r = wr + rr * WR;
      const uint4 pk = kact ? lds128(base + r * (K / 2) + k0 / 2) : make_uint4(0, 0, 0, 0);
      const float sv = f16_bits_to_f32(lds16(sS + (r * G + gik) * 2));
      const float zv = f16_bits_to_f32(lds16(sZ + (r * G + gik) * 2));
      float2 a2 = make_float2(0.0f, 0.0f);
      const uint32_t ws[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        float2 f[4];
        nibbles_to_f2(ws[w], f);
#pragma unroll
        for (int q = 0; q < 4; ++q) a2 = __ffma2_rn(x[4 * w + q], f[q], a2);
      }
      acc[rr] = kact ? sv * fmaf(-(128.0f + zv), sx, 256.0f * (a2.x + a2.y)) : 0.0f;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done reading the stage
    const float tot = warp_reduce_scatter<RW>(acc, lane);
    const int par = i & 1;
    float* rd = red + par * C * RB;
    if ((lane & (32 / RW - 1)) == 0) rd[slice * RB + wr + (lane / (32 / RW)) * WR] = tot;
    __syncwarp();
    if (lane == 0) mbar_arrive(&redbar[par]);
    if (!mbar_wait_bounded(&redbar[par], (i >> 1) & 1u, kWaitLimitNs)) {
      set_status(status, kStTimeout);
      return;
    }
    if (warp == 0 && lane < RB) {
      float t = 0.0f;
      for (int c = 0; c < C; ++c) t += rd[c * RB + lane];
      __nv_bfloat16 h = __float2bfloat16_rn(t);
      Y[blk * RB + lane] = *reinterpret_cast<uint16_t*>(&h);
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

template <int SEGS, int D, int RB>
cudaError_t launch_m1(const GemvArgs& a, int sms, cudaStream_t st) {
  const int C = (a.K + 1024 * SEGS - 1) / (1024 * SEGS);
  const int threads = 32 * C;
  static int occ[33] = {0};  // resident CTAs per SM, by warp count (kernel config fixed)
  if (occ[C] == 0) {
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, gemv_m1<SEGS, D, RB>, threads, 0) !=
            cudaSuccess || o < 1)
      o = 1;
    occ[C] = o;
  }
  const int nblk = (a.N + RB - 1) / RB;
  int grid = sms * occ[C];
  if (grid > nblk) grid = nblk;
  gemv_m1<SEGS, D, RB><<<grid, threads, 0, st>>>(a.X, a.P, a.S, a.Z, a.N, a.K, a.group, a.sz_row,
                                             a.Y);
  return cudaGetLastError();
}

template <int WR>
cudaError_t launch_m1_bulk(const GemvArgs& a, int sms, cudaStream_t st) {
  const int C = (a.K + 1023) / 1024;
  const int threads = 32 * (C * WR + 1);
  const int G = a.sz_row;
  const size_t stage = static_cast<size_t>(8) * (a.K / 2) + 2 * 8 * G * 2;
  const size_t fixed = 16 * 8 + 2 * 8 + static_cast<size_t>(2) * C * 8 * 4 + 128;
  auto kern = gemv_m1_bulk<WR>;
  // Pipeline depth and CTAs per SM for this (K, G), computed once per device.
  struct Cfg { int key = -1, stages = 0, occ = 0; };
  static Cfg cache[64][8];
  int dev = 0;
  cudaGetDevice(&dev);
  Cfg& c = cache[dev & 63][(a.K / 32 + G) & 7];
  const int key = a.K * 4096 + G;
  if (c.key != key) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    int stages = static_cast<int>((100 * 1024 - fixed) / stage);
    if (stages > 8) stages = 8;
    int occ = 0;
    if (stages >= 2)
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, fixed + stages * stage);
    if (occ <= 1) {  // one CTA per SM: give it the shared memory of two
      stages = static_cast<int>((200 * 1024 - fixed) / stage);
      if (stages > 8) stages = 8;
      occ = 1;
    }
    c.key = key;
    c.stages = stages;
    c.occ = occ;
  }
  if (c.stages < 2) return cudaErrorInvalidValue;
  const size_t smem = fixed + c.stages * stage;
  const int nblk = a.N / 8;
  int grid = sms * c.occ;
  if (grid > nblk) grid = nblk;
  kern<<<grid, threads, smem, st>>>(a.X, a.P, a.S, a.Z, a.N, a.K, a.group, G, c.stages, a.Y,
                                    a.status);
  return cudaGetLastError();
}

bool bulk_ok(const GemvArgs& a) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return a.M == 1 && a.N % 8 == 0 && a.sz_row > 0 && a.K <= 16 * 1024 && al16(a.P) &&
         al16(a.S) && al16(a.Z) && al16(a.X);
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

cudaError_t launch_gemv_w4a16(const GemvArgs& a, int sms, cudaStream_t st) {
  switch (a.M) {
    case 1:
      if (bulk_ok(a)) {
        const int C = (a.K + 1023) / 1024;
        const cudaError_t e = C <= 15 ? launch_m1_bulk<2>(a, sms, st) : launch_m1_bulk<1>(a, sms, st);
        if (e != cudaErrorInvalidValue) return e;
      }
      return a.K <= 16 * kSlice ? launch_m1<1, 3, 8>(a, sms, st) : launch_m1<2, 1, 8>(a, sms, st);
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
