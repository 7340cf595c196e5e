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
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "mma_frag.cuh"

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

// Small-M W4A16 matmul on the tensor cores' warp-level MMA (m16n8k16, bf16 x bf16 -> fp32),
// for decode: the CUDA-core form above needs ~2.3 instructions per weight (a byte-permute
// per code plus the FMAs); here a pair of codes becomes a bf16 pair (128 + q) with one LOP3,
// and one MMA consumes 256 weights per warp. M <= 8 tokens occupy the MMA's N = 8 columns.
//
// Layout of the work: a warp processes one 16-row tile of W against one group (128 k) per
// step: lane (r = lane/4, c = lane%4) loads bytes [16c, 16c + 16) of the group's 64 bytes for
// rows r and r + 8 (each load instruction reads 8 rows x 64 contiguous bytes). A 32-bit word
// holds 8 consecutive codes k0..k7; it unpacks to the pairs (k0,k4), (k1,k5), (k2,k6),
// (k3,k7). MMA j of the group (j = 0..7) takes pairs from word j/2 of the lane's 4 words; the
// X operand is permuted identically once per CTA into shared memory ("fragment order"), so
// the k order inside the MMA is irrelevant to the sum. One packed bf16 subtraction per pair
// turns (128 + q) into the exact small integer q - Z of its row, so each group's fp32 result
// is D = sum (q - Z) x with no large offset to cancel, and S' is applied once per group:
// acc += S' D.
// The CTA (8 warps) owns a 16-row tile, its warps split the groups, and the partial tiles
// are summed through shared memory in a fixed order.
// (128 + q) bf16 pairs of a word's codes: out[i] = (k_i, k_{i+4}) for i = 0..3.
__device__ __forceinline__ void unpack_bf16_pairs(uint32_t w, uint32_t (&out)[4]) {
  out[0] = (w & 0x000F000Fu) | 0x43004300u;
  out[1] = ((w >> 4) & 0x000F000Fu) | 0x43004300u;
  out[2] = ((w >> 8) & 0x000F000Fu) | 0x43004300u;
  out[3] = ((w >> 12) & 0x000F000Fu) | 0x43004300u;
}

template <int M>
__global__ void __launch_bounds__(256)
gemv_mma(const uint16_t* __restrict__ X, int64_t ldx, const uint8_t* __restrict__ P,
         const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K,
         int group, int sz_row, uint16_t* __restrict__ Y, int64_t ldy) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int G = K / 128;
  uint32_t* xf = reinterpret_cast<uint32_t*>(smem);                      // [G][4M][16]
  float* red = reinterpret_cast<float*>(smem + static_cast<size_t>(G) * 4 * M * 64);  // [8][16][8]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- X -> fragment order (once per CTA) and per-group token sums
  for (int e = threadIdx.x; e < G * 4 * M; e += blockDim.x) {
    const int g = e / (4 * M);
    const int L = e - g * 4 * M;  // fragment lane: token n = L/4, quarter c = L%4
    const int n = L >> 2, c = L & 3;
    const uint16_t* xs = X + n * ldx + g * 128 + 32 * c;
    uint32_t xw[16];  // x[32c + 2i], x[32c + 2i + 1] pairs
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = ld_nc_u4(xs + 8 * v);
      xw[4 * v] = u.x; xw[4 * v + 1] = u.y; xw[4 * v + 2] = u.z; xw[4 * v + 3] = u.w;
    }
    uint32_t frag[16];
    build_x_fragment(xw, frag);
    uint32_t* dst = xf + (static_cast<size_t>(g) * 4 * M + L) * 16;
#pragma unroll
    for (int j = 0; j < 16; ++j) dst[j] = frag[j];
  }
  __syncthreads();

  const int r = lane >> 2, c = lane & 3;
  const int t0 = 2 * c, t1 = 2 * c + 1;  // tokens (columns) of this lane's accumulators
  const int g_lo = (warp * G) / 8, g_hi = ((warp + 1) * G) / 8;
  const int ntiles = (N + 15) / 16;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int n0 = tile * 16 + r, n1 = n0 + 8;
    const bool v0 = n0 < N, v1 = n1 < N;
    const uint8_t* p0 = P + static_cast<int64_t>(n0) * (K / 2) + 16 * c;
    const uint8_t* p1 = P + static_cast<int64_t>(n1) * (K / 2) + 16 * c;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    uint4 wa = make_uint4(0, 0, 0, 0), wb = wa;
    if (g_lo < g_hi) {
      if (v0) wa = ld_stream_u4(p0 + g_lo * 64);
      if (v1) wb = ld_stream_u4(p1 + g_lo * 64);
    }
    for (int g = g_lo; g < g_hi; ++g) {
      const uint4 ca = wa, cb = wb;
      if (g + 1 < g_hi) {  // next group's codes in flight while this one computes
        if (v0) wa = ld_stream_u4(p0 + (g + 1) * 64);
        if (v1) wb = ld_stream_u4(p1 + (g + 1) * 64);
      }
      const int64_t gi0 = static_cast<int64_t>(n0) * sz_row + (sz_row ? (g * 128) / group : 0);
      const int64_t gi1 = static_cast<int64_t>(n1) * sz_row + (sz_row ? (g * 128) / group : 0);
      const float s0 = v0 ? f16_bits_to_f32(ld_nc_u16(S + gi0)) : 0.0f;
      const float z0 = v0 ? f16_bits_to_f32(ld_nc_u16(Zp + gi0)) : 0.0f;
      const float s1 = v1 ? f16_bits_to_f32(ld_nc_u16(S + gi1)) : 0.0f;
      const float z1 = v1 ? f16_bits_to_f32(ld_nc_u16(Zp + gi1)) : 0.0f;
      const __nv_bfloat162 zz0 = __floats2bfloat162_rn(128.0f + z0, 128.0f + z0);
      const __nv_bfloat162 zz1 = __floats2bfloat162_rn(128.0f + z1, 128.0f + z1);
      uint4 xb[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                     make_uint4(0, 0, 0, 0)};
      if (lane < 4 * M) {
        const uint4* src = reinterpret_cast<const uint4*>(xf + (static_cast<size_t>(g) * 4 * M + lane) * 16);
        xb[0] = src[0]; xb[1] = src[1]; xb[2] = src[2]; xb[3] = src[3];
      }
      const uint32_t bw[16] = {xb[0].x, xb[0].y, xb[0].z, xb[0].w, xb[1].x, xb[1].y, xb[1].z, xb[1].w,
                               xb[2].x, xb[2].y, xb[2].z, xb[2].w, xb[3].x, xb[3].y, xb[3].z, xb[3].w};
      const uint32_t wr0[4] = {ca.x, ca.y, ca.z, ca.w};
      const uint32_t wr1[4] = {cb.x, cb.y, cb.z, cb.w};
      float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t pa[4], pb[4];
        unpack_bf16_pairs(wr0[w], pa);
        unpack_bf16_pairs(wr1[w], pb);
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // (128 + q) - (128 + Z) = q - Z, exact in bf16
          __nv_bfloat162 ta = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&pa[i]), zz0);
          __nv_bfloat162 tb = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&pb[i]), zz1);
          pa[i] = *reinterpret_cast<uint32_t*>(&ta);
          pb[i] = *reinterpret_cast<uint32_t*>(&tb);
        }
        const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
        const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
        mma_bf16_16816(d, a0, bw[4 * w], bw[4 * w + 1]);
        mma_bf16_16816(d, a1, bw[4 * w + 2], bw[4 * w + 3]);
      }
      acc[0] = fmaf(s0, d[0], acc[0]);
      acc[1] = fmaf(s0, d[1], acc[1]);
      acc[2] = fmaf(s1, d[2], acc[2]);
      acc[3] = fmaf(s1, d[3], acc[3]);
    }
    // partial tile of this warp -> shared; sum over the 8 warps in a fixed order
    float* rw = red + warp * 128;
    rw[r * 8 + t0] = acc[0];
    rw[r * 8 + t1] = acc[1];
    rw[(r + 8) * 8 + t0] = acc[2];
    rw[(r + 8) * 8 + t1] = acc[3];
    __syncthreads();
    if (threadIdx.x < 16 * M) {
      const int row = threadIdx.x / M, tok = threadIdx.x - (threadIdx.x / M) * M;
      float t = 0.0f;
#pragma unroll
      for (int w = 0; w < 8; ++w) t += red[w * 128 + row * 8 + tok];
      const int n = tile * 16 + row;
      if (n < N) {
        __nv_bfloat16 hv = __float2bfloat16_rn(t);
        Y[tok * ldy + n] = *reinterpret_cast<uint16_t*>(&hv);
      }
    }
    __syncthreads();
  }
}

// Small-M W4A16 matmul: warp-level MMA consumers fed by bulk asynchronous copies.
// One producer lane streams 16-row tiles into a shared-memory ring: each row's K/2 packed
// bytes land at a row stride of 64 mod 128 bytes (so the MMA warps' 16-byte reads are
// bank-conflict free) and the tile's S' and Z (16 x G each, contiguous in HBM) follow.
// Sixteen MMA warps split the tile's groups. Codes are decoded with the bf16 magic
// 1 + q/16 (nibble in the top mantissa bits: one shift and one LOP3 per pair of codes), so
// one group's MMA result is D = sum x (1 + q/16) and, with sum x of the group,
//   sum x (q - Z) = 16 D - (16 + Z) sum x,      acc += S' (16 D - (16 + Z) sum x).
// The offset is small (16 against q - Z), so the fp32 cancellation costs only a few bits.
// The X fragments (see gemv_mma) and the per-group token sums are built once per CTA.
// Each group's 8 MMAs run as two independent accumulator chains.
// Shared-memory layout of gemv_mma_bulk (host and device agree through this).
struct MmaBulkLayout {
  uint32_t xf_bytes, sx_bytes, xq_bytes, stage_bytes, wbytes, szbytes, ring_off, bar_off, red_off,
      total;
  __host__ __device__ MmaBulkLayout(int M, int K, int wstride, int stages, int NW, int RT) {
    const uint32_t G = K / 128;
    xf_bytes = G * 4 * M * 64;
    sx_bytes = G * 8 * 4;
    xq_bytes = G * 4 * M * 4;  // per-quarter sums of x, [G][M][4]
    wbytes = 16u * RT * wstride;
    szbytes = 16u * RT * G * 2;
    stage_bytes = wbytes + 2 * szbytes;
    ring_off = (xf_bytes + sx_bytes + xq_bytes + 127) / 128 * 128;
    bar_off = ring_off + stages * stage_bytes;
    red_off = bar_off + (2 * stages + 2) * 8;
    total = red_off + 2u * NW * RT * 16 * (M < 2 ? 2 : M) * 4;
  }
};

// Small-M W4A16 matmul: warp-level MMA consumers fed by bulk asynchronous copies.
// One producer lane streams tiles of 16*RT rows into a shared-memory ring: each row's K/2
// packed bytes land at a row stride of 64 mod 128 bytes (so the MMA warps' 16-byte reads
// are bank-conflict free), followed by the tile's S' and Z (contiguous in HBM). NW MMA
// warps split the groups of K; per group a warp decodes and multiplies all RT 16-row
// sub-tiles, so the X fragments are read once per group and the RT accumulator chains are
// independent. Codes are decoded with the bf16 magic 1 + q/16 (nibble in the top mantissa
// bits: one shift and one 3-input LOP3 per pair of codes), so a group's MMA result is
// D = sum x (1 + q/16) and, with the group's sum of x,
//   sum x (q - Z) = 16 D - (16 + Z) sum x,      acc += S' (16 D - (16 + Z) sum x).
// The offset is small (16 against q - Z), so the fp32 cancellation costs only a few bits.
// Partial tiles are summed over the warps in shared memory behind a bounded mbarrier.
template <int M, int NW, int RT>
__global__ void __launch_bounds__(32 * (NW + 1), 1)
gemv_mma_bulk(const uint16_t* __restrict__ X, int64_t ldx, const uint8_t* __restrict__ P,
              const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K,
              int wstride, int stages, uint32_t prefetch_bytes, uint16_t* __restrict__ Y,
              int64_t ldy, unsigned* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int MR = M < 2 ? 2 : M;  // token slots kept in the reduction buffer
  constexpr int TR = 16 * RT;        // rows per tile
  const MmaBulkLayout L(M, K, wstride, stages, NW, RT);
  const int G = K / 128;
  uint32_t* xf = reinterpret_cast<uint32_t*>(smem);                  // [G][4M][16]
  float* sxs = reinterpret_cast<float*>(smem + L.xf_bytes);           // [G][8]
  uint8_t* ring = smem + L.ring_off;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + stages;
  uint64_t* redbar = empty + stages;  // [2]
  float* red = reinterpret_cast<float*>(smem + L.red_off);  // [2][NW][TR][MR]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = N / TR;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    mbar_init(&redbar[0], NW);
    mbar_init(&redbar[1], NW);
    fence_barrier_init();
  }
  __syncthreads();
  // Let the next kernel on the stream launch now; warm L2 with this CTA's weight tiles
  // (a hint, safe before the dependency wait), then wait for the previous kernel.
  if (threadIdx.x == 0) pdl_launch_dependents();
  const uint32_t tile_w = static_cast<uint32_t>(TR) * (K / 2);
  if (warp == NW && lane == 0) {
    uint32_t budget = prefetch_bytes;
    for (int tile = blockIdx.x; tile < ntiles && budget >= tile_w; tile += gridDim.x) {
      prefetch_l2_bulk(P + static_cast<int64_t>(tile) * tile_w, tile_w);
      budget -= tile_w;
    }
  }
  pdl_wait();

  if (warp == NW) {  // producer
    if (lane == 0) {
      int i = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
        const int st = i % stages;
        const uint32_t use = i / stages;
        if (use > 0 && !mbar_wait_bounded(&empty[st], (use - 1) & 1u, kWaitLimitNs)) {
          set_status(status, kStTimeout);
          break;
        }
        uint8_t* dst = ring + static_cast<size_t>(st) * L.stage_bytes;
        mbar_arrive_expect_tx(&full[st], tile_w + 2 * L.szbytes);
        const uint8_t* src = P + static_cast<int64_t>(tile) * tile_w;
        for (int r = 0; r < TR; ++r)
          bulk_g2s(dst + r * wstride, src + static_cast<int64_t>(r) * (K / 2), K / 2, &full[st]);
        bulk_g2s(dst + L.wbytes, S + static_cast<int64_t>(tile) * TR * G, L.szbytes, &full[st]);
        bulk_g2s(dst + L.wbytes + L.szbytes, Zp + static_cast<int64_t>(tile) * TR * G,
                 L.szbytes, &full[st]);
      }
      for (int st = 0; st < stages && st < i; ++st) {
        const uint32_t last = (i - 1 - st) / stages;
        if (!mbar_wait_bounded(&full[st], last & 1u, kWaitLimitNs)) set_status(status, kStTimeout);
      }
    }
    return;
  }

  // X -> fragment order and per-group token sums; overlaps with the producer's first copies.
  // A thread issues the loads of up to four of its entries (32 values of one token each) at
  // once, so the L2 latency is paid once per four entries, and sums each entry's values from
  // the same registers; the four quarter sums of a group are added in a fixed order below.
  {
    float* xq = reinterpret_cast<float*>(smem + L.xf_bytes + L.sx_bytes);  // [G][M][4]
    const int total = G * 4 * M;
    for (int e0 = threadIdx.x; e0 < total; e0 += 4 * 32 * NW) {
      uint4 u[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = e0 + j * 32 * NW;
        if (e < total) {
          const int g = e / (4 * M);
          const int Lf = e - g * 4 * M;
          const uint16_t* xs = X + (Lf >> 2) * ldx + g * 128 + 32 * (Lf & 3);
#pragma unroll
          for (int v = 0; v < 4; ++v) u[j][v] = ld_nc_u4(xs + 8 * v);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = e0 + j * 32 * NW;
        if (e < total) {
          const int g = e / (4 * M);
          const int Lf = e - g * 4 * M;
          uint32_t xw[16];
          float t = 0.0f;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            xw[4 * v] = u[j][v].x; xw[4 * v + 1] = u[j][v].y;
            xw[4 * v + 2] = u[j][v].z; xw[4 * v + 3] = u[j][v].w;
            t += ((bf16_lo(u[j][v].x) + bf16_hi(u[j][v].x)) + (bf16_lo(u[j][v].y) + bf16_hi(u[j][v].y))) +
                 ((bf16_lo(u[j][v].z) + bf16_hi(u[j][v].z)) + (bf16_lo(u[j][v].w) + bf16_hi(u[j][v].w)));
          }
          uint32_t frag[16];
          build_x_fragment(xw, frag);
          // chunks of quarter c rotated by 2 (c >> 1): a warp's four quarter loads hit four
          // bank groups
          uint32_t* dst = xf + (static_cast<size_t>(g) * 4 * M + Lf) * 16;
          const int xrot = 2 * ((Lf >> 1) & 1);
#pragma unroll
          for (int q = 0; q < 16; ++q) dst[(((q >> 2) + xrot) & 3) * 4 + (q & 3)] = frag[q];
          xq[e] = t;
        }
      }
    }
    named_barrier(1, 32 * NW);
    for (int e = threadIdx.x; e < G * 8; e += 32 * NW) {
      const int g = e >> 3, n = e & 7;
      const float* q = xq + (g * M + n) * 4;
      sxs[e] = n < M ? (q[0] + q[1]) + (q[2] + q[3]) : 0.0f;
    }
  }
  named_barrier(1, 32 * NW);

  const int r = lane >> 2, c = lane & 3;
  const int t0 = 2 * c, t1 = 2 * c + 1;
  const int g_lo = (warp * G) / NW, g_hi = ((warp + 1) * G) / NW;
  // lanes whose token column is >= M read a duplicate fragment: their columns are never
  // stored, and the loads stay uniform (no divergent branch)
  const uint32_t xf_lane = smem_u32(xf) + (lane % (4 * M)) * 64;
  // this lane's X fragment chunks 0, 1 sit at xlo, xlo + 16 and chunks 2, 3 at xhi, xhi + 16
  const uint32_t xlo = 32u * ((lane >> 1) & 1), xhi = 32u - xlo;
  const uint32_t ring_s = smem_u32(ring);
  const float* sx0p = sxs + t0;
  const float* sx1p = sxs + t1;
  uint32_t kMask = 0x00780078u, kMagic = 0x3F803F80u;  // register operands of the LOP3
  asm volatile("" : "+r"(kMask), "+r"(kMagic));
  int i = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
    const int st = i % stages;
    if (!mbar_wait_bounded(&full[st], (i / stages) & 1u, kWaitLimitNs)) {
      set_status(status, kStTimeout);
      return;
    }
    const uint32_t wb = ring_s + st * L.stage_bytes;
    const uint32_t sb = wb + L.wbytes, zb = sb + L.szbytes;
    float acc[RT][4];
#pragma unroll
    for (int t = 0; t < RT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
    for (int g = g_lo; g < g_hi; ++g) {
      const uint32_t xs = xf_lane + g * (4 * M * 64);
      const uint4 xb0 = lds128(xs + xlo), xb1 = lds128(xs + xlo + 16), xb2 = lds128(xs + xhi),
                  xb3 = lds128(xs + xhi + 16);
      const uint32_t bw[16] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w,
                               xb2.x, xb2.y, xb2.z, xb2.w, xb3.x, xb3.y, xb3.z, xb3.w};
      const float sx0 = sx0p[g * 8], sx1 = sx1p[g * 8];
#pragma unroll
      for (int t = 0; t < RT; ++t) {
        const int ra = 16 * t + r, rb = ra + 8;
        const uint4 ca = lds128(wb + ra * wstride + g * 64 + 16 * c);
        const uint4 cb = lds128(wb + rb * wstride + g * 64 + 16 * c);
        const uint32_t wr0[4] = {ca.x, ca.y, ca.z, ca.w};
        const uint32_t wr1[4] = {cb.x, cb.y, cb.z, cb.w};
        float de[4] = {0.0f, 0.0f, 0.0f, 0.0f}, dodd[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t pa[4], pb[4];
          unpack_bf16_hi(wr0[w], kMask, kMagic, pa);
          unpack_bf16_hi(wr1[w], kMask, kMagic, pb);
          const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
          const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
          mma_bf16_16816(de, a0, bw[4 * w], bw[4 * w + 1]);
          mma_bf16_16816(dodd, a1, bw[4 * w + 2], bw[4 * w + 3]);
        }
        const float s0 = f16_bits_to_f32(lds16(sb + (ra * G + g) * 2));
        const float z0 = f16_bits_to_f32(lds16(zb + (ra * G + g) * 2));
        const float s1 = f16_bits_to_f32(lds16(sb + (rb * G + g) * 2));
        const float z1 = f16_bits_to_f32(lds16(zb + (rb * G + g) * 2));
        acc[t][0] = fmaf(s0, fmaf(16.0f, de[0] + dodd[0], -(16.0f + z0) * sx0), acc[t][0]);
        acc[t][1] = fmaf(s0, fmaf(16.0f, de[1] + dodd[1], -(16.0f + z0) * sx1), acc[t][1]);
        acc[t][2] = fmaf(s1, fmaf(16.0f, de[2] + dodd[2], -(16.0f + z1) * sx0), acc[t][2]);
        acc[t][3] = fmaf(s1, fmaf(16.0f, de[3] + dodd[3], -(16.0f + z1) * sx1), acc[t][3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    const int par = i & 1;
    float* rw = red + (par * NW + warp) * TR * MR;
#pragma unroll
    for (int t = 0; t < RT; ++t) {
      const int ra = 16 * t + r, rb = ra + 8;
      if (t0 < M) {
        rw[ra * MR + t0] = acc[t][0];
        rw[rb * MR + t0] = acc[t][2];
      }
      if (t1 < M) {
        rw[ra * MR + t1] = acc[t][1];
        rw[rb * MR + t1] = acc[t][3];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&redbar[par]);
    if (!mbar_wait_bounded(&redbar[par], (i >> 1) & 1u, kWaitLimitNs)) {
      set_status(status, kStTimeout);
      return;
    }
    for (int e = threadIdx.x; e < TR * M; e += 32 * NW) {
      const int row = e / M, tok = e - (e / M) * M;
      const float* rp = red + par * NW * TR * MR + row * MR + tok;
      float t = 0.0f;
#pragma unroll
      for (int w = 0; w < NW; ++w) t += rp[w * TR * MR];
      __nv_bfloat16 hv = __float2bfloat16_rn(t);
      Y[tok * ldy + tile * TR + row] = *reinterpret_cast<uint16_t*>(&hv);
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
    set_smem_attrs(kern, 200 * 1024);
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

size_t mma_smem(int M, int K) {
  const size_t G = K / 128;
  return G * 4 * M * 64 + 8 * 128 * 4;
}

template <int M>
cudaError_t launch_mma(const GemvArgs& a, int sms, cudaStream_t st) {
  const size_t smem = mma_smem(M, a.K);
  static int occ_cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& occ = occ_cache[dev & 63];
  if (occ == 0) {
    set_smem_attrs(gemv_mma<M>, 96 * 1024);
    occ = -1;
  }
  int o = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, gemv_mma<M>, 256, smem) != cudaSuccess ||
      o < 1)
    o = 1;
  const int ntiles = (a.N + 15) / 16;
  int grid = sms * o;
  if (grid > ntiles) grid = ntiles;
  gemv_mma<M><<<grid, 256, smem, st>>>(a.X, a.ldx, a.P, a.S, a.Z, a.N, a.K, a.group, a.sz_row,
                                       a.Y, a.ldy);
  return cudaGetLastError();
}

template <int M, int NW, int RT>
cudaError_t launch_mma_bulk(const GemvArgs& a, int sms, cudaStream_t st) {
  const int half = a.K / 2;
  const int wstride = half + ((64 - half % 128) + 128) % 128;  // = 64 (mod 128)
  constexpr size_t kBudget = 220 * 1024;  // one CTA per SM
  int stages = 8;
  while (stages >= 2 && MmaBulkLayout(M, a.K, wstride, stages, NW, RT).total > kBudget) --stages;
  if (stages < 2) return cudaErrorInvalidValue;
  const size_t smem = MmaBulkLayout(M, a.K, wstride, stages, NW, RT).total;
  auto kern = gemv_mma_bulk<M, NW, RT>;
  static std::atomic<bool> attr[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 63].load(std::memory_order_acquire)) {
    set_smem_attrs(kern, static_cast<int>(kBudget));
    attr[dev & 63].store(true, std::memory_order_release);
  }
  const int ntiles = a.N / (16 * RT);
  const int grid = ntiles < sms ? ntiles : sms;
  // L2 warm-up per CTA: at most 48 MB for the whole grid
  const uint32_t prefetch = static_cast<uint32_t>((48ull << 20) / grid);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32 * (NW + 1));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a.X, a.ldx, a.P, a.S, a.Z, a.N, a.K, wstride, stages,
                            prefetch, a.Y, a.ldy, a.status);
}

// MMA warps per CTA of the bulk-fed decode kernel. Tiles are 32 rows when two stages of
// them fit in shared memory (more work per fragment load and per sync), else 16 rows.
constexpr int kDecodeWarps = 8;

template <int M>
cudaError_t launch_mma_bulk_any(const GemvArgs& a, int sms, cudaStream_t st) {
  if (a.N % 32 == 0) {
    const cudaError_t e = launch_mma_bulk<M, kDecodeWarps, 2>(a, sms, st);
    if (e != cudaErrorInvalidValue) return e;
  }
  return launch_mma_bulk<M, kDecodeWarps, 1>(a, sms, st);
}

bool mma_bulk_ok(const GemvArgs& a) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return a.K % 128 == 0 && a.sz_row > 0 && a.group == 128 && a.N % 16 == 0 &&
         (a.ldx % 8) == 0 && al16(a.X) && al16(a.P) && al16(a.S) && al16(a.Z);
}

bool mma_ok(const GemvArgs& a) {
  return a.K % 128 == 0 && (a.sz_row == 0 || a.group % 128 == 0) &&
         mma_smem(a.M, a.K) <= 96 * 1024 && (a.ldx % 8) == 0 &&
         (reinterpret_cast<uintptr_t>(a.X) & 15u) == 0;
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

// Token block b <= a.M (a.M itself if it fits, else the largest of 8, 4, 2, 1) for which a
// bulk-fed MMA decode kernel (gemv_mma_bulk, or for b <= 4 one of the streaming kernels)
// fits this shape; 0 if none.
int gemv_fast_block(const GemvArgs& a) {
  if (!mma_bulk_ok(a)) return 0;
  const int half = a.K / 2;
  const int wstride = half + ((64 - half % 128) + 128) % 128;
  auto bulk_fits = [&](int m) {
    return MmaBulkLayout(m, a.K, wstride, 2, kDecodeWarps, 1).total <= 220u * 1024;
  };
  for (int b : {a.M, 8, 4, 2, 1}) {  // the whole of M first, then blocks
    if (b > a.M || b > 8) continue;
    GemvArgs t = a;
    t.M = b;
    if (bulk_fits(b) || gemv_stream_fits(t) || gemv_tma_ok(t) || gemv_imma_bulk_ok(t)) return b;
  }
  return 0;
}

// Whether two stages of whole 32-row tiles fit the bulk-copy kernel's shared memory.
static bool mma_bulk_rt2_fits(const GemvArgs& a) {
  const int half = a.K / 2;
  const int wstride = half + ((64 - half % 128) + 128) % 128;
  return a.N % 32 == 0 && MmaBulkLayout(a.M, a.K, wstride, 2, kDecodeWarps, 2).total <= 220u * 1024;
}

cudaError_t launch_gemv_w4a16(const GemvArgs& a, int sms, cudaStream_t st) {
  // M <= 2, g = 128, short rows: the integer-MMA kernel on whole-row tiles (gemv_imma.cu)
  // where two stages of them fit in shared memory.
  if (a.M <= 2 && gemv_imma_bulk_ok(a)) {
    const cudaError_t e = launch_gemv_imma_bulk(a, sms, st);
    if (e != cudaErrorInvalidValue) return e;
  }
  // M <= 4 with long rows (two whole 32-row tiles do not fit the bulk-copy kernel's shared
  // memory): the TMA-fed kernel that streams 32-row tiles in K chunks (N % 32 == 0).
  // Otherwise M = 1: the bulk-copy kernel (whole rows; measured fastest for short rows);
  // M = 2..4: the streaming kernel on 16-row tiles.
  if (a.M <= 4 && !(mma_bulk_ok(a) && mma_bulk_rt2_fits(a)) && gemv_tma_ok(a)) {
    const cudaError_t e = launch_gemv_tma(a, sms, st);
    if (e != cudaErrorInvalidValue) return e;
  }
  if (a.M > 1 && gemv_stream_ok(a)) {
    const cudaError_t e = launch_gemv_stream(a, sms, st);
    if (e != cudaErrorInvalidValue) return e;
  }
  if (a.M == 1 && mma_bulk_ok(a)) {
    const cudaError_t e = launch_mma_bulk_any<1>(a, sms, st);
    if (e != cudaErrorInvalidValue) return e;
  }
  if (a.M == 1 && gemv_stream_ok(a)) {
    const cudaError_t e = launch_gemv_stream(a, sms, st);
    if (e != cudaErrorInvalidValue) return e;
  }
  if (mma_bulk_ok(a)) {
    cudaError_t e = cudaErrorInvalidValue;
    switch (a.M) {
      case 1: e = launch_mma_bulk_any<1>(a, sms, st); break;
      case 2: e = launch_mma_bulk_any<2>(a, sms, st); break;
      case 3: e = launch_mma_bulk_any<3>(a, sms, st); break;
      case 4: e = launch_mma_bulk_any<4>(a, sms, st); break;
      case 5: e = launch_mma_bulk_any<5>(a, sms, st); break;
      case 6: e = launch_mma_bulk_any<6>(a, sms, st); break;
      case 7: e = launch_mma_bulk_any<7>(a, sms, st); break;
      case 8: e = launch_mma_bulk_any<8>(a, sms, st); break;
      default: break;
    }
    if (e != cudaErrorInvalidValue) return e;
  }
  if (mma_ok(a)) {
    switch (a.M) {
      case 1: return launch_mma<1>(a, sms, st);
      case 2: return launch_mma<2>(a, sms, st);
      case 3: return launch_mma<3>(a, sms, st);
      case 4: return launch_mma<4>(a, sms, st);
      case 5: return launch_mma<5>(a, sms, st);
      case 6: return launch_mma<6>(a, sms, st);
      case 7: return launch_mma<7>(a, sms, st);
      case 8: return launch_mma<8>(a, sms, st);
      default: break;
    }
  }
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
