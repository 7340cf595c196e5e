// W4A16 decode, M <= 2 tokens, short rows: integer warp-level MMA (imma_digits.cuh) on tiles
// of whole rows. Y = X W_hat^T with g = 128.
// ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
// "The vocabulary" and "Overview": 4-bit weights dequantized inside the kernel; decode reads
// every weight once, so it is bound by the bytes of weights read from HBM.)
//
// gemv_imma_bulk<M, RT>: a tile is 16 RT rows; one producer lane copies each of its rows (K/2
// bytes, one bulk copy per row) into a ring of tile stages at a row stride of 64 mod 128
// bytes (so a quarter-warp's 16-byte reads of two rows fall on different banks), followed by
// the tile's S' and Z ([16 RT][G] each, contiguous in HBM). X is copied first, so that it
// lands ahead of the weights. Eight MMA warps split the groups of K, each a contiguous range;
// a warp prepares the digit fragments of its own range once, then for every tile and group
// multiplies all RT 16-row sub-tiles against one load of the fragments. The warps' partial
// rows are summed in shared memory in a fixed order (deterministic). Rows short enough that
// two stages of whole-row tiles fit in shared memory (K up to about 6K) take this kernel:
// whole-row copies of a few KB start streaming sooner than K-chunked tensor boxes.
// Programmatic dependent launch: the kernel lets the next one launch at once and warms L2 with
// its own tiles before it waits for the previous kernel (a hint, safe before the wait: L2 is
// coherent with later writes); it reads X and the weights only after that wait. Every
// mbarrier wait is bounded (2 s): on a timeout the kernel records kStTimeout, the producer
// waits (bounded) for the copies it issued, and the warps return.
#include <atomic>

#include "common.cuh"
#include "imma_digits.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace wq {
namespace {

constexpr uint64_t kWaitNs = 2000000000ull;

__host__ __device__ constexpr uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

constexpr int kBulkWarps = 8;

struct BulkLayout {
  uint32_t xraw, frag, xs, xp, stage, wbytes, szbytes, ring, bar, red, total;
  __host__ __device__ BulkLayout(int M, int K, int wstride, int stages, int RT) {
    const uint32_t G = K / 128, MR = M < 2 ? 2 : M;
    const uint32_t NB = (4 * M + 7) / 8, FC = M == 1 ? 3 : 8;
    xraw = 0;                                     // [M][K] bf16
    frag = xraw + M * G * 256u;                   // [G][NB * FC * 128]
    xs = align_up(frag + G * NB * FC * 128, 16);  // [G][NB * 8] f32
    xp = xs + G * NB * 32u;                       // [G][M] f32
    wbytes = 16u * RT * wstride;
    szbytes = align_up(16u * RT * G * 2, 16);
    stage = wbytes + 2 * szbytes;
    ring = align_up(xp + G * M * 4u, 128);
    bar = ring + stages * stage;
    red = bar + (2 * stages + 3) * 8;
    total = red + 2u * kBulkWarps * RT * 16 * MR * 4;
  }
};

template <int M, int RT>
__global__ void __launch_bounds__(32 * (kBulkWarps + 1), 1)
gemv_imma_bulk(const uint16_t* __restrict__ X, int64_t ldx, const uint8_t* __restrict__ P,
               const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K,
               int wstride, int stages, uint32_t prefetch_bytes, uint16_t* __restrict__ Y,
               int64_t ldy, unsigned* status) {
  using C = Cols<M>;
  constexpr int NB = C::NB, FC = C::FC, NW = kBulkWarps;
  constexpr int MR = M < 2 ? 2 : M;
  constexpr int TR = 16 * RT;  // rows per tile
  extern __shared__ __align__(128) uint8_t smem[];
  const BulkLayout L(M, K, wstride, stages, RT);
  const int G = K / 128;
  const uint32_t base_s = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + stages;
  uint64_t* redbar = empty + stages;  // [2]
  uint64_t* xfull = redbar + 2;
  float* red = reinterpret_cast<float*>(smem + L.red);  // [2][NW][TR][MR]
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
    mbar_init(xfull, 1);
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

  if (warp == NW) {  // ------------------------------------------------------- producer
    if (lane == 0) {
      mbar_arrive_expect_tx(xfull, static_cast<uint32_t>(M) * K * 2);
      for (int m = 0; m < M; ++m)
        bulk_g2s(smem + L.xraw + static_cast<uint32_t>(m) * K * 2, X + m * ldx, K * 2u, xfull);
      int i = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
        const int st = i % stages;
        const uint32_t use = i / stages;
        if (use > 0 && !mbar_wait_spin_bounded(&empty[st], (use - 1) & 1u, kWaitNs)) {
          set_status(status, kStTimeout);
          break;
        }
        uint8_t* dst = smem + L.ring + static_cast<size_t>(st) * L.stage;
        const uint32_t szb = static_cast<uint32_t>(TR) * G * 2;
        mbar_arrive_expect_tx(&full[st], tile_w + 2 * szb);
        const uint8_t* src = P + static_cast<int64_t>(tile) * tile_w;
        for (int r = 0; r < TR; ++r)
          bulk_g2s(dst + r * wstride, src + static_cast<int64_t>(r) * (K / 2), K / 2, &full[st]);
        bulk_g2s(dst + L.wbytes, S + static_cast<int64_t>(tile) * TR * G, szb, &full[st]);
        bulk_g2s(dst + L.wbytes + L.szbytes, Zp + static_cast<int64_t>(tile) * TR * G, szb,
                 &full[st]);
      }
      for (int st = 0; st < stages && st < i; ++st) {
        const uint32_t last = (i - 1 - st) / stages;
        if (!mbar_wait_spin_bounded(&full[st], last & 1u, kWaitNs)) set_status(status, kStTimeout);
      }
      if (!mbar_wait_spin_bounded(xfull, 0, kWaitNs)) set_status(status, kStTimeout);
    }
    return;
  }

  // ----------------------------------------------------------------------- MMA warps
  const int g_lo = (warp * G) / NW, g_hi = ((warp + 1) * G) / NW;
  if (!mbar_wait_spin_bounded(xfull, 0, kWaitNs)) {
    set_status(status, kStTimeout);
    return;
  }
  for (int gi = g_lo; gi < g_hi; ++gi) {  // digit fragments of this warp's own groups
    uint2 xv[M];
#pragma unroll
    for (int m = 0; m < M; ++m)
      xv[m] = *reinterpret_cast<const uint2*>(smem + L.xraw + (m * G + gi) * 256 + 8 * lane);
    prep_group<M>(smem + L.frag + gi * C::kFragBytes,
                  reinterpret_cast<float*>(smem + L.xs) + gi * NB * 8,
                  reinterpret_cast<float*>(smem + L.xp) + gi * M, xv, lane);
  }
  __syncwarp();
  const float* xs_all = reinterpret_cast<const float*>(smem + L.xs);
  const float* xp_all = reinterpret_cast<const float*>(smem + L.xp);
  const int g = lane >> 2, c = lane & 3;
  const float w0 = (c & 1) ? 65536.0f : 1.0f, w1 = (c & 1) ? 16777216.0f : 256.0f;
  const bool bcol = g < FC;
  const uint32_t ring_s = base_s + L.ring;
  uint32_t mask4 = 0x0F0F0F0Fu;
  asm volatile("" : "+r"(mask4));
  int i = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
    const int st = i % stages;
    if (!mbar_wait_spin_bounded(&full[st], (i / stages) & 1u, kWaitNs)) {
      set_status(status, kStTimeout);
      return;
    }
    const uint32_t wb = ring_s + st * L.stage;
    const uint32_t sb = wb + L.wbytes, zb = sb + L.szbytes;
    float acc[RT][NB][2];
#pragma unroll
    for (int t = 0; t < RT; ++t)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) acc[t][nb][0] = acc[t][nb][1] = 0.0f;
    for (int gi = g_lo; gi < g_hi; ++gi) {
      const uint32_t frag_s = base_s + L.frag + gi * C::kFragBytes;
      uint32_t bw[NB][8];
      float2 xsum[NB];
      float p[NB];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const uint32_t blk = frag_s + nb * FC * 128 + (g * 4 + c) * 16;
        uint4 b01 = make_uint4(0u, 0u, 0u, 0u), b23 = b01;
        if (bcol) {
          b01 = lds128(blk);
          b23 = lds128(blk + FC * 64);
        }
        bw[nb][0] = b01.x; bw[nb][1] = b01.y; bw[nb][2] = b01.z; bw[nb][3] = b01.w;
        bw[nb][4] = b23.x; bw[nb][5] = b23.y; bw[nb][6] = b23.z; bw[nb][7] = b23.w;
        xsum[nb] = *reinterpret_cast<const float2*>(xs_all + gi * NB * 8 + nb * 8 + 2 * c);
        const int m = 2 * nb + (c >> 1);
        p[nb] = m < M ? xp_all[gi * M + (m < M ? m : 0)] : 0.0f;
      }
#pragma unroll
      for (int t = 0; t < RT; ++t) {
        const int ra = 16 * t + g, rb = ra + 8;
        const uint4 ca = lds128(wb + ra * wstride + gi * 64 + 16 * c);
        const uint4 cb = lds128(wb + rb * wstride + gi * 64 + 16 * c);
        const float sa = f16_bits_to_f32(lds16(sb + (ra * G + gi) * 2));
        const float sbv = f16_bits_to_f32(lds16(sb + (rb * G + gi) * 2));
        const float za = f16_bits_to_f32(lds16(zb + (ra * G + gi) * 2));
        const float zbv = f16_bits_to_f32(lds16(zb + (rb * G + gi) * 2));
        const uint32_t wa[4] = {ca.x, ca.y, ca.z, ca.w};
        const uint32_t wbw[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          int d[4] = {kImmaMagicBits, kImmaMagicBits, kImmaMagicBits, kImmaMagicBits};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t a[4] = {wa[q] & mask4, wbw[q] & mask4, (wa[q] >> 4) & mask4,
                                   (wbw[q] >> 4) & mask4};
            imma_16832(d, a, bw[nb][2 * q], bw[nb][2 * q + 1]);
          }
          const float e0 = __int_as_float(d[0]) - fmaf(za, xsum[nb].x, kImmaMagic);
          const float e1 = __int_as_float(d[1]) - fmaf(za, xsum[nb].y, kImmaMagic);
          const float e2 = __int_as_float(d[2]) - fmaf(zbv, xsum[nb].x, kImmaMagic);
          const float e3 = __int_as_float(d[3]) - fmaf(zbv, xsum[nb].y, kImmaMagic);
          float va = fmaf(e1, w1, e0 * w0), vb = fmaf(e3, w1, e2 * w0);
          va += __shfl_xor_sync(0xffffffffu, va, 1);
          vb += __shfl_xor_sync(0xffffffffu, vb, 1);
          acc[t][nb][0] = fmaf(sa * p[nb], va, acc[t][nb][0]);
          acc[t][nb][1] = fmaf(sbv * p[nb], vb, acc[t][nb][1]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    const int par = i & 1;
    float* rw = red + (par * NW + warp) * TR * MR;
    if ((c & 1) == 0) {
#pragma unroll
      for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const int m = 2 * nb + (c >> 1);
          if (m < M) {
            rw[(16 * t + g) * MR + m] = acc[t][nb][0];
            rw[(16 * t + g + 8) * MR + m] = acc[t][nb][1];
          }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&redbar[par]);
    if (!mbar_wait_spin_bounded(&redbar[par], (i >> 1) & 1u, kWaitNs)) {
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

template <int M, int RT>
cudaError_t launch_imma_bulk(const GemvArgs& a, int sms, cudaStream_t st) {
  const int half = a.K / 2;
  const int wstride = half + ((64 - half % 128) + 128) % 128;  // = 64 (mod 128)
  constexpr uint32_t kBudget = 227 * 1024;  // one CTA per SM
  int stages = 8;
  while (stages >= 2 && BulkLayout(M, a.K, wstride, stages, RT).total > kBudget) --stages;
  if (stages < 2) return cudaErrorInvalidValue;
  const size_t smem = BulkLayout(M, a.K, wstride, stages, RT).total;
  auto kern = gemv_imma_bulk<M, RT>;
  static std::atomic<bool> attr[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 63].load(std::memory_order_acquire)) {
    const cudaError_t e = set_smem_attrs(kern, static_cast<int>(kBudget));
    if (e != cudaSuccess) return e;
    attr[dev & 63].store(true, std::memory_order_release);
  }
  const int ntiles = a.N / (16 * RT);
  const int grid = ntiles < sms ? ntiles : sms;
  const uint32_t prefetch = static_cast<uint32_t>((48ull << 20) / grid);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32 * (kBulkWarps + 1));
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

// Whether two stages of RT x 16-row tiles of whole rows fit the bulk kernel's shared memory.
template <int M>
bool imma_bulk_fits(int K, int RT) {
  const int half = K / 2;
  const int wstride = half + ((64 - half % 128) + 128) % 128;
  return BulkLayout(M, K, wstride, 2, RT).total <= 227u * 1024;
}

template <int M>
cudaError_t launch_imma_bulk_m(const GemvArgs& a, int sms, cudaStream_t st) {
  if (a.N % 32 == 0 && imma_bulk_fits<M>(a.K, 2)) return launch_imma_bulk<M, 2>(a, sms, st);
  if (a.N % 16 == 0 && imma_bulk_fits<M>(a.K, 1)) return launch_imma_bulk<M, 1>(a, sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace

bool gemv_imma_bulk_ok(const GemvArgs& a) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  // one or two tokens (one n-block of digit columns); more take the bf16-MMA kernels
  if (!(a.M >= 1 && a.M <= 2 && a.group == 128 && a.K % 128 == 0 && a.sz_row == a.K / 128 &&
        a.N % 16 == 0 && (a.ldx % 8) == 0 && al16(a.X) && al16(a.P) && al16(a.S) && al16(a.Z)))
    return false;
  const int rt = a.N % 32 == 0 ? 2 : 1;
  return a.M == 1 ? imma_bulk_fits<1>(a.K, rt) || imma_bulk_fits<1>(a.K, 1)
                  : imma_bulk_fits<2>(a.K, rt) || imma_bulk_fits<2>(a.K, 1);
}

cudaError_t launch_gemv_imma_bulk(const GemvArgs& a, int sms, cudaStream_t st) {
  switch (a.M) {
    case 1: return launch_imma_bulk_m<1>(a, sms, st);
    case 2: return launch_imma_bulk_m<2>(a, sms, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wq
