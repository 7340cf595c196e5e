// Tensor-core W4A16 / W8A16 GEMM for B200 (tcgen05 + TMEM + TMA), Y = X W_hat^T.
// ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
// "The vocabulary": 4-bit weights dequantized to 16 bits inside the kernel, 16-bit matmul;
// the prefill "still runs 16-bit math", so this is the compute-bound half of the path.)
//
// Tile: 128 weight rows (MMA M) x 256 tokens (MMA N), K in stages of 64. The weight tile is
// the MMA's A operand so that a dequantized tile feeds 256 tokens at once. Per CTA
// (persistent, one per SM), warp roles:
//   warp 0      TMA producer: X tiles [256 tokens x 64 k] bf16, 128-byte swizzle, and the
//               tile's raw codes of the same 64 k into the stage ring (both complete on the
//               stage's "raw_full" mbarrier); a stage is refilled once its MMAs are done.
//   warp 1      allocates TMEM (512 columns: one 128 x 256 fp32 accumulator, then the A
//               tile of every stage, 32 columns each); lane 0 issues tcgen05.mma
//               (kind::f16, A from tensor memory, B from shared memory, fp32 accumulation),
//               4 per stage, and commits each stage to its "empty" barrier and each tile to
//               "acc_full".
//   warps 2-9   dequantizers: thread (h, r) owns half h of weight row r of the stage (r is
//               its TMEM lane); it keeps S', Z of the next two stages in flight, forms
//               W_hat = S'(q - Z) exactly in fp32 (one byte-permute per weight, packed
//               fp32x2 FMAs), rounds to bf16 and writes its 32 values as 16 bf16 pairs into
//               its TMEM lane of the stage's A columns (tcgen05.st), so the dequantized
//               tile never passes through shared memory.
//   warps 10-13 epilogue: tcgen05.ld the accumulator (32 rows per warp, its TMEM lane
//               quarter), round to bf16, stage [32 tokens x 128 rows] in shared memory and
//               write it to Y with one TMA store per 32 tokens; the next tile's MMAs start
//               once the accumulator has been read.
// Every mbarrier wait is bounded (2 s): on a timeout the kernel records kStTimeout and all
// roles leave their loops; the TMA lane waits (bounded) for the copies it issued, the MMA
// lane for its last commit, and the CTA frees TMEM and exits.
#include <atomic>

#include "common.cuh"
#include "ptx.cuh"
#include "tc_gemm.h"
#include "tcgen05.cuh"
#include "tma_host.h"

namespace wq {
namespace {

constexpr int kRows = 128;     // weight rows per tile (MMA M)
constexpr int kToks = 256;     // tokens per tile (MMA N)
constexpr int kBK = 64;        // k per stage (one 128-byte swizzle atom of bf16)
constexpr int kBBytes = kToks * kBK * 2;    // 32 KB: X tile
constexpr int kEpiToks = 32;                // tokens per epilogue store
constexpr int kEpiBytes = kEpiToks * kRows * 2;  // 8 KB
// Stage ring depth and raw-code bytes per stage: INT4 keeps 32 B/row, INT8 64 B/row. The
// dequantized weight tile of a stage lives in tensor memory, so shared memory holds only
// the X tile and the raw codes per stage: six stages (five for INT8) cover the copies'
// latency.
template <bool kInt8> struct Cfg {
  static constexpr int kRBytes = kRows * (kInt8 ? kBK : kBK / 2);
  static constexpr int kStages = kInt8 ? 5 : 6;
};
constexpr int kMaxStages = 6;
constexpr int kThreads = 448;  // 14 warps: TMA, MMA, 8 dequant, 4 epilogue
constexpr int kDqWarps = 8;
// TMEM: the 128 x 256 fp32 accumulator in columns 0..255, then per stage the A tile
// (128 lanes x 64 k as bf16 pairs = 32 columns).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACol0 = kToks;
static_assert(kACol0 + 32 * kMaxStages <= kTmemCols, "TMEM");
constexpr uint64_t kLimitNs = 2000000000ull;

struct Smem {
  uint64_t raw_full[kMaxStages];  // TMA: X tile + raw weight codes landed (tx bytes)
  uint64_t full[kMaxStages];      // dequant warps: bf16 weight tile written
  uint64_t empty[kMaxStages];     // tcgen05.commit: the stage's MMAs are done
  uint64_t acc_full;   // the tile's accumulator is complete
  uint64_t acc_empty;  // the epilogue has read it
  uint64_t done;
  uint32_t tmem_base;
  volatile int abort;
};
template <bool kInt8>
constexpr size_t smem_bytes() {
  return 1024 + Cfg<kInt8>::kStages * (kBBytes + Cfg<kInt8>::kRBytes) + kEpiBytes +
         sizeof(Smem);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, M = 128, N = 256.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((kToks >> 3) << 17) |
                            ((kRows >> 4) << 24);

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Smem* sm,
                                              unsigned* status) {
  if (mbar_wait_bounded(bar, parity, kLimitNs)) return true;
  set_status(status, kStTimeout);
  atomicExch(const_cast<int*>(&sm->abort), 1);
  return false;
}

// Eight codes of a 32-bit word (nibble i = code of k = i) -> S'(q - Z), exact in fp32:
// f = 0.5 + q/256 from one byte-permute; 256 S' f - S'(128 + Z) = S'(q - Z).
__device__ __forceinline__ void dq8_int4(uint32_t word, float s256, float c0, float* w) {
  const uint32_t lo = word & 0x0F0F0F0Fu;
  const uint32_t hi = (word >> 4) & 0x0F0F0F0Fu;
  const float2 a2 = make_float2(s256, s256), c2 = make_float2(c0, c0);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t sel = 0x7044u | (static_cast<uint32_t>(j) << 8);
    const float2 f = make_float2(__uint_as_float(__byte_perm(lo, 0x3F000000u, sel)),
                                 __uint_as_float(__byte_perm(hi, 0x3F000000u, sel)));
    const float2 v = __ffma2_rn(f, a2, c2);
    w[2 * j] = v.x;
    w[2 * j + 1] = v.y;
  }
}

// Four int8 codes of a word -> s' q, exact in fp32 (q from 2^23 + (b ^ 0x80) - 2^23 - 128).
__device__ __forceinline__ void dq4_int8(uint32_t word, float s, float* w) {
  const uint32_t u = word ^ 0x80808080u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float q = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440u | j)) - 8388736.0f;
    w[j] = s * q;
  }
}

template <bool kInt8>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
               const __grid_constant__ CUtensorMap tmW, const uint8_t* __restrict__ P,
               const int8_t* __restrict__ Q8,
               const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int M, int N,
               int K, int group, int sz_row, unsigned* status) {
  constexpr int kStages = Cfg<kInt8>::kStages;
  constexpr int kRBytes = Cfg<kInt8>::kRBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* tileB = base;                              // [kStages][kBBytes]
  uint8_t* tileR = tileB + kStages * kBBytes;         // [kStages][kRBytes]
  uint8_t* epi = tileR + kStages * kRBytes;           // [kEpiToks][kRows] bf16
  Smem* sm = reinterpret_cast<Smem*>(epi + kEpiBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = (N + kRows - 1) / kRows;
  const int m_tiles = (M + kToks - 1) / kToks;
  const int tiles = n_tiles * m_tiles;
  const int KB = K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->raw_full[s], 1);       // TMA arrive.expect_tx
      mbar_init(&sm->full[s], kDqWarps);    // dequant warps
      mbar_init(&sm->empty[s], 1);     // tcgen05.commit
    }
    mbar_init(&sm->acc_full, 1);
    mbar_init(&sm->acc_empty, 4);
    mbar_init(&sm->done, 1);
    sm->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      const uint32_t rbytes = kInt8 ? kRows * kBK : kRows * kBK / 2;
      for (int t = blockIdx.x; t < tiles && !sm->abort; t += gridDim.x) {
        const int nt = t / m_tiles, mt = t % m_tiles;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t u = it / kStages;
          if (u > 0 && !wait_or_abort(&sm->empty[s], (u - 1) & 1u, sm, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm->raw_full[s], kBBytes + rbytes);
          tma_load_2d(tileB + s * kBBytes, &tmX, kb * kBK, mt * kToks, &sm->raw_full[s]);
          tma_load_2d(tileR + s * kRBytes, &tmW, kb * (kInt8 ? kBK : kBK / 2), nt * kRows,
                      &sm->raw_full[s]);
        }
        if (!ok) break;
      }
      // never leave with copies in flight (also after an abort): wait, bounded, for the last
      // fill of every stage this lane issued
      for (uint32_t s = 0; s < static_cast<uint32_t>(kStages) && s < it; ++s) {
        const uint32_t last = (it - 1 - s) / kStages;
        if (!mbar_wait_bounded(&sm->raw_full[s], last & 1u, kLimitNs)) set_status(status, kStTimeout);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0, j = 0;
      for (int t = blockIdx.x; t < tiles && !sm->abort; t += gridDim.x, ++j) {
        if (j >= 1 && !wait_or_abort(&sm->acc_empty, (j - 1) & 1u, sm, status)) break;
        tc_fence_after();
        const uint32_t d = tmem;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          if (!wait_or_abort(&sm->raw_full[s], (it / kStages) & 1u, sm, status) ||
              !wait_or_abort(&sm->full[s], (it / kStages) & 1u, sm, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = tmem + kACol0 + 32 * s;  // A: 8 TMEM columns per K = 16
          const uint8_t* bt = tileB + s * kBBytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            tc_mma_tmem_a(d, a + 8 * k, sw128_desc(bt + 32 * k), kIdesc, (kb | k) != 0 ? 1u : 0u);
          tc_commit(&sm->empty[s]);
        }
        if (!ok) break;
        tc_commit(&sm->acc_full);
      }
      // all issued MMAs have completed once this commit arrives
      tc_commit(&sm->done);
      if (!mbar_wait_bounded(&sm->done, 0, kLimitNs)) set_status(status, kStTimeout);
    }
  } else if (warp < 2 + kDqWarps) {
    // ------------------------------------------------------------------ dequantizers
    // Thread = weight row r of the tile (its warp's TMEM lane quarter, its lane) and half h
    // (32 k) of the stage: it writes its 16 bf16 pairs into TMEM lane r, columns 16 h ..
    // 16 h + 15 of the stage's A tile.
    const int quarter = warp & 3;
    const int h = (warp - 2) >> 2;                    // which 32-k half of the stage
    const int r = quarter * 32 + lane;                // weight row within the tile
    const uint32_t a_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kACol0 + 16 * h;
    // (tile, kb) of the iteration whose scales are fetched next, advanced incrementally
    int f_t = blockIdx.x, f_kb = 0;
    auto fetch = [&](float& fa, float& fc) {
      fa = fc = 0.0f;
      if (f_t >= tiles) return;
      const int n = (f_t / m_tiles) * kRows + r;
      if (n < N) {
        if (!kInt8) {
          const int k0 = f_kb * kBK + 32 * h;
          const int64_t gi = static_cast<int64_t>(n) * sz_row + (sz_row ? k0 / group : 0);
          const float sv = f16_bits_to_f32(ld_nc_u16(S + gi));
          const float zv = f16_bits_to_f32(ld_nc_u16(Zp + gi));
          fa = 256.0f * sv;
          fc = -sv * (128.0f + zv);
        } else {
          fa = f16_bits_to_f32(ld_nc_u16(S + n));
        }
      }
      if (++f_kb == KB) {
        f_kb = 0;
        f_t += gridDim.x;
      }
    };
    float a0, c0, a1, c1;
    fetch(a0, c0);
    fetch(a1, c1);
    const uint32_t tileR_s = smem_u32(tileR);
    uint32_t it = 0;
    for (int t = blockIdx.x; t < tiles && !sm->abort; t += gridDim.x) {
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const float ca = a0, cc = c0;
        a0 = a1;
        c0 = c1;
        fetch(a1, c1);
        const int s = it % kStages;
        const uint32_t u = it / kStages;
        // the raw codes of this stage have landed (which also means the stage's previous
        // MMAs, which read its A columns, are done: the TMA for it was issued only after
        // "empty")
        if (!wait_or_abort(&sm->raw_full[s], u & 1u, sm, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t raw = tileR_s + s * kRBytes;
        float w[32];
        if (!kInt8) {
          const uint4 p = lds128(raw + r * (kBK / 2) + 16 * h);
          const uint32_t words[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) dq8_int4(words[q], ca, cc, w + 8 * q);
        } else {
          const uint4 p0 = lds128(raw + r * kBK + 32 * h);
          const uint4 p1 = lds128(raw + r * kBK + 32 * h + 16);
          const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) dq4_int8(words[q], ca, w + 4 * q);
        }
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = pack_bf16x2(w[2 * i], w[2 * i + 1]);
        tmem_st16(a_lane + 32 * s, v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->full[s]);
      }
      if (!ok) break;
    }
  } else {
    // ---------------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 (this warp's access window)
    const int row = quarter * 32 + lane;
    const bool leader = (threadIdx.x == 32 * (2 + kDqWarps));
    uint32_t j = 0;
    for (int t = blockIdx.x; t < tiles && !sm->abort; t += gridDim.x, ++j) {
      const int nt = t / m_tiles, mt = t % m_tiles;
      if (!wait_or_abort(&sm->acc_full, j & 1u, sm, status)) break;
      tc_fence_after();
      const uint32_t st = smem_u32(epi);
      for (int hf = 0; hf < kToks / kEpiToks; ++hf) {
        if (leader) bulk_wait_read0();  // the previous store has read the staging buffer
        named_barrier(2, 128);
        for (int c = 0; c < kEpiToks / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + hf * kEpiToks + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            __nv_bfloat16 hv = __float2bfloat16_rn(__uint_as_float(v[i]));
            sts16(st + ((c * 32 + i) * kRows + row) * 2, *reinterpret_cast<uint16_t*>(&hv));
          }
        }
        if (hf == kToks / kEpiToks - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm->acc_empty);
        }
        fence_async_smem();
        named_barrier(2, 128);
        if (leader) {
          tma_store_2d(&tmY, epi, nt * kRows, mt * kToks + hf * kEpiToks);
          bulk_commit();
        }
      }
    }
    if (leader) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// --- host: tensor maps -----------------------------------------------------------------

bool make_map(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  return make_map_2d(map, ptr, inner, outer, row_bytes, box_inner, box_outer, swizzle128, dtype);
}

}  // namespace

wq_status launch_tc_gemm(const TcGemmArgs& a, int sms, unsigned* status, cudaStream_t st) {
  const bool int8 = a.Q8 != nullptr;
  if (a.K % kBK != 0) return WQ_ERR_SHAPE;
  if (!int8 && a.sz_row && a.group % 32 != 0) return WQ_ERR_SHAPE;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al16(a.X) || !al16(a.Y) || a.ldx % 8 != 0 || a.ldy % 8 != 0) return WQ_ERR_ALIGN;
  if (!al16(int8 ? static_cast<const void*>(a.Q8) : static_cast<const void*>(a.P)))
    return WQ_ERR_ALIGN;
  CUtensorMap mx, my, mw;
  if (!make_map(&mx, a.X, a.K, a.M, a.ldx * 2, kBK, kToks, true)) return WQ_ERR_CUDA;
  if (!make_map(&my, a.Y, a.N, a.M, a.ldy * 2, kRows, kEpiToks, false)) return WQ_ERR_CUDA;
  if (int8) {
    if (!make_map(&mw, a.Q8, a.K, a.N, a.K, kBK, kRows, false, CU_TENSOR_MAP_DATA_TYPE_UINT8))
      return WQ_ERR_CUDA;
  } else if (!make_map(&mw, a.P, a.K / 2, a.N, a.K / 2, kBK / 2, kRows, false,
                       CU_TENSOR_MAP_DATA_TYPE_UINT8)) {
    return WQ_ERR_CUDA;
  }
  auto kern = int8 ? tc_gemm_kernel<true> : tc_gemm_kernel<false>;
  const size_t smem = int8 ? smem_bytes<true>() : smem_bytes<false>();
  // the attribute is per device: set it on each device's first call (flags by device)
  static std::atomic<bool> attr[64][2];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
  if (!attr[dev & 63][int8].load(std::memory_order_acquire)) {
    if (set_smem_attrs(kern, static_cast<int>(smem)) != cudaSuccess)
      return WQ_ERR_CUDA;
    attr[dev & 63][int8].store(true, std::memory_order_release);
  }
  const int tiles = ((a.N + kRows - 1) / kRows) * ((a.M + kToks - 1) / kToks);
  const int grid = tiles < sms ? tiles : sms;
  kern<<<grid, kThreads, smem, st>>>(mx, my, mw, a.P, a.Q8, a.S, a.Z, a.M, a.N, a.K, a.group,
                                           a.sz_row, status);
  return cudaGetLastError() == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

}  // namespace wq
