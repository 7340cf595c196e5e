// Skinny W4A16 / W8A16 matmul (a handful to 64 tokens) on the 5th-generation tensor core:
// Y = X W_hat^T, the weights read once for every token count.
// ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
// "The vocabulary": 4-bit weights, 16-bit activations, fp32 accumulation; "Overview": decode
// reads every weight once.)
//
// INT4, g = 128. Per group of 128 k and weight row n,
//     sum_k x_k S'(q_k - Z) = S' D,   D = sum_k (q_k - Z) x_k,
// where the centred codes q - Z (integers in [-15, 15], exact in bf16) are the MMA's A
// operand (M = 128 weight rows) and the activations, bf16 as stored, its B operand
// (N = MT token columns): eight tcgen05.mma kind::f16 (K = 16) per group into a fresh fp32
// TMEM accumulator. Every product is exact in fp32; D is their fp32 sum, and the epilogue
// adds S' D into the row's fp32 accumulators.
//
// W8A16 (s' per row): per group, sum_k x_k q_k = 2^-s sum_i 2^(8i) D_i, where per token x_k 2^s
// is rounded to an integer below 2^22 in magnitude (s from the token's largest exponent in the
// group: exact within 2^14 of the group's largest |x|, else off by at most 2^-23 of it) and
// split into three signed bytes d_i (balanced digits), and D_i = sum_k q_k d_i,k are exact
// s32 dot products: the s8 codes are A (copied by TMA as stored), the digit planes B
// (N = 3 MT columns), one tcgen05.mma kind::i8 per 32 k; s' multiplies the finished row.
//
// A CTA owns a 128-row tile and a contiguous range of its groups; the CTAs of a cluster
// split K and sum their partial rows through distributed shared memory in rank order
// (deterministic). Warp roles per CTA:
//   warp 0       TMA producer. INT4: per group, the tile's packed codes ([128 rows x 64 B]
//                box) into the load ring, and the activations (two 128-byte-swizzled
//                [MT tokens x 64 k] bf16 boxes) into the operand stage. W8A16: the s8 code
//                box (128-byte swizzled) into the operand stage, the activations
//                ([MT tokens x 128 k]) into the load ring;
//   warp 1       TMEM allocation; lane 0 issues the MMAs of a group once its A and B tiles
//                are in place and a TMEM accumulator is free, commits the stage and the
//                accumulator;
//   INT4: 8 warps of code expansion: each thread turns a half row (32 packed bytes) into
//                bf16 pairs q - Z in the 128-byte-swizzled K-major A tile (two atoms);
//   W8A16: 8 warps of activation digits: 8 threads per token, 16 k each: the group's
//                exponent, the digit planes into the swizzled B tile, and 2^-s;
//   last 4 (8 at MT = 64) warps  epilogue: thread = TMEM lane = weight row (at MT = 64 two
//                warps per lane quarter, each for half the tokens); reads the group's
//                accumulator columns, scales them, accumulates fp32.
// Every mbarrier wait is bounded (2 s): on a timeout the kernel records kStTimeout, every role
// leaves its loop, the producer waits (bounded) for its copies, the MMA lane for its last
// commit, and the CTA frees TMEM and returns.
#include <atomic>
#include <cooperative_groups.h>

#include "common.cuh"
#include "imma_digits.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tcgen05.cuh"
#include "tma_host.h"

namespace cg = cooperative_groups;

namespace wq {
namespace {

constexpr int kRows = 128;                 // weight rows per tile (MMA M)
constexpr int kGK = 128;                   // k per group (one stage)
constexpr int kRawBytes = kRows * kGK / 2;  // packed codes of a stage: 8 KB
constexpr int kABytes = kRows * kGK;        // u8 codes, 128-byte rows: 16 KB
constexpr uint64_t kLimitNs = 2000000000ull;
constexpr uint32_t kTmemCols = 512;
// The expansion and epilogue roles load Z and S' of a group this many groups ahead, into
// register rings: a group's work is much shorter than a round trip to DRAM.
constexpr int kAhead = 8;

// Operand modes:
//   kModeW8     INT8 symmetric per-channel weights (W8A16): the s8 codes are the A operand
//               as they are. The producer copies each [128 rows x 128 k] box with TMA
//               straight into the operand stage in the 128-byte-swizzled layout, so there is
//               no expansion role; the row's scale s' is applied once, to the finished row.
//   kModeI4Bf   INT4 codes: centred codes q - Z as bf16 (exact: integers in [-15, 15]) x the
//               activations as they are, bf16 (kind::f16 with fp32 accumulation; every
//               product is exact in fp32). The producer copies X with TMA straight into the
//               operand stage (two 128-byte-swizzled boxes of 64 k per group), so there is no
//               digit role, and the epilogue applies S' to one accumulator column per token.
enum SkMode { kModeW8 = 1, kModeI4Bf = 2 };

template <int MT, int kMode>
struct SkCfg {
  static constexpr bool kW8m = kMode == kModeW8, kBf = kMode == kModeI4Bf;
  static constexpr int NC = kBf ? MT : 3 * MT;           // accumulator columns per group
  static constexpr int kA = kBf ? 2 * kABytes : kABytes;  // A operand bytes (bf16: two atoms)
  static constexpr int kBBytes = kBf ? MT * kGK * 2 : NC * kGK;  // X tile or digit planes
  static constexpr int kXBytes = kBf ? 0 : MT * kGK * 2;  // activations in the load ring
  static constexpr int kMetaBytes = kBf ? 0 : MT * 4;     // per token: 2^-s
  // operand ring (A | B | 2^-s), freed by the MMA (and the epilogue, which reads 2^-s)
  static constexpr int kMetaOff = kA + kBBytes;
  static constexpr int kOpBytes = (kMetaOff + kMetaBytes + 1023) / 1024 * 1024;
  static constexpr int kOpStages = kBf ? 4 : (MT <= 16 ? 6 : (MT <= 32 ? 4 : 3));
  // load ring (packed codes | activations), freed once expansion and digits have read it
  static constexpr int kRawLd = kW8m ? 0 : kRawBytes;
  static constexpr int kXOff = kRawLd;
  static constexpr int kLdBytes = (kRawLd + kXBytes + 1023) / 1024 * 1024;
  static constexpr int kLdStages = MT <= 16 ? 6 : (MT <= 32 ? (kBf ? 6 : 5) : 3);
  static constexpr int kBufs = (kBf || MT <= 32) ? 4 : 2;  // TMEM accumulators in flight
  static constexpr int kChunk = (kBf || MT <= 16) ? 16 : 8;  // tokens per epilogue TMEM load
  // code-expansion warps (INT4): 8, one half row per thread
  static constexpr int kDecWarps = kW8m ? 0 : 8;
  static constexpr int kPrepWarps = kBf ? 0 : 8;  // activation digits
  // epilogue warps: one per TMEM lane quarter, or two at MT = 64, each then keeping the
  // accumulators of half the tokens (32 registers instead of 64)
  static constexpr int kEpiWarps = MT <= 32 ? 4 : 8;
  static constexpr int kEpiTok = MT / (kEpiWarps / 4);  // tokens per epilogue thread
  static constexpr int kThreads = 32 * (2 + kDecWarps + kPrepWarps + kEpiWarps);
  static_assert(kBufs * NC <= static_cast<int>(kTmemCols), "TMEM");
  static_assert(kRows * MT * 4 <= kOpBytes, "cluster partials fit in operand stage 0");
  static_assert(kOpStages <= 6 && kLdStages <= 6, "barrier arrays");
  static_assert(kEpiTok % kChunk == 0, "epilogue chunks");
};

struct SkBars {
  uint64_t ld_full[6];   // TMA: a load stage's codes and activations landed
  uint64_t ld_empty[6];  // expansion and digit warps have read the load stage
  uint64_t a_full[6];    // code expansion (W8A16: the TMA copy) into the operand stage done
  uint64_t b_full[6];    // digit planes and 2^-s done
  uint64_t op_empty[6];  // operand stage free: the MMAs are done and the epilogue read 2^-s
  uint64_t acc_full[4];  // a group's accumulator is complete
  uint64_t acc_empty[4]; // the epilogue has read it
  uint64_t done;
  uint32_t tmem_base;
  volatile int abort;
};

template <int MT, int kMode>
constexpr size_t sk_smem_bytes() {
  using C = SkCfg<MT, kMode>;
  return 1024 + C::kOpStages * C::kOpBytes + C::kLdStages * C::kLdBytes + sizeof(SkBars);
}

// Instruction descriptor, kind::i8: D s32, A s8, B s8, both K-major, M = 128, N = nc.
__host__ __device__ constexpr uint32_t idesc_i8(int nc) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nc >> 3) << 17) |
         (static_cast<uint32_t>(kRows >> 4) << 24);
}
// Instruction descriptor, kind::f16: D fp32, A bf16, B bf16, both K-major, M = 128, N = nc.
__host__ __device__ constexpr uint32_t idesc_bf16(int nc) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nc >> 3) << 17) |
         (static_cast<uint32_t>(kRows >> 4) << 24);
}

// Every handoff of this kernel is on the critical path of a short stage, so waits poll
// (bounded) instead of suspending the warp, whose wake-up is coarser than a stage.
__device__ __forceinline__ bool sk_wait(uint64_t* bar, uint32_t parity, SkBars* sb,
                                        unsigned* status) {
  if (mbar_wait_spin_bounded(bar, parity, kLimitNs)) return true;
  set_status(status, kStTimeout);
  atomicExch(const_cast<int*>(&sb->abort), 1);
  return false;
}

// a - b on two packed bf16 values (exact where the difference is representable)
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  const __nv_bfloat162 d =
      __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&a), *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<const uint32_t*>(&d);
}

// 16-byte chunk c (0..7) of row r in a K-major tile with 128-byte rows, 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
}

template <int MT, int kMode>
__global__ void __launch_bounds__(SkCfg<MT, kMode>::kThreads, 1)
tc_skinny_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                 const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int M, int N,
                 int K, uint16_t* __restrict__ Y, int64_t ldy, unsigned* status) {
  using C = SkCfg<MT, kMode>;
  constexpr bool kW8m = C::kW8m, kBf = C::kBf;
  constexpr int kPrepWarps = C::kPrepWarps, kA = C::kA;
  constexpr int NC = C::NC, kOpStages = C::kOpStages, kLdStages = C::kLdStages,
                kBufs = C::kBufs;
  constexpr int kDecWarps = C::kDecWarps, kThreads = C::kThreads, kEpiWarps = C::kEpiWarps;
  constexpr int kEpiTok = C::kEpiTok;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ldbase = base + kOpStages * C::kOpBytes;
  SkBars* sb = reinterpret_cast<SkBars*>(ldbase + kLdStages * C::kLdBytes);
  auto opst = [&](int s) { return base + s * C::kOpBytes; };    // A | B | 2^-s
  auto ldst = [&](int s) { return ldbase + s * C::kLdBytes; };  // codes | activations

  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int csize = static_cast<int>(cluster.num_blocks());
  const int tile = blockIdx.x / csize;
  const int n0 = tile * kRows;
  const int G = K / kGK;
  const int g0 = static_cast<int>((static_cast<int64_t>(crank) * G) / csize);
  const int g1 = static_cast<int>((static_cast<int64_t>(crank + 1) * G) / csize);
  const int ng = g1 - g0;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLdStages; ++s) {
      mbar_init(&sb->ld_full[s], 1);
      mbar_init(&sb->ld_empty[s], kDecWarps + kPrepWarps);
    }
    for (int s = 0; s < kOpStages; ++s) {
      mbar_init(&sb->a_full[s], kW8m ? 1 : kDecWarps);
      mbar_init(&sb->b_full[s], kBf ? 1 : kPrepWarps);
      mbar_init(&sb->op_empty[s], kBf ? 1 : 1 + kEpiWarps);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(&sb->acc_full[b], 1);
      mbar_init(&sb->acc_empty[b], kEpiWarps);
    }
    mbar_init(&sb->done, 1);
    sb->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sb->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sb->tmem_base;
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();  // X, the codes, S and Z are read only after the previous kernel completed

  float acc[kEpiTok];
#pragma unroll
  for (int m = 0; m < kEpiTok; ++m) acc[m] = 0.0f;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int nld = 0, nop = 0;  // load-ring fills and operand-stage copies issued
      for (int it = 0; it < ng && !sb->abort; ++it) {
        const int s = it % kLdStages;
        const uint32_t u = it / kLdStages;
        if (u > 0 && !sk_wait(&sb->ld_empty[s], (u - 1) & 1u, sb, status)) break;
        mbar_arrive_expect_tx(&sb->ld_full[s], C::kRawLd + C::kXBytes);
        if constexpr (!kW8m) tma_load_2d(ldst(s), &tmW, (g0 + it) * (kGK / 2), n0, &sb->ld_full[s]);
        if constexpr (!kBf) tma_load_2d(ldst(s) + C::kXOff, &tmX, (g0 + it) * kGK, 0, &sb->ld_full[s]);
        ++nld;
        if constexpr (kW8m || kBf) {
          // straight into the operand stage (swizzled): the s8 codes (A) or the activations (B)
          const int os = it % kOpStages;
          const uint32_t ou = it / kOpStages;
          if (ou > 0 && !sk_wait(&sb->op_empty[os], (ou - 1) & 1u, sb, status)) break;
          if constexpr (kW8m) {
            mbar_arrive_expect_tx(&sb->a_full[os], kABytes);
            tma_load_2d(opst(os), &tmW, (g0 + it) * kGK, n0, &sb->a_full[os]);
          } else {
            mbar_arrive_expect_tx(&sb->b_full[os], C::kBBytes);
            tma_load_2d(opst(os) + kA, &tmX, (g0 + it) * kGK, 0, &sb->b_full[os]);
            tma_load_2d(opst(os) + kA + MT * 128, &tmX, (g0 + it) * kGK + 64, 0, &sb->b_full[os]);
          }
          ++nop;
        }
      }
      // no copy left in flight on exit: wait (bounded) for the last fill of every stage
      for (int s = 0; s < kLdStages && s < nld; ++s) {
        const uint32_t last = (nld - 1 - s) / kLdStages;
        if (!mbar_wait_bounded(&sb->ld_full[s], last & 1u, kLimitNs)) set_status(status, kStTimeout);
      }
      for (int s = 0; s < kOpStages && s < nop; ++s) {
        const uint32_t last = (nop - 1 - s) / kOpStages;
        uint64_t* bar = kW8m ? &sb->a_full[s] : &sb->b_full[s];
        if (!mbar_wait_bounded(bar, last & 1u, kLimitNs)) set_status(status, kStTimeout);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int it = 0;
      for (; it < ng && !sb->abort; ++it) {
        const int s = it % kOpStages, b = it % kBufs;
        const uint32_t u = it / kOpStages, v = it / kBufs;
        if (!sk_wait(&sb->a_full[s], u & 1u, sb, status) ||
            !sk_wait(&sb->b_full[s], u & 1u, sb, status) ||
            (v > 0 && !sk_wait(&sb->acc_empty[b], (v - 1) & 1u, sb, status)))
          break;
        tc_fence_after();
        const uint8_t* a = opst(s);
        const uint8_t* bt = opst(s) + kA;
        const uint32_t d = tmem + b * NC;
        if constexpr (kBf) {
          // K = 16 per MMA; k 0..63 in the first 128-byte-swizzled atom of each operand
#pragma unroll
          for (int k = 0; k < kGK / 16; ++k)
            tc_mma(d, sw128_desc(a + (k >> 2) * kABytes + 32 * (k & 3)),
                   sw128_desc(bt + (k >> 2) * (MT * 128) + 32 * (k & 3)), idesc_bf16(NC),
                   k != 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int k = 0; k < kGK / 32; ++k)
            tc_mma_i8(d, sw128_desc(a + 32 * k), sw128_desc(bt + 32 * k), idesc_i8(NC),
                      k != 0 ? 1u : 0u);
        }
        tc_commit(&sb->op_empty[s]);
        tc_commit(&sb->acc_full[b]);
      }
      tc_commit(&sb->done);  // arrives once every MMA issued above has completed
      if (!mbar_wait_bounded(&sb->done, 0, kLimitNs)) set_status(status, kStTimeout);
    }
  } else if (warp < 2 + kDecWarps) {
    if constexpr (kBf) {
    // --------------------------------------------------------------- code expansion
    // Half h of a row (64 k) is that row of A's atom h. The 8 threads of a quarter-warp take
    // 8 consecutive rows (distinct store slots) and both halves (reads spread over 4 slots);
    // the quarter-warp after it takes the same rows' other halves.
    constexpr int kPairs = 256 / (32 * kDecWarps);
    const int t = threadIdx.x - 64;
    const int G = K / kGK;
    auto pair_rh = [&](int pp, int& r, int& h) {
      const int pr = t + 32 * kDecWarps * pp;
      r = 8 * (pr >> 4) + (pr & 7);
      h = ((pr >> 3) & 1) ^ ((pr >> 1) & 1);
    };
    int64_t zrow[kPairs];
#pragma unroll
    for (int pp = 0; pp < kPairs; ++pp) {
      int r, h;
      pair_rh(pp, r, h);
      const int n = n0 + r;
      zrow[pp] = n < N ? static_cast<int64_t>(n) * G : -1;  // rows past N: codes and Z are 0
    }
    // Z of the rows, as 128 + Z in both bf16 halves
    auto ld_z = [&](int it, uint32_t (&z4)[kPairs]) {
#pragma unroll
      for (int pp = 0; pp < kPairs; ++pp) {
        const uint32_t z =
            it < ng && zrow[pp] >= 0
                ? static_cast<uint32_t>(f16_bits_to_f32(ld_nc_u16(Zp + zrow[pp] + g0 + it)))
                : 0u;
        z4[pp] = z * 0x00010001u + 0x43004300u;
      }
    };
    uint32_t zq[kAhead][kPairs];
#pragma unroll
    for (int j = 0; j < kAhead; ++j) ld_z(j, zq[j]);
    for (int it0 = 0; it0 < ng && !sb->abort; it0 += kAhead) {
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      const int it = it0 + j;
      if (it >= ng || sb->abort) break;
      const int ls = it % kLdStages, os = it % kOpStages;
      const uint32_t ou = it / kOpStages;
      if (!sk_wait(&sb->ld_full[ls], (it / kLdStages) & 1u, sb, status) ||
          (ou > 0 && !sk_wait(&sb->op_empty[os], (ou - 1) & 1u, sb, status)))
        break;
      const uint32_t raw = smem_u32(ldst(ls));
      const uint32_t at = smem_u32(opst(os));
#pragma unroll
      for (int pp = 0; pp < kPairs; ++pp) {
        int r, h;
        pair_rh(pp, r, h);
        const uint4 p0 = lds128(raw + r * 64 + 32 * h), p1 = lds128(raw + r * 64 + 32 * h + 16);
        const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        const uint32_t zb = zq[j][pp];  // Z of this group (ring slot j)
        // word c = codes 8c .. 8c + 7 of the half row = 16-byte chunk c of its atom row.
        // bf16 pair e: byte e of the word (low half) and of the word >> 4 (high half), low
        // nibbles kept and 0x4300 set: 128 + code exactly; minus 128 + Z: q - Z exactly.
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t x = w[c], y = w[c] >> 4;
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t sel = static_cast<uint32_t>(e | (e << 4) | ((4 + e) << 8) | ((4 + e) << 12));
            o[e] = bf16x2_sub((__byte_perm(x, y, sel) & 0x000F000Fu) | 0x43004300u, zb);
          }
          sts128(at + h * kABytes + sw128_off(r, c), make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sb->ld_empty[ls]);
        mbar_arrive(&sb->a_full[os]);
      }
      ld_z(it + kAhead, zq[j]);
    }
    }
    }
  } else if (warp < 2 + kDecWarps + kPrepWarps) {
    if constexpr (!kBf) {
    // ------------------------------------------------------------- activation digits
    const int tp = threadIdx.x - 32 * (2 + kDecWarps);  // 0..255
    constexpr int kPrepThreads = 32 * kPrepWarps;
    // (token, 16-k chunk) items per thread: MT * 8 items in all; with fewer items than
    // threads, whole warps past them stay idle (the test below is warp-uniform)
    constexpr int kItems = (MT * 8 + kPrepThreads - 1) / kPrepThreads;
    for (int it = 0; it < ng && !sb->abort; ++it) {
      const int ls = it % kLdStages, os = it % kOpStages;
      const uint32_t ou = it / kOpStages;
      if (!sk_wait(&sb->ld_full[ls], (it / kLdStages) & 1u, sb, status) ||
          (ou > 0 && !sk_wait(&sb->op_empty[os], (ou - 1) & 1u, sb, status)))
        break;
      const uint32_t xs_s = smem_u32(ldst(ls) + C::kXOff);   // [MT tokens][128 k] bf16
      const uint32_t bt = smem_u32(opst(os) + kABytes);
      float* meta = reinterpret_cast<float*>(opst(os) + C::kMetaOff);
#pragma unroll
      for (int j = 0; j < kItems; ++j) {
        const int item = tp + kPrepThreads * j;
        if (item >= MT * 8) break;
        const int m = item >> 3, c = item & 7;  // token, 16-k chunk (8 lanes per token)
        const uint4 u0 = lds128(xs_s + m * 256 + 32 * c), u1 = lds128(xs_s + m * 256 + 32 * c + 16);
        const uint32_t wds[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        uint32_t e2 = 0;  // exponent fields of both halves, maximised pairwise
#pragma unroll
        for (int i = 0; i < 8; ++i) e2 = __vmaxu2(e2, wds[i] & 0x7F807F80u);
        uint32_t e = max(e2 & 0xFFFFu, e2 >> 16) >> 7;
        e = max(e, __shfl_xor_sync(0xffffffffu, e, 1));
        e = max(e, __shfl_xor_sync(0xffffffffu, e, 2));
        e = max(e, __shfl_xor_sync(0xffffffffu, e, 4));
        uint32_t z[16];
        float p;
        if (e == 0xFFu) {  // inf or NaN in the token's group: its products are not finite
          p = __uint_as_float(0x7FC00000u);
#pragma unroll
          for (int i = 0; i < 16; ++i) z[i] = 0u;
        } else {
          // s = 21 - (exponent of the largest |x|), so |x 2^s| < 2^22. Two values per packed
          // FMA: x 2^s + 1.5 2^23 with one rounding (x 2^s is exact; for groups below 2^-106,
          // 2^s is applied as 2^100 2^(s - 100)), i.e. x_int in the low bits; then the
          // balanced signed bytes as in the integer decode path.
          const int sc = 21 - (static_cast<int>(e < 1u ? 1u : e) - 127);
          const bool split = sc > 127;
          const float f1 = pow2i(100);
          const float sf = split ? pow2i(sc - 100) : pow2i(sc);
          const float2 sf2 = make_float2(sf, sf), mg2 = make_float2(kImmaMagic, kImmaMagic);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float2 v = make_float2(__uint_as_float(wds[i] << 16),
                                   __uint_as_float(wds[i] & 0xFFFF0000u));
            if (split) {
              v.x *= f1;
              v.y *= f1;
            }
            const float2 t = __ffma2_rn(v, sf2, mg2);
            constexpr uint32_t kOff = 0x808080u - static_cast<uint32_t>(kImmaMagicBits);
            z[2 * i] = (static_cast<uint32_t>(__float_as_int(t.x)) + kOff) ^ 0x808080u;
            z[2 * i + 1] = (static_cast<uint32_t>(__float_as_int(t.y)) + kOff) ^ 0x808080u;
          }
          p = pow2i(-sc);
        }
        // digit plane i: bytes i of z[0..15], 16 consecutive k of token m
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const uint32_t sel = static_cast<uint32_t>(i | ((4 + i) << 4));
          uint32_t v[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            v[q] = __byte_perm(__byte_perm(z[4 * q], z[4 * q + 1], sel),
                               __byte_perm(z[4 * q + 2], z[4 * q + 3], sel), 0x5410);
          sts128(bt + sw128_off(i * MT + m, c), make_uint4(v[0], v[1], v[2], v[3]));
        }
        if (c == 0) meta[m] = m < M ? p : 0.0f;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sb->ld_empty[ls]);
        mbar_arrive(&sb->b_full[os]);
      }
    }
    }
  } else {
    // ---------------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32 quarter .. + 31 (this warp's window)
    const int row = quarter * 32 + lane;
    const int tb = ((warp - (2 + kDecWarps + kPrepWarps)) >> 2) * kEpiTok;  // first token
    const int n = n0 + row;
    const bool live = n < N;
    const int64_t szrow = static_cast<int64_t>(live ? n : 0) * G;
    // S' of this row (W8A16: the row's scale is applied once, to the finished row)
    auto ld_s = [&](int it) {
      if constexpr (kW8m) return live ? 1.0f : 0.0f;
      else return it < ng && live ? f16_bits_to_f32(ld_nc_u16(S + szrow + g0 + it)) : 0.0f;
    };
    float sq[kAhead];
#pragma unroll
    for (int j = 0; j < kAhead; ++j) sq[j] = ld_s(j);
    for (int it0 = 0; it0 < ng && !sb->abort; it0 += kAhead) {
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      const int it = it0 + j;
      if (it >= ng || sb->abort) break;
      const int s = it % kOpStages, b = it % kBufs;
      if (!sk_wait(&sb->acc_full[b], (it / kBufs) & 1u, sb, status)) break;
      tc_fence_after();
      const float* meta = reinterpret_cast<const float*>(opst(s) + C::kMetaOff);  // 2^-s
      const float sv = sq[j];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + b * NC;
      constexpr int CH = C::kChunk;
#pragma unroll
      for (int mc = 0; mc < kEpiTok / CH; ++mc) {
        if constexpr (kBf) {  // one fp32 column per token: acc += S' D
          uint32_t d[16];
          tmem_ld16(taddr + tb + CH * mc, d);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < CH; ++i) acc[CH * mc + i] = fmaf(sv, __uint_as_float(d[i]), acc[CH * mc + i]);
          continue;
        }
        uint32_t d0[CH], d1[CH], d2[CH];
        const uint32_t col = tb + CH * mc;
        if constexpr (CH == 16) {
          tmem_ld16(taddr + 0 * MT + col, d0);
          tmem_ld16(taddr + 1 * MT + col, d1);
          tmem_ld16(taddr + 2 * MT + col, d2);
        } else {
          tmem_ld8(taddr + 0 * MT + col, d0);
          tmem_ld8(taddr + 1 * MT + col, d1);
          tmem_ld8(taddr + 2 * MT + col, d2);
        }
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < CH; ++i) {
          const int m = CH * mc + i;
          // |D_i| < 2^21 (2^18 with INT4 codes): digits 0 and 1 combine exactly in 32 bits
          const int d01 = static_cast<int>(d0[i]) + 256 * static_cast<int>(d1[i]);
          const float v = fmaf(65536.0f, static_cast<float>(static_cast<int>(d2[i])),
                               static_cast<float>(d01));
          acc[m] = fmaf(sv * meta[tb + m], v, acc[m]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sb->acc_empty[b]);
        if constexpr (!kBf) mbar_arrive(&sb->op_empty[s]);  // 2^-s read
      }
      sq[j] = ld_s(it + kAhead);
    }
    }
  }

  // ---- sum the cluster's partial rows in rank order and write Y. Every thread of every CTA
  // of the cluster takes a share of the tile's (token, row) outputs and issues its reads of
  // the ranks' partials together (one distributed-shared-memory latency, not one per value).
  tc_fence_before();
  __syncthreads();  // every role is done with the stages: the partials reuse operand stage 0
  float* part = reinterpret_cast<float*>(base);  // [MT][kRows]
  if (warp >= 2 + kDecWarps + kPrepWarps) {
    const int row = (warp & 3) * 32 + lane;
    const int tb = ((warp - (2 + kDecWarps + kPrepWarps)) >> 2) * kEpiTok;
#pragma unroll
    for (int j = 0; j < kEpiTok; ++j) part[(tb + j) * kRows + row] = acc[j];
  }
  cluster.sync();
  if (!sb->abort) {
    const float* parts[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) parts[r] = cluster.map_shared_rank(part, r < csize ? r : 0);
    for (int o = crank * kThreads + threadIdx.x; o < M * kRows; o += csize * kThreads) {
      const int m = o / kRows, row = o - m * kRows;
      float v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) v[r] = r < csize ? parts[r][o] : 0.0f;
      float t = v[0];
#pragma unroll
      for (int r = 1; r < 8; ++r)
        if (r < csize) t += v[r];  // rank order
      if (n0 + row < N) {
        if constexpr (kW8m) t *= f16_bits_to_f32(ld_nc_u16(S + n0 + row));
        __nv_bfloat16 hv = __float2bfloat16_rn(t);
        Y[static_cast<int64_t>(m) * ldy + n0 + row] = *reinterpret_cast<uint16_t*>(&hv);
      }
    }
  }
  cluster.sync();  // the other CTAs' partials stay alive until every rank has read them
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Split-K factor (cluster size) for a shape: the smallest of 1, 2, 4, 8 that minimises the
// makespan, waves x (groups per CTA + a CTA's fixed cost of about six groups' time: launch,
// pipeline fill, cluster reduction), at one CTA per SM.
int pick_split(int tiles, int G, int sms) {
  constexpr int64_t kFixedGroups = 6;
  int best = 1;
  int64_t best_cost = -1;
  for (int cs : {1, 2, 4, 8}) {
    if (cs > G) break;
    const int64_t ctas = static_cast<int64_t>(tiles) * cs;
    const int64_t waves = (ctas + sms - 1) / sms;
    const int64_t cost = waves * ((G + cs - 1) / cs + kFixedGroups);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = cs;
    }
  }
  return best;
}

template <int MT, int kMode>
cudaError_t launch_mt(const GemvArgs& a, const CUtensorMap& map, int sms, cudaStream_t st) {
  // activations as [M rows][K] bf16: boxes of 128 k x MT tokens (rows past M read as zero),
  // or, as the bf16 MMA operand, 128-byte-swizzled boxes of 64 k x MT tokens; kept per
  // thread for the last few activation buffers (decode loops reuse them)
  constexpr bool kBf = kMode == kModeI4Bf;
  struct XEntry {
    const void* p;
    int m, k;
    int64_t ld;
    CUtensorMap map;
  };
  constexpr int kXCache = 8;
  thread_local XEntry xcache[kXCache];
  thread_local int xnext = 0;
  const CUtensorMap* xmap = nullptr;
  for (const XEntry& e : xcache)
    if (e.p == a.X && e.m == a.M && e.k == a.K && e.ld == a.ldx) xmap = &e.map;
  if (!xmap) {
    XEntry& e = xcache[xnext];
    e.p = nullptr;
    if (!make_map_2d(&e.map, a.X, static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M),
                     static_cast<uint64_t>(a.ldx) * 2, kBf ? 64 : kGK, MT, kBf,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      return cudaErrorInvalidValue;
    e.p = a.X;
    e.m = a.M;
    e.k = a.K;
    e.ld = a.ldx;
    xnext = (xnext + 1) % kXCache;
    xmap = &e.map;
  }
  auto kern = tc_skinny_kernel<MT, kMode>;
  const size_t smem = sk_smem_bytes<MT, kMode>();
  static std::atomic<bool> attr[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 63].load(std::memory_order_acquire)) {
    const cudaError_t e = set_smem_attrs(kern, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr[dev & 63].store(true, std::memory_order_release);
  }
  const int tiles = (a.N + kRows - 1) / kRows;
  const int G = a.K / kGK;
  const int cs = pick_split(tiles, G, sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * cs);
  cfg.blockDim = dim3(SkCfg<MT, kMode>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = cs;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, map, *xmap, a.S, a.Z, a.M, a.N, a.K, a.Y, a.ldy,
                            a.status);
}

}  // namespace

namespace {

// Tensor map of the weights, kept per thread for the last few matrices (decode calls
// repeat): INT4 packed codes as [N rows][K/2 bytes] in boxes of 64 bytes (one group) x 128
// rows; INT8 codes as [N rows][K bytes] in 128-byte-swizzled boxes of 128 x 128 bytes.
const CUtensorMap* weight_map(const void* P, int N, int K, bool w8) {
  struct MapEntry {
    const void* p;
    int n, k;
    bool w8;
    CUtensorMap map;
  };
  constexpr int kMapCache = 16;
  thread_local MapEntry cache[kMapCache];
  thread_local int next_slot = 0;
  for (const MapEntry& e : cache)
    if (e.p == P && e.n == N && e.k == K && e.w8 == w8) return &e.map;
  MapEntry& e = cache[next_slot];
  e.p = nullptr;
  const uint64_t row = w8 ? static_cast<uint64_t>(K) : static_cast<uint64_t>(K / 2);
  if (!make_map_2d(&e.map, P, row, static_cast<uint64_t>(N), row, w8 ? kGK : kGK / 2, kRows,
                   w8, CU_TENSOR_MAP_DATA_TYPE_UINT8))
    return nullptr;
  e.p = P;
  e.n = N;
  e.k = K;
  e.w8 = w8;
  next_slot = (next_slot + 1) % kMapCache;
  return &e.map;
}

template <int kMode>
cudaError_t launch_skinny(const GemvArgs& a, int sms, cudaStream_t st) {
  const CUtensorMap* map = weight_map(a.P, a.N, a.K, kMode == kModeW8);
  if (!map) return cudaErrorInvalidValue;
  if (a.M <= 16) return launch_mt<16, kMode>(a, *map, sms, st);
  if (a.M <= 32) return launch_mt<32, kMode>(a, *map, sms, st);
  return launch_mt<64, kMode>(a, *map, sms, st);
}

bool skinny_common_ok(const GemvArgs& a) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return a.M >= 1 && a.M <= kSkinnyMaxTokens && a.K % 128 == 0 && a.N >= 1 &&
         a.ldx % 8 == 0 && al16(a.X) && al16(a.P);
}

}  // namespace

bool tc_skinny_ok(const GemvArgs& a) {
  return skinny_common_ok(a) && a.group == 128 && a.sz_row == a.K / 128;
}

cudaError_t launch_tc_skinny(const GemvArgs& a, int sms, cudaStream_t st) {
  if (!tc_skinny_ok(a)) return cudaErrorInvalidValue;
  return launch_skinny<kModeI4Bf>(a, sms, st);
}

bool tc_skinny8_ok(const GemvArgs& a) { return skinny_common_ok(a); }

cudaError_t launch_tc_skinny8(const GemvArgs& a, int sms, cudaStream_t st) {
  if (!tc_skinny8_ok(a)) return cudaErrorInvalidValue;
  return launch_skinny<kModeW8>(a, sms, st);
}

}  // namespace wq
