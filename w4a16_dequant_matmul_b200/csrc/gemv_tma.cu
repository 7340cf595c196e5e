// Small-M W4A16 matmul (decode) on 32-row weight tiles fed by TMA: Y = X W_hat^T for
// M <= 4 tokens, group size 128, N a multiple of 32. Used where a 32-row tile of whole rows is
// too large to double-buffer in shared memory (long rows, K above about 6K).
// ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
// "The vocabulary" and the decode discussion: 4-bit weights dequantized inside the kernel;
// at decode the matmul is bound by the bytes of weights read from memory.)
//
// Work: tiles of 32 weight rows; a CTA (one per SM) owns a contiguous, balanced range of them.
// A tile streams in chunks of CG = 32, 16 or 8 groups (the largest whose ring fits): one TMA
// box of 64 bytes x 32 rows x CG groups that lands as [group][row][64 B], so the two rows a
// quarter-warp reads sit 64 bytes apart and its 16-byte loads cover all 32 banks. The tile's
// S' and Z (32 x G each, contiguous in HBM) arrive by two bulk copies into a slot of their own.
// X is copied into shared memory first, when that leaves at least 64 KB of ring; otherwise it
// is read from global memory once, up front. Before it waits for the previous kernel
// (programmatic dependent launch), each CTA warms L2 with its codes past the first ring's
// worth (hints only, so safe before the wait).
//
// Warp roles:
//   producer  one lane: X, then per tile the S'/Z copies and the chunk boxes into the ring.
//   consumers 16 warps. Every warp takes every chunk and its share of the chunk's groups, so
//             each warp waits for every fill of every stage in order (the parity waits
//             cannot alias). The arithmetic is the integer warp-level MMA of imma_digits.cuh:
//             per group a warp prepares the digit fragments of X once (only that warp reads
//             them), then multiplies both 16-row halves of the tile against one load of
//             them, exactly in integers, and applies S' and the group's scale in fp32.
//   epilogue  sums the 16 warps' partials of a tile in warp order (deterministic) and writes
//             Y in bf16.
// Every wait is bounded (2 s): on a timeout the kernel records kStTimeout, the producer waits
// (bounded) for the copies it issued, and all warps return.
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "imma_digits.cuh"
#include "mma_frag.cuh"
#include "ptx.cuh"
#include "tma_host.h"

namespace wq {
namespace {

constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kNW = 16;                          // consumer warps
constexpr int kTR = 32;                          // weight rows per tile
constexpr int kMaxCG = 32;                       // groups per chunk, at most (64 KB)
constexpr int kPartSlots = 2;                    // tiles between consumers and epilogue
constexpr int kMaxStages = 8;
constexpr int kThreads = 32 * (kNW + 2);
constexpr uint32_t kSmemBudget = 227 * 1024;     // one CTA per SM
constexpr uint64_t kPrefetchBudget = 48ull << 20;  // L2 warm-up per launch, all CTAs
constexpr uint32_t kSlack = 128;                 // aligning the dynamic base

__host__ __device__ constexpr uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Shared-memory layout (byte offsets from a 128-aligned base; host and device agree).
struct TmaLayout {
  uint32_t xraw, frag, xs, xp, xf, xsp, sx, sz, sz_slot, part, part_slot, ring, bar, total;
  __host__ __device__ TmaLayout(int M, int G, int NS, int CG, bool kInt, bool x_staged,
                                int sz_slots) {
    const uint32_t MR = M < 2 ? 2 : M;
    const uint32_t NB = (4 * M + 7) / 8, FC = M == 1 ? 3 : 8;
    uint32_t end;
    xraw = xf = xsp = sx = frag = xs = xp = 0;
    if (kInt) {
      xraw = 0;                                      // [M][K] bf16: X as copied (if staged)
      frag = xraw + (x_staged ? M * G * 256u : 0u);  // [G][NB * FC * 128] digit fragments
      xs = align_up(frag + G * NB * FC * 128, 16);   // [G][NB * 8] f32 column sums
      xp = xs + G * NB * 32u;                        // [G][M] f32 scales 2^-s
      end = xp + G * M * 4u;
    } else {
      xf = 0;                                  // [M][G][4][16] u32 X fragments (bf16 MMA)
      xsp = xf + G * 4u * M * 64;              // [M][G][4] f32 partial sums of x
      sx = xsp + G * 4u * M * 4;               // [G][8] f32 sums of x per token
      end = sx + G * 32u;
    }
    sz = align_up(end, 128);
    sz_slot = align_up(128u * G, 128);       // S' [32][G] u16, then Z [32][G] u16
    part = sz + sz_slots * sz_slot;
    part_slot = kNW * kTR * MR * 4;          // [16 warps][32 rows][MR] f32
    ring = align_up(part + kPartSlots * part_slot, 128);
    bar = ring + NS * (kTR * 64u * CG);
    total = bar + (2u * NS + 2u * sz_slots + 2u * kPartSlots + 1u) * 8;
  }
};

template <int M, bool kInt>
__global__ void __launch_bounds__(kThreads, 1)
gemv_tma(const __grid_constant__ CUtensorMap tmW, const uint16_t* __restrict__ X, int64_t ldx,
         const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K, int NS,
         int CG, int x_staged, int sz_slots, int prefetch_tiles, uint16_t* __restrict__ Y,
         int64_t ldy, unsigned* status) {
  constexpr int MR = M < 2 ? 2 : M;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  const uint32_t base_s = smem_u32(smem);
  const int G = K / 128;
  const int NCH = (G + CG - 1) / CG;
  const uint32_t stage = kTR * 64u * CG;  // bytes of one chunk
  const TmaLayout L(M, G, NS, CG, kInt, x_staged != 0, sz_slots);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + NS;
  uint64_t* szfull = empty + NS;
  uint64_t* szempty = szfull + sz_slots;
  uint64_t* tdone = szempty + sz_slots;
  uint64_t* pempty = tdone + kPartSlots;
  uint64_t* xfull = pempty + kPartSlots;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = N / kTR;
  const int t_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * ntiles / gridDim.x);
  const int t_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * ntiles / gridDim.x);
  const int my_tiles = t_end - t_begin;
  const uint32_t szbytes = 64u * G;  // one of S', Z for a tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kNW);
    }
    for (int i = 0; i < sz_slots; ++i) {
      mbar_init(&szfull[i], 1);
      mbar_init(&szempty[i], kNW);
    }
    for (int i = 0; i < kPartSlots; ++i) {
      mbar_init(&tdone[i], kNW);
      mbar_init(&pempty[i], 1);
    }
    mbar_init(xfull, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) pdl_launch_dependents();
  if (warp == kNW && lane == 0) {
    // warm L2 with this CTA's codes past the first NS chunks (hints only): those reads then
    // run at the full HBM rate ahead of the ring, while the chunks the ring fetches at once
    // keep the bandwidth to themselves (warming those too measured slower)
    prefetch_tensormap(&tmW);
    const int nchunks = (t_end - t_begin) * NCH;
    for (int c = NS; c < nchunks && c < prefetch_tiles * NCH; ++c)
      tma_prefetch_3d(&tmW, 0, (t_begin + c / NCH) * kTR, (c % NCH) * CG);
  }
  pdl_wait();

  if (warp == kNW) {  // ---------------------------------------------------------- producer
    if (lane != 0) return;
    if (!kInt || x_staged) {  // X first, so that it lands ahead of the weights
      mbar_arrive_expect_tx(xfull, static_cast<uint32_t>(M) * K * 2);
      for (int n = 0; n < M; ++n)
        bulk_g2s(smem + L.xraw + static_cast<uint32_t>(n) * K * 2, X + n * ldx, K * 2u, xfull);
    }
    int i = 0, tl = 0;
    bool ok = true;
    for (; tl < my_tiles && ok; ++tl) {
      const int tile = t_begin + tl, ss = tl % sz_slots;
      if (tl >= sz_slots &&
          !mbar_wait_spin_bounded(&szempty[ss], ((tl / sz_slots) - 1) & 1u, kWaitNs)) {
        set_status(status, kStTimeout);
        break;
      }
      uint8_t* sd = smem + L.sz + ss * L.sz_slot;
      mbar_arrive_expect_tx(&szfull[ss], 2u * szbytes);
      bulk_g2s(sd, S + static_cast<int64_t>(tile) * kTR * G, szbytes, &szfull[ss]);
      bulk_g2s(sd + szbytes, Zp + static_cast<int64_t>(tile) * kTR * G, szbytes, &szfull[ss]);
      for (int ch = 0; ch < NCH; ++ch, ++i) {
        const int st = i % NS;
        const uint32_t use = i / NS;
        if (use > 0 && !mbar_wait_spin_bounded(&empty[st], (use - 1) & 1u, kWaitNs)) {
          set_status(status, kStTimeout);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[st], stage);
        tma_load_3d(smem + L.ring + st * stage, &tmW, 0, tile * kTR, ch * CG, &full[st]);
      }
    }
    // never leave the CTA with copies in flight
    for (int st = 0; st < NS && st < i; ++st)
      if (!mbar_wait_spin_bounded(&full[st], ((i - 1 - st) / NS) & 1u, kWaitNs))
        set_status(status, kStTimeout);
    for (int ss = 0; ss < sz_slots && ss < tl; ++ss)
      if (!mbar_wait_spin_bounded(&szfull[ss], ((tl - 1 - ss) / sz_slots) & 1u, kWaitNs))
        set_status(status, kStTimeout);
    if ((!kInt || x_staged) && !mbar_wait_spin_bounded(xfull, 0, kWaitNs))
      set_status(status, kStTimeout);
    return;
  }

  if (warp == kNW + 1) {  // ------------------------------------------------------ epilogue
    for (int tl = 0; tl < my_tiles; ++tl) {
      const int ps = tl % kPartSlots;
      if (!mbar_wait_spin_bounded(&tdone[ps], (tl / kPartSlots) & 1u, kWaitNs)) {
        set_status(status, kStTimeout);
        return;
      }
      const float* part = reinterpret_cast<const float*>(smem + L.part + ps * L.part_slot);
      const int tile = t_begin + tl;
      for (int e = lane; e < kTR * M; e += 32) {
        const int row = e / M, tok = e - (e / M) * M;
        float t = 0.0f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) t += part[(w * kTR + row) * MR + tok];
        __nv_bfloat16 hv = __float2bfloat16_rn(t);
        Y[tok * ldy + tile * kTR + row] = *reinterpret_cast<uint16_t*>(&hv);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pempty[ps]);
    }
    return;
  }

  if constexpr (kInt) {
  // ---------------------------------------------------------------------- consumer warps
  // Warp w takes, of every chunk, the groups [qa, qb) of its even share. Before the first
  // tile's chunk ch is consumed it turns the X of its groups of chunk ch + 1 into digit
  // fragments (imma_digits.cuh; only this warp reads them), so that work overlaps the wait.
  using C = Cols<M>;
  constexpr int NB = C::NB, FC = C::FC;
  auto share = [&](int ch, int& ga, int& gb) {  // this warp's groups of chunk ch
    const int g0 = ch * CG, gn = min(CG, G - g0);
    ga = g0 + (warp * gn) / kNW;
    gb = g0 + ((warp + 1) * gn) / kNW;
  };
  auto prep_one = [&](int gi, const uint2 (&xv)[M]) {
    prep_group<M>(smem + L.frag + gi * C::kFragBytes,
                  reinterpret_cast<float*>(smem + L.xs) + gi * NB * 8,
                  reinterpret_cast<float*>(smem + L.xp) + gi * M, xv, lane);
  };
  auto prep_chunk = [&](int ch) {  // from the staged copy of X
    int ga, gb;
    share(ch, ga, gb);
    for (int gi = ga; gi < gb; ++gi) {
      uint2 xv[M];
#pragma unroll
      for (int m = 0; m < M; ++m)
        xv[m] = *reinterpret_cast<const uint2*>(smem + L.xraw + (m * G + gi) * 256 + 8 * lane);
      prep_one(gi, xv);
    }
    __syncwarp();
  };
  if (x_staged) {
    if (!mbar_wait_spin_bounded(xfull, 0, kWaitNs)) {
      set_status(status, kStTimeout);
      return;
    }
    prep_chunk(0);
  } else {
    // X from global memory, all of this warp's groups at once: the loads of a batch are all
    // issued before any is used, so their latency is paid once per batch
    constexpr int BG = 16 / M;
    int gl[BG];
    int n = 0;
    auto flush = [&]() {
      uint2 xv[BG][M];
#pragma unroll
      for (int u = 0; u < BG; ++u)
#pragma unroll
        for (int m = 0; m < M; ++m)
          xv[u][m] = u < n ? *reinterpret_cast<const uint2*>(X + m * ldx + gl[u] * 128 + 4 * lane)
                           : make_uint2(0u, 0u);
#pragma unroll
      for (int u = 0; u < BG; ++u)
        if (u < n) prep_one(gl[u], xv[u]);
      n = 0;
    };
    for (int ch = 0; ch < NCH; ++ch) {
      int ga, gb;
      share(ch, ga, gb);
      for (int gi = ga; gi < gb; ++gi) {
        gl[n++] = gi;
        if (n == BG) flush();
      }
    }
    if (n > 0) flush();
    __syncwarp();
  }
  const float* xs_all = reinterpret_cast<const float*>(smem + L.xs);
  const float* xp_all = reinterpret_cast<const float*>(smem + L.xp);
  const int r = lane >> 2, c = lane & 3;
  const float w0 = (c & 1) ? 65536.0f : 1.0f, w1 = (c & 1) ? 16777216.0f : 256.0f;
  const bool bcol = r < FC;  // this lane's B column is stored (else its digits are zero)
  const uint32_t ring_lane = base_s + L.ring + r * 64 + 16 * c;
  uint32_t mask4 = 0x0F0F0F0Fu;
  asm volatile("" : "+r"(mask4));
  int i = 0;
  for (int tl = 0; tl < my_tiles; ++tl) {
    const int ss = tl % sz_slots, ps = tl % kPartSlots;
    const uint32_t sb = base_s + L.sz + ss * L.sz_slot, zb = sb + szbytes;
    float acc[2][NB][2];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) acc[t][nb][0] = acc[t][nb][1] = 0.0f;
    for (int ch = 0; ch < NCH; ++ch, ++i) {
      const int st = i % NS;
      if (x_staged && tl == 0 && ch + 1 < NCH) prep_chunk(ch + 1);
      bool ok = mbar_wait_spin_bounded(&full[st], (i / NS) & 1u, kWaitNs);
      if (ok && ch == 0) ok = mbar_wait_spin_bounded(&szfull[ss], (tl / sz_slots) & 1u, kWaitNs);
      if (!ok) {
        set_status(status, kStTimeout);
        return;
      }
      const uint32_t wst = ring_lane + st * stage;
      int ga, gb;
      share(ch, ga, gb);
      for (int g = ga; g < gb; ++g) {
        const int q = g - ch * CG;
        const uint32_t frag_s = base_s + L.frag + g * C::kFragBytes;
        uint32_t bw[NB][8];
        float2 xsum[NB];
        float p[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const uint32_t blk = frag_s + nb * FC * 128 + (r * 4 + c) * 16;
          uint4 b01 = make_uint4(0u, 0u, 0u, 0u), b23 = b01;
          if (bcol) {
            b01 = lds128(blk);
            b23 = lds128(blk + FC * 64);
          }
          bw[nb][0] = b01.x; bw[nb][1] = b01.y; bw[nb][2] = b01.z; bw[nb][3] = b01.w;
          bw[nb][4] = b23.x; bw[nb][5] = b23.y; bw[nb][6] = b23.z; bw[nb][7] = b23.w;
          xsum[nb] = *reinterpret_cast<const float2*>(xs_all + g * NB * 8 + nb * 8 + 2 * c);
          const int m = 2 * nb + (c >> 1);
          p[nb] = m < M ? xp_all[g * M + (m < M ? m : 0)] : 0.0f;
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint32_t wa = wst + q * (kTR * 64) + t * (16 * 64);
          const uint4 ca = lds128(wa);
          const uint4 cb = lds128(wa + 8 * 64);
          const int ra = 16 * t + r, rb = ra + 8;
          const float sa = f16_bits_to_f32(lds16(sb + (ra * G + g) * 2));
          const float za = f16_bits_to_f32(lds16(zb + (ra * G + g) * 2));
          const float sbv = f16_bits_to_f32(lds16(sb + (rb * G + g) * 2));
          const float zbv = f16_bits_to_f32(lds16(zb + (rb * G + g) * 2));
          const uint32_t wr0[4] = {ca.x, ca.y, ca.z, ca.w};
          const uint32_t wr1[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            // accumulators start at the magic so that each reads back as 1.5 * 2^23 + D
            int d[4] = {kImmaMagicBits, kImmaMagicBits, kImmaMagicBits, kImmaMagicBits};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const uint32_t a[4] = {wr0[w] & mask4, wr1[w] & mask4, (wr0[w] >> 4) & mask4,
                                     (wr1[w] >> 4) & mask4};
              imma_16832(d, a, bw[nb][2 * w], bw[nb][2 * w + 1]);
            }
            // D_i - Z X_i, exactly (both sides carry the same magic offset)
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
    }
    if (lane == 0) mbar_arrive(&szempty[ss]);
    if (tl >= kPartSlots &&
        !mbar_wait_spin_bounded(&pempty[ps], ((tl / kPartSlots) - 1) & 1u, kWaitNs)) {
      set_status(status, kStTimeout);
      return;
    }
    float* part = reinterpret_cast<float*>(smem + L.part + ps * L.part_slot) + warp * kTR * MR;
    if ((c & 1) == 0) {
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const int m = 2 * nb + (c >> 1);
          if (m < M) {
            part[(16 * t + r) * MR + m] = acc[t][nb][0];
            part[(16 * t + r + 8) * MR + m] = acc[t][nb][1];
          }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tdone[ps]);
  }
  } else {
  // ---------------------------------------------------------------------- consumer warps
  // X (landed in natural order) -> fragment order in place, 64 bytes (32 values of one
  // token, one quarter c of a group) per thread, and per-group token sums, each formed from
  // four partial sums of 32 values in a fixed order. The four 16-byte chunks of quarter c
  // land rotated by 2 (c >> 1), so that the four quarters a warp reads at once (64 bytes
  // apart) fall on different banks.
  float* xsp = reinterpret_cast<float*>(smem + L.xsp);
  float* sxs = reinterpret_cast<float*>(smem + L.sx);
  if (!mbar_wait_spin_bounded(xfull, 0, kWaitNs)) {
    set_status(status, kStTimeout);
    return;
  }
  for (int e = threadIdx.x; e < M * G * 4; e += 32 * kNW) {  // e = (n * G + g) * 4 + c
    const uint32_t blk = base_s + L.xf + e * 64;
    const int xrot = 2 * ((e >> 1) & 1);
    uint32_t xw[16];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = lds128(blk + 16 * v);
      xw[4 * v] = u.x; xw[4 * v + 1] = u.y; xw[4 * v + 2] = u.z; xw[4 * v + 3] = u.w;
    }
    uint32_t frag[16];
    build_x_fragment(xw, frag);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      sts128(blk + 16 * ((j + xrot) & 3),
             make_uint4(frag[4 * j], frag[4 * j + 1], frag[4 * j + 2], frag[4 * j + 3]));
    float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int v = 0; v < 16; ++v) ps[v & 3] += bf16_lo(xw[v]) + bf16_hi(xw[v]);
    xsp[e] = (ps[0] + ps[1]) + (ps[2] + ps[3]);
  }
  named_barrier(1, 32 * kNW);
  for (int e = threadIdx.x; e < G * 8; e += 32 * kNW) {
    const int g = e >> 3, n = e & 7;
    float t = 0.0f;
    if (n < M) {
      const float* q = xsp + (n * G + g) * 4;
      t = (q[0] + q[1]) + (q[2] + q[3]);
    }
    sxs[e] = t;
  }
  named_barrier(1, 32 * kNW);

  const int r = lane >> 2, c = lane & 3;
  const int t0 = 2 * c, t1 = 2 * c + 1;
  // lanes whose token column is >= M read a duplicate fragment: their columns are never
  // stored, and the loads stay uniform
  const int xn = (lane >> 2) % M;
  const uint32_t xf_lane = base_s + L.xf + xn * (G * 256) + c * 64;
  // this lane's X fragment chunks 0, 1 sit at xlo, xlo + 16 and chunks 2, 3 at xhi, xhi + 16
  const uint32_t xlo = 32u * (c >> 1), xhi = 32u - xlo;
  const uint32_t ring_lane = base_s + L.ring + r * 64 + 16 * c;
  uint32_t kMask = 0x00780078u, kMagic = 0x3F803F80u;  // register operands of the LOP3
  asm volatile("" : "+r"(kMask), "+r"(kMagic));
  int i = 0;
  for (int tl = 0; tl < my_tiles; ++tl) {
    const int ss = tl % sz_slots, ps = tl % kPartSlots;
    const uint32_t sb = base_s + L.sz + ss * L.sz_slot, zb = sb + szbytes;
    float acc[2][4] = {};
    for (int ch = 0; ch < NCH; ++ch, ++i) {
      const int st = i % NS;
      bool ok = mbar_wait_spin_bounded(&full[st], (i / NS) & 1u, kWaitNs);
      if (ok && ch == 0) ok = mbar_wait_spin_bounded(&szfull[ss], (tl / sz_slots) & 1u, kWaitNs);
      if (!ok) {
        set_status(status, kStTimeout);
        return;
      }
      const uint32_t wst = ring_lane + st * stage;
      const int g0 = ch * CG;
      const int gn = min(CG, G - g0);
      const int qa = (warp * gn) / kNW, qb = ((warp + 1) * gn) / kNW;
      for (int q = qa; q < qb; ++q) {
        const int g = g0 + q;
        const uint32_t xs = xf_lane + g * 256;
        const uint4 xb0 = lds128(xs + xlo), xb1 = lds128(xs + xlo + 16),
                    xb2 = lds128(xs + xhi), xb3 = lds128(xs + xhi + 16);
        const uint32_t bw[16] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w,
                                 xb2.x, xb2.y, xb2.z, xb2.w, xb3.x, xb3.y, xb3.z, xb3.w};
        const float sx0 = sxs[g * 8 + t0];
        [[maybe_unused]] const float sx1 = M > 1 ? sxs[g * 8 + t1] : 0.0f;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint32_t wa = wst + q * (kTR * 64) + t * (16 * 64);
          const uint4 ca = lds128(wa);
          const uint4 cb = lds128(wa + 8 * 64);
          const uint32_t wr0[4] = {ca.x, ca.y, ca.z, ca.w};
          const uint32_t wr1[4] = {cb.x, cb.y, cb.z, cb.w};
          float d[4][4] = {};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t pa[4], pb[4];
            unpack_bf16_hi(wr0[w], kMask, kMagic, pa);
            unpack_bf16_hi(wr1[w], kMask, kMagic, pb);
            const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
            const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
            mma_bf16_16816(d[(w & 1) * 2], a0, bw[4 * w], bw[4 * w + 1]);
            mma_bf16_16816(d[(w & 1) * 2 + 1], a1, bw[4 * w + 2], bw[4 * w + 3]);
          }
          const int ra = 16 * t + r, rb = ra + 8;
          const float s0 = f16_bits_to_f32(lds16(sb + (ra * G + g) * 2));
          const float z0 = f16_bits_to_f32(lds16(zb + (ra * G + g) * 2));
          const float s1 = f16_bits_to_f32(lds16(sb + (rb * G + g) * 2));
          const float z1 = f16_bits_to_f32(lds16(zb + (rb * G + g) * 2));
          const float e0 = (d[0][0] + d[2][0]) + (d[1][0] + d[3][0]);
          const float e2 = (d[0][2] + d[2][2]) + (d[1][2] + d[3][2]);
          acc[t][0] = fmaf(s0, fmaf(16.0f, e0, -(16.0f + z0) * sx0), acc[t][0]);
          acc[t][2] = fmaf(s1, fmaf(16.0f, e2, -(16.0f + z1) * sx0), acc[t][2]);
          if constexpr (M > 1) {
            const float e1 = (d[0][1] + d[2][1]) + (d[1][1] + d[3][1]);
            const float e3 = (d[0][3] + d[2][3]) + (d[1][3] + d[3][3]);
            acc[t][1] = fmaf(s0, fmaf(16.0f, e1, -(16.0f + z0) * sx1), acc[t][1]);
            acc[t][3] = fmaf(s1, fmaf(16.0f, e3, -(16.0f + z1) * sx1), acc[t][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (lane == 0) mbar_arrive(&szempty[ss]);
    if (tl >= kPartSlots &&
        !mbar_wait_spin_bounded(&pempty[ps], ((tl / kPartSlots) - 1) & 1u, kWaitNs)) {
      set_status(status, kStTimeout);
      return;
    }
    float* part = reinterpret_cast<float*>(smem + L.part + ps * L.part_slot) + warp * kTR * MR;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int ra = 16 * t + r, rb = ra + 8;
      if (t0 < M) {
        part[ra * MR + t0] = acc[t][0];
        part[rb * MR + t0] = acc[t][2];
      }
      if constexpr (M > 1) {
        if (t1 < M) {
          part[ra * MR + t1] = acc[t][1];
          part[rb * MR + t1] = acc[t][3];
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tdone[ps]);
  }
  }
}

// Chunk size (groups) and ring depth for this shape: the largest chunk of 32, 16 or 8 groups
// whose ring has at least two stages in shared memory; NS = 0 if none fits.
struct TmaCfg {
  int CG, NS;
  bool x_staged;
  int sz_slots;
};
// Chunk size, ring depth, X staging and S'/Z slots for this shape. The bf16 path takes the
// largest chunk whose ring has two stages. The integer path also stages X in shared memory
// (when that leaves at least 64 KB of ring; otherwise X is read once from global memory) and
// falls back to one S'/Z slot when two leave no ring.
TmaCfg tma_config(int M, int G, bool kInt) {
  for (int slots : {2, 1}) {
    for (bool xs : {true, false}) {
      if (!kInt && !xs) continue;
      const uint32_t fixed = TmaLayout(M, G, 0, 8, kInt, xs, slots).total + kSlack;
      for (int cg : {kMaxCG, 16, 8}) {
        if (fixed > kSmemBudget) break;
        int ns = static_cast<int>((kSmemBudget - fixed) / (kTR * 64u * cg + 16));
        if (ns > kMaxStages) ns = kMaxStages;
        if (ns >= 2 && (!kInt || !xs || ns * kTR * 64u * cg >= 64u * 1024))
          return {cg, ns, xs, slots};
      }
    }
    if (!kInt) break;
  }
  return {8, 0, false, 2};
}

// The integer MMA for one token while K <= 16384 (G <= 128 groups); beyond that, and for
// two to four tokens, the digit fragments (3 bytes per k and token, besides the staged X)
// leave too small a ring and the bf16 MMA, whose X fragments take 2 bytes per k, is faster.
constexpr int kIntMaxG = 128;

template <int M, bool kInt>
cudaError_t launch_tma_k(const GemvArgs& a, int sms, cudaStream_t st) {
  const int G = a.K / 128;
  const int ntiles = a.N / kTR;
  if (ntiles == 0) return cudaSuccess;
  const TmaCfg c = tma_config(M, G, kInt);
  if (c.NS == 0) return cudaErrorInvalidValue;
  // codes as [G groups][N rows][64 bytes]: boxes of CG groups x 32 rows x 64 bytes. The
  // encoded map is kept per thread for the last few weight matrices (decode calls repeat).
  struct MapEntry {
    const void* p;
    int n, k, cg;
    CUtensorMap map;
  };
  constexpr int kMapCache = 16;
  thread_local MapEntry cache[kMapCache];
  thread_local int next_slot = 0;
  const CUtensorMap* map = nullptr;
  for (const MapEntry& e : cache)
    if (e.p == a.P && e.n == a.N && e.k == a.K && e.cg == c.CG) map = &e.map;
  if (!map) {
    MapEntry& e = cache[next_slot];
    const uint64_t dims[3] = {64, static_cast<uint64_t>(a.N), static_cast<uint64_t>(G)};
    const uint64_t strides[2] = {static_cast<uint64_t>(a.K / 2), 64};
    const uint32_t box[3] = {64, kTR, static_cast<uint32_t>(c.CG)};
    e.p = nullptr;
    if (!make_map_3d(&e.map, a.P, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8))
      return cudaErrorInvalidValue;
    e.p = a.P;
    e.n = a.N;
    e.k = a.K;
    e.cg = c.CG;
    next_slot = (next_slot + 1) % kMapCache;
    map = &e.map;
  }
  const size_t smem =
      TmaLayout(M, G, c.NS, c.CG, kInt, c.x_staged, c.sz_slots).total + kSlack;
  auto kern = gemv_tma<M, kInt>;
  static std::atomic<bool> attr[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 63].load(std::memory_order_acquire)) {
    const cudaError_t e = set_smem_attrs(kern, static_cast<int>(kSmemBudget));
    if (e != cudaSuccess) return e;
    attr[dev & 63].store(true, std::memory_order_release);
  }
  const int grid = ntiles < sms ? ntiles : sms;
  const uint64_t tile_bytes = static_cast<uint64_t>(kTR) * (a.K / 2 + 4 * G);
  const int prefetch_tiles = static_cast<int>(kPrefetchBudget / grid / tile_bytes);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, *map, a.X, a.ldx, a.S, a.Z, a.N, a.K, c.NS, c.CG,
                            c.x_staged ? 1 : 0, c.sz_slots, prefetch_tiles, a.Y, a.ldy,
                            a.status);
}

template <int M>
cudaError_t launch_tma_m(const GemvArgs& a, int sms, cudaStream_t st) {
  if (M == 1 && a.K / 128 <= kIntMaxG) return launch_tma_k<M, true>(a, sms, st);
  return launch_tma_k<M, false>(a, sms, st);
}

}  // namespace

bool gemv_tma_ok(const GemvArgs& a) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return a.M >= 1 && a.M <= 4 && a.K % 128 == 0 && a.group == 128 && a.sz_row == a.K / 128 &&
         a.N % kTR == 0 && (a.ldx % 8) == 0 && al16(a.X) && al16(a.P) && al16(a.S) &&
         al16(a.Z) &&
         tma_config(a.M, a.K / 128, a.M == 1 && a.K / 128 <= kIntMaxG).NS > 0;
}

cudaError_t launch_gemv_tma(const GemvArgs& a, int sms, cudaStream_t st) {
  switch (a.M) {
    case 1: return launch_tma_m<1>(a, sms, st);
    case 2: return launch_tma_m<2>(a, sms, st);
    case 3: return launch_tma_m<3>(a, sms, st);
    case 4: return launch_tma_m<4>(a, sms, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wq
