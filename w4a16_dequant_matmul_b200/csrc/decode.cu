// Small-M W4A16 matmul (decode), Y = X W_hat^T for M <= 4 tokens, group size 128.
// ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
// "The vocabulary" and the decode discussion: 4-bit weights dequantized inside the kernel;
// at decode the matmul is bound by the bytes of weights read from memory.)
//
// Work: tiles of 16 weight rows; a CTA owns a contiguous range of tiles, the same number
// for every CTA (the grid is sized so). Each tile's rows are streamed whole (up to 3 KB per
// row, K <= 6144; longer rows go to the K-chunked TMA kernel): on B200 the bulk-copy engine
// keeps about 32 copies in flight per SM, so copies this large are what fills HBM.
//
// Warp roles (one CTA per SM):
//   producer  one lane. X (one bulk copy per token), then per chunk: 16 row copies into a
//             ring stage whose rows are padded to a pitch of 64 mod 128 bytes, so the MMA
//             warps' 16-byte reads of two adjacent rows fall on all 32 banks. It never
//             waits for S'/Z, so the weight stream runs ahead on its own.
//   prep      keeps S' and Z of the next RS tiles in flight (two contiguous bulk copies
//             per tile, into its own ring) and transposes each landed tile into
//             [group][row pair](s_r, z_r, s_r+8, z_r+8): one 8-byte shared load per group
//             for a consumer lane.
//   consumers 8 warps. Every warp takes every chunk and a fixed share of its groups, so each
//             warp consumes each stage's fills in order (parity waits cannot alias). Codes
//             are decoded to bf16 (1 + q/16, one shift and one 3-input logic op per two
//             codes) and multiplied with eight m16n8k16 MMAs per group (four independent
//             accumulator chains) against X fragments in shared memory (X arrives by one
//             bulk copy per token and is permuted into fragment order in place); per group,
//             with D = sum x (1 + q/16) and sum x precomputed,
//               acc += S' (16 D - (16 + Z) sum x).
//             At the end of a tile each warp writes its 16 x M partial sums.
//   epilogue  sums the 8 partials of a tile in warp order (deterministic), writes Y in
//             bf16 and frees the tile's slots.
//
// Programmatic dependent launch: the kernel lets the next launch on the stream start at
// once (its CTAs take SMs as this kernel's CTAs leave) and reads nothing (X, codes, S', Z)
// before it has waited for the previous kernel.
//
// Every wait is bounded (2 s): on a timeout the kernel records kStTimeout, the producer
// waits (bounded) for the copies it issued to land, and all warps return.
#include <type_traits>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "mma_frag.cuh"
#include "ptx.cuh"

namespace wq {
namespace {

constexpr uint64_t kDecWaitNs = 2000000000ull;
constexpr int kDecWarps = 8;    // consumer warps
constexpr int kRawSlotsMax = 4; // raw S'/Z tiles in flight (fewer if shared memory is short)
constexpr int kTileSlots = 4;   // tiles in flight past the S'/Z transpose
// Tiles multiplied together per group by a consumer warp (1 or 2). Two share the X
// fragment reads but make a warp wait for two stages; one measured faster on B200.
constexpr int kPairTiles = 1;
constexpr int kMaxStages = 16;
constexpr uint32_t kSmemBudget = 227 * 1024;
constexpr int kChunkMax = 3072;  // bytes of a row per chunk, at most

__host__ __device__ constexpr uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Shared-memory layout (byte offsets from a 128-aligned base; host and device agree).
struct DecodeLayout {
  uint32_t xf, xsp, sx, raw, raw_slot, prep, prep_slot, part, part_slot, ring, stage, bar, total;
  __host__ __device__ DecodeLayout(int M, int G, int pitch, int NS, int RS) {
    const uint32_t MR = M < 2 ? 2 : M;
    xf = 0;                                   // [M][G][4][16] u32 X fragments
    xsp = xf + G * 4u * M * 64;               // [G][4M] f32 partial sums of x
    sx = xsp + G * 4u * M * 4;                // [G][8] f32 sums of x per token
    raw = align_up(sx + G * 32u, 128);
    raw_slot = 64u * G;                       // S' [16][G] u16, then Z [16][G] u16
    prep = raw + RS * raw_slot;
    prep_slot = 64u * G;                      // [G][8](s_r, z_r, s_r+8, z_r+8) u16
    part = prep + kTileSlots * prep_slot;
    part_slot = kDecWarps * 16u * MR * 4;     // [8 warps][16 rows][MR] f32
    ring = align_up(part + kTileSlots * part_slot, 128);
    stage = 16u * pitch;
    bar = ring + NS * stage;
    total = bar + (2u * NS + RS + 3u * kTileSlots + 1u) * 8;
  }
};

template <int M>
__global__ void __launch_bounds__(32 * (kDecWarps + 3), 1)
gemv_decode(const uint16_t* __restrict__ X, int64_t ldx, const uint8_t* __restrict__ P,
            const uint16_t* __restrict__ S, const uint16_t* __restrict__ Zp, int N, int K,
            int CK, int NCH, int pitch, int NS, int RS, int tpc, uint16_t* __restrict__ Y,
            int64_t ldy, unsigned* status) {
  constexpr int NW = kDecWarps;
  constexpr int MR = M < 2 ? 2 : M;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  const uint32_t base_s = smem_u32(smem);
  const int G = K / 128;
  const uint32_t row_bytes = K / 2;
  const DecodeLayout L(M, G, pitch, NS, RS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + NS;
  uint64_t* rawfull = empty + NS;
  uint64_t* prepfull = rawfull + RS;
  uint64_t* prepempty = prepfull + kTileSlots;
  uint64_t* tdone = prepempty + kTileSlots;
  uint64_t* xfull = tdone + kTileSlots;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = N / 16;
  const int t_begin = blockIdx.x * tpc;
  const int my_tiles = min(ntiles, t_begin + tpc) - t_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    for (int i = 0; i < RS; ++i) mbar_init(&rawfull[i], 1);
    for (int i = 0; i < kTileSlots; ++i) {
      mbar_init(&prepfull[i], 1);
      mbar_init(&prepempty[i], 1);
      mbar_init(&tdone[i], NW);
    }
    mbar_init(xfull, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();

  if (warp == NW) {  // ---------------------------------------------------------- producer
    if (lane != 0) return;
    // X first: row n of X lands at fragment block n (in natural order; the consumers
    // permute it in place)
    mbar_arrive_expect_tx(xfull, static_cast<uint32_t>(M) * K * 2);
    for (int n = 0; n < M; ++n)
      bulk_g2s(smem + L.xf + static_cast<uint32_t>(n) * K * 2, X + n * ldx, K * 2u, xfull);
    // Tiles go in pairs (the consumers multiply two 16-row tiles per group); a pair's
    // chunks are issued chunk by chunk, (tile, chunk) then (tile + 1, chunk).
    int i = 0;  // chunk fills issued
    bool ok = true;
    for (int tp = 0; tp < my_tiles && ok; tp += kPairTiles) {
      const int nt = min(kPairTiles, my_tiles - tp);
      for (int ch = 0; ch < NCH && ok; ++ch) {
        for (int u = 0; u < nt; ++u) {
          const int st = i % NS;
          const uint32_t use = i / NS;
          if (use > 0 && !mbar_wait_spin_bounded(&empty[st], (use - 1) & 1u, kDecWaitNs)) {
            set_status(status, kStTimeout);
            ok = false;
            break;
          }
          const uint8_t* src = P + static_cast<int64_t>(t_begin + tp + u) * 16 * row_bytes;
          const uint32_t off = static_cast<uint32_t>(ch) * CK;
          const uint32_t bytes = min(static_cast<uint32_t>(CK), row_bytes - off);
          uint8_t* dst = smem + L.ring + st * L.stage;
          mbar_arrive_expect_tx(&full[st], 16u * bytes);
          for (int r = 0; r < 16; ++r)
            bulk_g2s(dst + r * pitch, src + static_cast<int64_t>(r) * row_bytes + off, bytes,
                     &full[st]);
          ++i;
        }
      }
    }
    // never leave the CTA with copies in flight
    for (int st = 0; st < NS && st < i; ++st)
      if (!mbar_wait_spin_bounded(&full[st], ((i - 1 - st) / NS) & 1u, kDecWaitNs))
        set_status(status, kStTimeout);
    if (!mbar_wait_spin_bounded(xfull, 0, kDecWaitNs)) set_status(status, kStTimeout);
    return;
  }

  if (warp == NW + 1) {  // ---------------------------------------------------------- prep
    // This warp alone uses the raw S'/Z ring: it keeps the next RS tiles' copies in flight,
    // transposes tile tl when it lands and refills the slot with tile tl + RS.
    auto issue_raw = [&](int t) {
      const int tile = t_begin + t, rs = t % RS;
      uint8_t* rd = smem + L.raw + rs * L.raw_slot;
      mbar_arrive_expect_tx(&rawfull[rs], L.raw_slot);
      bulk_g2s(rd, S + static_cast<int64_t>(tile) * 16 * G, 32u * G, &rawfull[rs]);
      bulk_g2s(rd + 32u * G, Zp + static_cast<int64_t>(tile) * 16 * G, 32u * G, &rawfull[rs]);
    };
    const int first = RS < my_tiles ? RS : my_tiles;
    if (lane == 0)
      for (int t = 0; t < first; ++t) issue_raw(t);
    int issued = first, tl = 0;
    for (; tl < my_tiles; ++tl) {
      const int rs = tl % RS, ps = tl % kTileSlots;
      if (!mbar_wait_spin_bounded(&rawfull[rs], (tl / RS) & 1u, kDecWaitNs) ||
          (tl >= kTileSlots &&
           !mbar_wait_spin_bounded(&prepempty[ps], ((tl / kTileSlots) - 1) & 1u, kDecWaitNs))) {
        set_status(status, kStTimeout);
        break;
      }
      const uint16_t* rsv = reinterpret_cast<const uint16_t*>(smem + L.raw + rs * L.raw_slot);
      const uint16_t* rzv = rsv + 16 * G;
      uint2* pv = reinterpret_cast<uint2*>(smem + L.prep + ps * L.prep_slot);
      for (int e = lane; e < 8 * G; e += 32) {
        const int g = e >> 3, r = e & 7;
        const uint32_t a = static_cast<uint32_t>(rsv[r * G + g]) |
                           (static_cast<uint32_t>(rzv[r * G + g]) << 16);
        const uint32_t b = static_cast<uint32_t>(rsv[(r + 8) * G + g]) |
                           (static_cast<uint32_t>(rzv[(r + 8) * G + g]) << 16);
        pv[e] = make_uint2(a, b);
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&prepfull[ps]);
        if (issued < my_tiles) {
          fence_proxy_async_smem();  // the slot's reads above precede the copy's writes
          issue_raw(issued);
        }
      }
      if (issued < my_tiles) ++issued;
    }
    // on a timeout, wait (bounded) for the copies still in flight
    if (lane == 0)
      for (int t = tl; t < issued; ++t)
        if (!mbar_wait_spin_bounded(&rawfull[t % RS], (t / RS) & 1u, kDecWaitNs))
          set_status(status, kStTimeout);
    return;
  }

  if (warp == NW + 2) {  // ------------------------------------------------------ epilogue
    for (int tl = 0; tl < my_tiles; ++tl) {
      const int ps = tl % kTileSlots;
      if (!mbar_wait_spin_bounded(&tdone[ps], (tl / kTileSlots) & 1u, kDecWaitNs)) {
        set_status(status, kStTimeout);
        return;
      }
      const float* part = reinterpret_cast<const float*>(smem + L.part + ps * L.part_slot);
      const int tile = t_begin + tl;
      for (int e = lane; e < 16 * M; e += 32) {
        const int row = e / M, tok = e - (e / M) * M;
        float t = 0.0f;
#pragma unroll
        for (int w = 0; w < NW; ++w) t += part[(w * 16 + row) * MR + tok];
        __nv_bfloat16 hv = __float2bfloat16_rn(t);
        Y[tok * ldy + tile * 16 + row] = *reinterpret_cast<uint16_t*>(&hv);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&prepempty[ps]);
    }
    return;
  }

  // ---------------------------------------------------------------------- consumer warps
  // X (landed in natural order) -> fragment order in place, 64 bytes (32 values of one
  // token, one quarter of a group) per thread, and per-group token sums, each formed from
  // four partial sums of 32 values in a fixed order.
  float* xsp = reinterpret_cast<float*>(smem + L.xsp);
  float* sxs = reinterpret_cast<float*>(smem + L.sx);
  if (!mbar_wait_spin_bounded(xfull, 0, kDecWaitNs)) {
    set_status(status, kStTimeout);
    return;
  }
  for (int e = threadIdx.x; e < M * G * 4; e += 32 * NW) {  // e = (n * G + g) * 4 + c
    const uint32_t blk = base_s + L.xf + e * 64;
    uint32_t xw[16];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = lds128(blk + 16 * v);
      xw[4 * v] = u.x; xw[4 * v + 1] = u.y; xw[4 * v + 2] = u.z; xw[4 * v + 3] = u.w;
    }
    uint32_t frag[16];
    build_x_fragment(xw, frag);
    // chunks of quarter c rotated by 2 (c >> 1): a warp's four quarter loads hit four bank groups
    const int xrot = 2 * ((e >> 1) & 1);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      sts128(blk + 16 * ((j + xrot) & 3),
             make_uint4(frag[4 * j], frag[4 * j + 1], frag[4 * j + 2], frag[4 * j + 3]));
    float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int v = 0; v < 16; ++v) ps[v & 3] += bf16_lo(xw[v]) + bf16_hi(xw[v]);
    xsp[e] = (ps[0] + ps[1]) + (ps[2] + ps[3]);
  }
  named_barrier(1, 32 * NW);
  for (int e = threadIdx.x; e < G * 8; e += 32 * NW) {
    const int g = e >> 3, n = e & 7;
    float t = 0.0f;
    if (n < M) {
      const float* q = xsp + (n * G + g) * 4;
      t = (q[0] + q[1]) + (q[2] + q[3]);
    }
    sxs[e] = t;
  }
  named_barrier(1, 32 * NW);

  const int r = lane >> 2, c = lane & 3;
  const int t0 = 2 * c, t1 = 2 * c + 1;
  // lanes whose token column is >= M read a duplicate fragment: their columns are never
  // stored, and the loads stay uniform
  const int xn = (lane >> 2) % M;  // token of this lane's fragment (duplicates past M)
  const uint32_t xf_lane = base_s + L.xf + xn * (G * 256) + c * 64;
  // this lane's X fragment chunks 0, 1 sit at xlo, xlo + 16 and chunks 2, 3 at xhi, xhi + 16
  const uint32_t xlo = 32u * (c >> 1), xhi = 32u - xlo;
  const uint32_t ring_lane = base_s + L.ring + r * pitch + 16 * c;
  uint32_t kMask = 0x00780078u, kMagic = 0x3F803F80u;  // register operands of the LOP3
  asm volatile("" : "+r"(kMask), "+r"(kMagic));
  const int gpc = CK / 64;  // groups per full chunk
  // One group (128 codes) of RT consecutive 16-row tiles: the X fragments are read once for
  // all of them. wst[t] / prep[t]: this lane's row in the chunk stage / S'Z slot of tile t.
  auto group = [&](auto rt, int q, int g, const uint32_t (&wst)[2], const uint32_t (&prep)[2],
                   float (&acc)[2][4]) {
    constexpr int RT = decltype(rt)::value;
    const uint32_t xs = xf_lane + g * 256;
    const uint4 xb0 = lds128(xs + xlo), xb1 = lds128(xs + xlo + 16), xb2 = lds128(xs + xhi),
                xb3 = lds128(xs + xhi + 16);
    const uint32_t bw[16] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w,
                             xb2.x, xb2.y, xb2.z, xb2.w, xb3.x, xb3.y, xb3.z, xb3.w};
    const float sx0 = sxs[g * 8 + t0];
    [[maybe_unused]] const float sx1 = M > 1 ? sxs[g * 8 + t1] : 0.0f;
#pragma unroll
    for (int t = 0; t < RT; ++t) {
      const uint4 ca = lds128(wst[t] + q * 64);
      const uint4 cb = lds128(wst[t] + q * 64 + 8 * pitch);
      const uint32_t wr0[4] = {ca.x, ca.y, ca.z, ca.w};
      const uint32_t wr1[4] = {cb.x, cb.y, cb.z, cb.w};
      // four independent accumulator chains of two MMAs each
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
      uint32_t sz0, sz1;  // (s_r, z_r), (s_r+8, z_r+8) as binary16 pairs
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(sz0), "=r"(sz1) : "r"(prep[t] + g * 64));
      const float s0 = f16_bits_to_f32(sz0 & 0xFFFFu), z0 = f16_bits_to_f32(sz0 >> 16);
      const float s1 = f16_bits_to_f32(sz1 & 0xFFFFu), z1 = f16_bits_to_f32(sz1 >> 16);
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
  };
  int i = 0;
  for (int tp = 0; tp < my_tiles; tp += kPairTiles) {
    const int nt = min(kPairTiles, my_tiles - tp);
    int ps[2];
    uint32_t prep[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      ps[u] = (tp + u) % kTileSlots;
      prep[u] = base_s + L.prep + ps[u] * L.prep_slot + r * 8;
    }
    float acc[2][4] = {};
    for (int ch = 0; ch < NCH; ++ch) {
      // Every consumer warp waits for every fill of every stage, in order, so the parity
      // names the right fill. The tiles' S'/Z transposes are awaited after their first
      // chunks: the transposes run in tile order and this warp has finished the previous
      // pair, so the slots' parities cannot alias either.
      bool ok = true;
      uint32_t wst[2];
      for (int u = 0; u < nt && ok; ++u) {
        const int st = (i + u) % NS;
        wst[u] = ring_lane + st * L.stage;
        ok = mbar_wait_spin_bounded(&full[st], ((i + u) / NS) & 1u, kDecWaitNs);
      }
      for (int u = 0; u < nt && ok && ch == 0; ++u)
        ok = mbar_wait_spin_bounded(&prepfull[ps[u]], ((tp + u) / kTileSlots) & 1u, kDecWaitNs);
      if (!ok) {
        set_status(status, kStTimeout);
        return;
      }
      if (nt == 1) wst[1] = wst[0];
      const int g0 = ch * gpc;
      const int gn = min(gpc, G - g0);
      const int qa = (warp * gn) / NW, qb = ((warp + 1) * gn) / NW;
      if (kPairTiles == 2 && nt == 2) {
        for (int q = qa; q < qb; ++q) group(std::integral_constant<int, 2>{}, q, g0 + q, wst, prep, acc);
      } else {
        for (int q = qa; q < qb; ++q) group(std::integral_constant<int, 1>{}, q, g0 + q, wst, prep, acc);
      }
      __syncwarp();
      if (lane == 0)
        for (int u = 0; u < nt; ++u) mbar_arrive(&empty[(i + u) % NS]);
      i += nt;
    }
    for (int u = 0; u < nt; ++u) {
      float* part = reinterpret_cast<float*>(smem + L.part + ps[u] * L.part_slot) + warp * 16 * MR;
      if (t0 < M) {
        part[r * MR + t0] = acc[u][0];
        part[(r + 8) * MR + t0] = acc[u][2];
      }
      if constexpr (M > 1) {
        if (t1 < M) {
          part[r * MR + t1] = acc[u][1];
          part[(r + 8) * MR + t1] = acc[u][3];
        }
      }
    }
    __syncwarp();
    if (lane == 0)
      for (int u = 0; u < nt; ++u) mbar_arrive(&tdone[ps[u]]);
  }
}

template <int M>
cudaError_t launch_decode_m(const GemvArgs& a, int sms, cudaStream_t st) {
  const int G = a.K / 128;
  const int ntiles = a.N / 16;
  if (ntiles == 0) return cudaSuccess;
  const int row_bytes = a.K / 2;
  const int NCH = (row_bytes + kChunkMax - 1) / kChunkMax;
  // whole rows only: rows split into several K-chunks are left to the other kernels
  if (NCH != 1) return cudaErrorInvalidValue;
  const int CK = static_cast<int>(align_up((row_bytes + NCH - 1) / NCH, 64));
  if ((NCH - 1) * CK >= row_bytes) return cudaErrorInvalidValue;  // no empty last chunk
  const int pitch = CK + ((64 - CK % 128) + 128) % 128;  // = 64 (mod 128)
  const uint32_t slack = 128;  // for aligning the dynamic base
  int RS = kRawSlotsMax, NS = 0;
  for (; RS >= 2; RS /= 2) {  // deepest S'/Z prefetch that leaves two ring stages
    const DecodeLayout base(M, G, pitch, 0, RS);
    if (base.total + slack > kSmemBudget) continue;
    NS = static_cast<int>((kSmemBudget - slack - base.total) / (base.stage + 16));
    if (NS >= 2) break;
  }
  if (NS > kMaxStages) NS = kMaxStages;
  if (RS < 2 || NS < 2) return cudaErrorInvalidValue;
  const DecodeLayout L(M, G, pitch, NS, RS);
  const size_t smem = L.total + slack;

  auto kern = gemv_decode<M>;
  static std::atomic<bool> attr[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 63].load(std::memory_order_acquire)) {
    const cudaError_t e = set_smem_attrs(kern, static_cast<int>(kSmemBudget));
    if (e != cudaSuccess) return e;
    attr[dev & 63].store(true, std::memory_order_release);
  }
  const int tpc = (ntiles + sms - 1) / sms;
  const int grid = (ntiles + tpc - 1) / tpc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32 * (kDecWarps + 3));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a.X, a.ldx, a.P, a.S, a.Z, a.N, a.K, CK, NCH, pitch, NS,
                            RS, tpc, a.Y, a.ldy, a.status);
}

}  // namespace

bool gemv_stream_fits(const GemvArgs& a) {
  if (a.M < 1 || a.M > 4 || a.K % 128 != 0) return false;
  const int row_bytes = a.K / 2;
  const int NCH = (row_bytes + kChunkMax - 1) / kChunkMax;
  if (NCH != 1) return false;  // whole rows only (K <= 6144)
  const int CK = static_cast<int>(align_up((row_bytes + NCH - 1) / NCH, 64));
  if ((NCH - 1) * CK >= row_bytes) return false;
  const int pitch = CK + ((64 - CK % 128) + 128) % 128;
  const DecodeLayout base(a.M, a.K / 128, pitch, 2, 2);
  return base.total + 128 <= kSmemBudget;
}

bool gemv_stream_ok(const GemvArgs& a) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return a.M >= 1 && a.M <= 4 && a.K % 128 == 0 && a.sz_row > 0 && a.group == 128 &&
         a.N % 16 == 0 && (a.ldx % 8) == 0 && al16(a.X) && al16(a.P) && al16(a.S) && al16(a.Z);
}

cudaError_t launch_gemv_stream(const GemvArgs& a, int sms, cudaStream_t st) {
  switch (a.M) {
    case 1: return launch_decode_m<1>(a, sms, st);
    case 2: return launch_decode_m<2>(a, sms, st);
    case 3: return launch_decode_m<3>(a, sms, st);
    case 4: return launch_decode_m<4>(a, sms, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wq
