// Per-input-channel scale folding ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 &
// INT4/INT8 Trade-offs", sections "Granularity and outliers" (SmoothQuant) and "GPTQ vs
// AWQ"; "DL S067 - Quantization", section 5 "AWQ intuition"): a factor s_j per input
// channel multiplies column j of the weights before round-to-nearest and divides column j of
// the activations, which leaves X W^T unchanged.
//
//  * channel_stat: max |A_ij| or mean |A_ij| over the rows of each column. A cluster of
//    CTAs splits the rows of one 128-column strip; each CTA reduces its rows in registers,
//    and the cluster's first CTA combines the partials through distributed shared memory in
//    a fixed order (deterministic, no atomics, no workspace).
//  * smooth_scales / awq_scales: the two factor formulas, in float64, rounded to float32.
//  * quant_scaled: RTN INT4 of w * s_k, the product rounded once to float32, with the same
//    exact scale / zero-point / code decisions as the unscaled quantizer.
//  * scale_activations: bf16(x / s_k), the float32 quotient rounded to bfloat16.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace wq {
namespace {

constexpr int kStatCols = 128;  // columns per strip: 32 lanes x 4
constexpr int kStatWarps = 8;

__device__ __forceinline__ void load4(const uint16_t* p, float v[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
  v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
}
__device__ __forceinline__ void load4(const float* p, float v[4]) {
  const float4 u = *reinterpret_cast<const float4*>(p);
  v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
}

// Correctly rounded float32 of sum / n for an exact float64 sum >= 0 and 0 < n < 2^53: the
// float64 quotient q can only mislead the float32 rounding when q lies exactly halfway
// between two floats while the true quotient does not; the FMA remainder sum - q n (exact)
// says on which side the true quotient lies, and q moves one float64 step that way.
__device__ __forceinline__ float div_to_f32(double sum, double n) {
  double q = sum / n;  // >= 0
  const float f = __double2float_rn(q);
  const double lo = static_cast<double>(f);
  if (isfinite(q) && q != lo) {
    // the float on q's other side (f > 0 whenever q < f, so one bit step is the neighbour)
    const float g = __int_as_float(__float_as_int(f) + (q > lo ? 1 : -1));
    if (q == 0.5 * (lo + static_cast<double>(g))) {  // q is a float32 midpoint
      const double r = fma(-q, n, sum);
      const long long b = __double_as_longlong(q);
      if (r > 0.0) q = __longlong_as_double(b + 1);
      else if (r < 0.0) q = __longlong_as_double(b - 1);
    }
  }
  return __double2float_rn(q);
}

// One 128-column strip per cluster; the cluster's CTAs (cluster dim y) split the rows.
// kMean: mean |a| (float64 sums), else max |a| (NaN-propagating).
template <typename T, bool kMean>
__global__ void __launch_bounds__(32 * kStatWarps)
channel_stat_kernel(const T* __restrict__ A, int64_t lda, int64_t rows, int cols,
                    float* __restrict__ out) {
  using Acc = typename std::conditional<kMean, double, float>::type;
  __shared__ Acc part[kStatWarps][kStatCols];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int csize = static_cast<int>(cluster.num_blocks());
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col = blockIdx.x * kStatCols + 4 * lane;
  Acc acc[4] = {Acc(0), Acc(0), Acc(0), Acc(0)};
  if (col < cols) {
    const int64_t step = static_cast<int64_t>(csize) * kStatWarps;
    for (int64_t r = static_cast<int64_t>(crank) * kStatWarps + warp; r < rows; r += step) {
      float v[4];
      load4(A + r * lda + col, v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if constexpr (kMean) acc[i] += static_cast<double>(fabsf(v[i]));
        else acc[i] = fmax_nan(acc[i], fabsf(v[i]));
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) part[warp][4 * lane + i] = acc[i];
  cluster.sync();
  if (crank == 0 && threadIdx.x < kStatCols) {
    const int c = blockIdx.x * kStatCols + threadIdx.x;
    Acc t = Acc(0);
    for (int b = 0; b < csize; ++b) {
      const Acc* p = cluster.map_shared_rank(&part[0][0], b);
      for (int w = 0; w < kStatWarps; ++w) {
        const Acc x = p[w * kStatCols + threadIdx.x];
        if constexpr (kMean) t += x;
        else t = fmax_nan(t, x);
      }
    }
    if (c < cols) {
      if constexpr (kMean) out[c] = div_to_f32(t, static_cast<double>(rows));
      else out[c] = t;
    }
  }
  cluster.sync();  // the other CTAs' shared memory stays alive until it has been read
}

// s_j = xmax_j^alpha / wmax_j^(1 - alpha), or 1 where either statistic is not > 0.
__global__ void smooth_scales_kernel(const float* __restrict__ xmax,
                                     const float* __restrict__ wmax, int K, float alpha,
                                     float* __restrict__ s) {
  const double a = alpha, b = 1.0 - static_cast<double>(alpha);
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < K; j += gridDim.x * blockDim.x) {
    const float x = xmax[j], w = wmax[j];
    float r = 1.0f;
    if (x > 0.0f && w > 0.0f) r = __double2float_rn(pow(static_cast<double>(x), a) /
                                                    pow(static_cast<double>(w), b));
    s[j] = r;
  }
}

// s_j = p_j / sqrt(max p * min p) with p_j = a_j^alpha over the channels with a_j > 0;
// 1 for the others. One CTA: the max / min reduction, then the factors.
constexpr int kAwqThreads = 1024;
__global__ void __launch_bounds__(kAwqThreads)
awq_scales_kernel(const float* __restrict__ a_mag, int K, float alpha, float* __restrict__ s) {
  __shared__ double smax[32], smin[32];
  const double e = alpha;
  double mx = -INFINITY, mn = INFINITY;
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    const float a = a_mag[j];
    if (a > 0.0f) {
      const double p = pow(static_cast<double>(a), e);
      mx = fmax(mx, p);
      mn = fmin(mn, p);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    smax[warp] = mx;
    smin[warp] = mn;
  }
  __syncthreads();
  mx = -INFINITY;
  mn = INFINITY;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
    mx = fmax(mx, smax[w]);
    mn = fmin(mn, smin[w]);
  }
  const double norm = sqrt(mx * mn);
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    const float a = a_mag[j];
    s[j] = a > 0.0f ? __double2float_rn(pow(static_cast<double>(a), e) / norm) : 1.0f;
  }
}

// Four folded weights w * s (float32 products) starting at column k. A factor that is not
// finite and positive is flagged and its column folds to 0, so that it is reported as a bad
// factor (WQ_ERR_RANGE) rather than through the non-finite products it would make.
template <typename T>
__device__ __forceinline__ void fold4(const T* w, const float* s, float v[4], bool& bad_s) {
  float x[4];
  load4(w, x);
  const float4 f = *reinterpret_cast<const float4*>(s);
  const float fs[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool bad = !(fs[i] > 0.0f) || isinf(fs[i]);
    bad_s |= bad;
    v[i] = bad ? 0.0f : __fmul_rn(x[i], fs[i]);
  }
}

// RTN INT4 of the folded weights. A warp takes one group (g >= 128) or one 128-weight
// chunk holding 128/g groups (g = 32, 64); lane l owns 4 consecutive weights of every
// 128-weight step. Pass 1 reduces the range over the group's lanes, pass 2 re-reads the
// weights (L1 hits) and writes the codes.
template <typename T>
__global__ void __launch_bounds__(256)
quant_scaled_kernel(const T* __restrict__ W, int64_t ldw, int N, int K, int group,
                    const float* __restrict__ s, uint8_t* __restrict__ packed,
                    uint16_t* __restrict__ S, uint16_t* __restrict__ Z, bool sym,
                    unsigned* status) {
  const int lane = threadIdx.x & 31;
  const int span = group >= 128 ? group : 128;   // weights per warp unit
  const int lanes = group >= 128 ? 32 : group / 4;  // lanes sharing one group
  const int units_per_row = K / span;
  const int64_t units = static_cast<int64_t>(N) * units_per_row;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  bool bad_s = false;
  for (int64_t u = warp; u < units; u += nwarps) {
    const int64_t n = u / units_per_row;
    const int k0 = static_cast<int>(u - n * units_per_row) * span;
    const T* wrow = W + n * ldw;
    float mn = 0.0f, mx = 0.0f;
    for (int k = k0 + 4 * lane; k < k0 + span; k += 128) {
      float v[4];
      fold4(wrow + k, s + k, v, bad_s);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mn = fmin_nan(mn, v[i]);
        mx = fmax_nan(mx, v[i]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float omn = __shfl_xor_sync(0xffffffffu, mn, o);
      const float omx = __shfl_xor_sync(0xffffffffu, mx, o);
      if (o < lanes) {
        mn = fmin_nan(mn, omn);
        mx = fmax_nan(mx, omx);
      }
    }
    const AsymScale sz = sym ? sym4_scale_zero(mn, mx) : asym_scale_zero(mn, mx);
    uint8_t* dst = packed + n * (K / 2);
    for (int k = k0 + 4 * lane; k < k0 + span; k += 128) {
      float v[4];
      fold4(wrow + k, s + k, v, bad_s);
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float q = rne_quotient(v[i], sz.s, sz.inv_s) + sz.z;
        q = fminf(fmaxf(q, 0.0f), 15.0f);
        word |= static_cast<uint32_t>(__float2int_rz(q)) << (4 * i);
      }
      *reinterpret_cast<uint16_t*>(dst + k / 2) = static_cast<uint16_t>(word);
    }
    if (lane % lanes == 0) {
      const int64_t gi = n * (K / group) + (k0 + 4 * lane) / group;
      S[gi] = static_cast<uint16_t>(sz.sbits);
      Z[gi] = static_cast<uint16_t>(f32_to_f16_bits(sz.z));
      if (sz.bad) set_status(status, kStNonFinite);
    }
  }
  if (__any_sync(0xffffffffu, bad_s) && lane == 0) set_status(status, kStRange);
}

// Xs = bf16(x / s_k): 8 activations per thread (16-byte loads and stores).
__global__ void __launch_bounds__(256)
scale_activations_kernel(const uint16_t* __restrict__ X, int64_t ldx, int M, int K,
                         const float* __restrict__ s, uint16_t* __restrict__ Xs,
                         int64_t ldxs) {
  const int per_row = K / 8;
  const int64_t total = static_cast<int64_t>(M) * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / per_row;
    const int k = static_cast<int>(i - m * per_row) * 8;
    const uint4 x = *reinterpret_cast<const uint4*>(X + m * ldx + k);
    const float4 f0 = *reinterpret_cast<const float4*>(s + k);
    const float4 f1 = *reinterpret_cast<const float4*>(s + k + 4);
    uint4 y;
    y.x = pack_bf16x2(__fdiv_rn(bf16_lo(x.x), f0.x), __fdiv_rn(bf16_hi(x.x), f0.y));
    y.y = pack_bf16x2(__fdiv_rn(bf16_lo(x.y), f0.z), __fdiv_rn(bf16_hi(x.y), f0.w));
    y.z = pack_bf16x2(__fdiv_rn(bf16_lo(x.z), f1.x), __fdiv_rn(bf16_hi(x.z), f1.y));
    y.w = pack_bf16x2(__fdiv_rn(bf16_lo(x.w), f1.z), __fdiv_rn(bf16_hi(x.w), f1.w));
    *reinterpret_cast<uint4*>(Xs + m * ldxs + k) = y;
  }
}

int blocks_for(int64_t items, int per_block, int sms) {
  int64_t b = (items + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (b > cap) b = cap;
  return static_cast<int>(b < 1 ? 1 : b);
}

template <typename T, bool kMean>
cudaError_t launch_stat_t(const T* A, int64_t lda, int64_t rows, int cols, float* out, int sms,
                          cudaStream_t st) {
  const int strips = (cols + kStatCols - 1) / kStatCols;
  // Row splits per strip: enough clusters to cover the SMs about twice, at most 8 CTAs
  // (the portable cluster size) and at most one CTA per 8 rows.
  int cy = 1;
  while (cy < 8 && static_cast<int64_t>(strips) * cy < 2 * sms &&
         static_cast<int64_t>(cy) * 2 * kStatWarps <= rows)
    cy *= 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(strips, cy, 1);
  cfg.blockDim = dim3(32 * kStatWarps, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = cy;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, channel_stat_kernel<T, kMean>, A, lda, rows, cols, out);
}

}  // namespace

cudaError_t launch_channel_stat(const void* A, bool bf16, int64_t lda, int64_t rows, int cols,
                                bool mean, float* out, int sms, cudaStream_t st) {
  if (bf16) {
    const uint16_t* a = static_cast<const uint16_t*>(A);
    return mean ? launch_stat_t<uint16_t, true>(a, lda, rows, cols, out, sms, st)
                : launch_stat_t<uint16_t, false>(a, lda, rows, cols, out, sms, st);
  }
  const float* a = static_cast<const float*>(A);
  return mean ? launch_stat_t<float, true>(a, lda, rows, cols, out, sms, st)
              : launch_stat_t<float, false>(a, lda, rows, cols, out, sms, st);
}

cudaError_t launch_smooth_scales(const float* xmax, const float* wmax, int K, float alpha,
                                 float* s, int sms, cudaStream_t st) {
  smooth_scales_kernel<<<blocks_for(K, 256, sms), 256, 0, st>>>(xmax, wmax, K, alpha, s);
  return cudaGetLastError();
}

cudaError_t launch_awq_scales(const float* a_mag, int K, float alpha, float* s,
                              cudaStream_t st) {
  awq_scales_kernel<<<1, kAwqThreads, 0, st>>>(a_mag, K, alpha, s);
  return cudaGetLastError();
}

cudaError_t launch_quant_scaled(const void* W, bool bf16, int64_t ldw, int N, int K, int group,
                                const float* s, uint8_t* packed, uint16_t* S, uint16_t* Z,
                                bool sym, unsigned* status, int sms, cudaStream_t st) {
  const int span = group >= 128 ? group : 128;
  const int grid = blocks_for(static_cast<int64_t>(N) * (K / span), 8, sms);
  if (bf16)
    quant_scaled_kernel<uint16_t><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(W), ldw, N,
                                                        K, group, s, packed, S, Z, sym, status);
  else
    quant_scaled_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(W), ldw, N, K,
                                                     group, s, packed, S, Z, sym, status);
  return cudaGetLastError();
}

cudaError_t launch_scale_activations(const uint16_t* X, int64_t ldx, int M, int K,
                                     const float* s, uint16_t* Xs, int64_t ldxs, int sms,
                                     cudaStream_t st) {
  const int grid = blocks_for(static_cast<int64_t>(M) * (K / 8), 256, sms);
  scale_activations_kernel<<<grid, 256, 0, st>>>(X, ldx, M, K, s, Xs, ldxs);
  return cudaGetLastError();
}

}  // namespace wq
