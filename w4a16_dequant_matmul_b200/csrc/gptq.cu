// GPTQ into the library's INT4 format ("LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8
// & INT4/INT8 Trade-offs", section "GPTQ vs AWQ: two ways to choose what error to keep";
// "DL S067 - Quantization", section 4; "Model Quantization", section 2.1): quantize one input
// column at a time and move each column's rounding error onto the columns not yet quantized
// through the inverse of the dampened layer-input Hessian H = X^T X + damp mean(diag) I,
// dropping the finished column from the inverse after each step. The quantization grid
// (S', Z of every group) is that of round-to-nearest on the original weights, fixed before
// the sweep. All arithmetic of the sweep and the inverse is float64.
//
//  * hessian_kernel: H = X^T X from bf16 calibration activations, 64 x 64 tiles per CTA.
//  * damp_kernel: adds damp * mean(diag H) to the diagonal (one CTA).
//  * gj_step_kernel: one pivot of an in-place Gauss-Jordan inversion (no pivoting: H is
//    symmetric positive definite once dampened), from snapshots of the pivot row and column
//    that the previous step wrote; the next pivot's row and column are snapshotted by the
//    threads that finalise them. One launch per pivot.
//  * downdate_step_kernel: drops column i from the symmetric inverse (the trailing block
//    minus v v^T / v_i, v = row i); row i itself stays as it is: the row the sweep uses for
//    column i.
//  * sweep_kernel: one CTA per weight row, the row in shared memory; per column: the code
//    on the fixed grid, the error e = (w_i - S'(q - Z)) / F_ii, and w_j -= e F_ij for j > i.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace wq {
namespace {

constexpr int kHT = 64;  // Hessian tile

__global__ void __launch_bounds__(256)
hessian_kernel(const uint16_t* __restrict__ X, int64_t ldx, int T, int K, double* __restrict__ H) {
  __shared__ double xa[32][kHT + 1], xb[32][kHT + 1];
  const int i0 = blockIdx.y * kHT, j0 = blockIdx.x * kHT;
  const int ti = threadIdx.x >> 4, tj = threadIdx.x & 15;  // 16 x 16 threads, 4 x 4 each
  double acc[4][4] = {};
  for (int t0 = 0; t0 < T; t0 += 32) {
    for (int e = threadIdx.x; e < 32 * kHT; e += 256) {
      const int tt = e / kHT, c = e - tt * kHT;
      const bool ok = t0 + tt < T;
      const uint16_t* row = X + static_cast<int64_t>(t0 + tt) * ldx;
      xa[tt][c] = ok ? static_cast<double>(bf16_lo(row[i0 + c])) : 0.0;
      xb[tt][c] = ok ? static_cast<double>(bf16_lo(row[j0 + c])) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int tt = 0; tt < 32; ++tt) {
      double a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = xa[tt][ti + 16 * u];
        b[u] = xb[tt][tj + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v)
      H[static_cast<int64_t>(i0 + ti + 16 * u) * K + j0 + tj + 16 * v] = acc[u][v];
}

// diag += damp * mean(diag), then the snapshots of pivot 0's row and column.
__global__ void __launch_bounds__(1024)
damp_kernel(double* __restrict__ H, int K, double damp, double* __restrict__ rowv,
            double* __restrict__ colv) {
  __shared__ double part[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < K; i += blockDim.x) s += H[static_cast<int64_t>(i) * K + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  double tot = 0.0;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += part[w];  // fixed order
  const double add = damp * (tot / K);
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += blockDim.x) H[static_cast<int64_t>(i) * K + i] += add;
  __syncthreads();
  for (int c = threadIdx.x; c < K; c += blockDim.x) {
    rowv[c] = H[c];                          // row 0
    colv[c] = H[static_cast<int64_t>(c) * K];  // column 0
  }
}

// Gauss-Jordan pivot i in place: A <- A - col (row / p) off row i, row i <- row / p, and
// column i <- -col / p (A[i][i] <- 1 / p). rowv / colv hold pivot i's row and column; the
// threads that finalise row i + 1 and column i + 1 write them to nrow / ncol.
__global__ void __launch_bounds__(256)
gj_step_kernel(double* __restrict__ A, int K, int i, const double* __restrict__ rowv,
               const double* __restrict__ colv, double* __restrict__ nrow,
               double* __restrict__ ncol, unsigned* status) {
  const int64_t total = static_cast<int64_t>(K) * K;
  const double p = rowv[i];
  const double ip = 1.0 / p;
  if (blockIdx.x == 0 && threadIdx.x == 0 && !(p > 0.0 && isfinite(p))) set_status(status, kStNonFinite);
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(e / K), c = static_cast<int>(e - static_cast<int64_t>(r) * K);
    double v;
    if (r == i) v = c == i ? ip : rowv[c] * ip;
    else if (c == i) v = -colv[r] * ip;
    else v = A[e] - colv[r] * (rowv[c] * ip);
    A[e] = v;
    if (i + 1 < K) {
      if (r == i + 1) nrow[c] = v;
      if (c == i + 1) ncol[r] = v;
    }
  }
}

// Downdate pivot i of the symmetric inverse: for r, c > i, A[r][c] -= (v_r v_c) / v_i with
// v = row i (a snapshot; the product first, so the block stays exactly symmetric). Row i is
// left as it is. Row i + 1 of the result is snapshotted into nrow for the next pivot.
__global__ void __launch_bounds__(256)
downdate_step_kernel(double* __restrict__ A, int K, int i, const double* __restrict__ v,
                     double* __restrict__ nrow, unsigned* status) {
  const int n = K - i - 1;  // trailing block past row / column i
  const int64_t total = static_cast<int64_t>(n) * n;
  const double p = v[i];
  if (blockIdx.x == 0 && threadIdx.x == 0 && !(p > 0.0 && isfinite(p))) set_status(status, kStNonFinite);
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = i + 1 + static_cast<int>(e / n), c = i + 1 + static_cast<int>(e % n);
    double* a = A + static_cast<int64_t>(r) * K + c;
    const double x = *a - (v[r] * v[c]) / p;
    *a = x;
    if (r == i + 1) nrow[c] = x;
  }
}

// One weight row per CTA: the sweep over its K columns (the row lives in shared memory).
__global__ void __launch_bounds__(256)
sweep_kernel(const void* __restrict__ W, bool bf16, int64_t ldw, int K, int group,
             const double* __restrict__ F, const uint16_t* __restrict__ S,
             const uint16_t* __restrict__ Z, uint8_t* __restrict__ packed, unsigned* status) {
  extern __shared__ double w[];
  __shared__ double err_s;
  const int64_t n = blockIdx.x;
  const int G = K / group;
  for (int k = threadIdx.x; k < K; k += blockDim.x)
    w[k] = bf16 ? static_cast<double>(bf16_lo(static_cast<const uint16_t*>(W)[n * ldw + k]))
                : static_cast<double>(static_cast<const float*>(W)[n * ldw + k]);
  __syncthreads();
  uint32_t even = 0;
  bool bad = false;
  for (int i = 0; i < K; ++i) {
    if (threadIdx.x == 0) {
      const double s = f16_bits_to_f32(S[n * G + i / group]);
      const double z = f16_bits_to_f32(Z[n * G + i / group]);
      const double wi = w[i];
      double q = rint(wi / s) + z;  // round half to even, as the fixed grid's codes
      q = fmin(fmax(q, 0.0), 15.0);
      bad |= !isfinite(wi);
      err_s = (wi - s * (q - z)) / F[static_cast<int64_t>(i) * K + i];
      const uint32_t code = static_cast<uint32_t>(q);
      if (i & 1) packed[n * (K / 2) + i / 2] = static_cast<uint8_t>(even | (code << 4));
      else even = code;
    }
    __syncthreads();
    const double e = err_s;
    const double* f = F + static_cast<int64_t>(i) * K;
    for (int j = i + 1 + threadIdx.x; j < K; j += blockDim.x) w[j] -= e * f[j];
    __syncthreads();
  }
  if (threadIdx.x == 0 && bad) set_status(status, kStNonFinite);
}

}  // namespace

size_t gptq_workspace_bytes(int64_t K) {
  return static_cast<size_t>(K) * static_cast<size_t>(K) * sizeof(double) + 4 * K * sizeof(double);
}

int gptq_max_k() { return 8192; }

cudaError_t launch_gptq(const void* W, bool bf16, int64_t ldw, int N, int K, int group,
                        const uint16_t* X, int64_t ldx, int T, double damp, uint8_t* packed,
                        const uint16_t* S, const uint16_t* Z, void* workspace, unsigned* status,
                        int sms, cudaStream_t st) {
  double* A = static_cast<double*>(workspace);
  double* vec = A + static_cast<int64_t>(K) * K;  // [4][K]: two row / column snapshot pairs
  double* rowv[2] = {vec, vec + 2 * K};
  double* colv[2] = {vec + K, vec + 3 * K};
  hessian_kernel<<<dim3(K / kHT, K / kHT), 256, 0, st>>>(X, ldx, T, K, A);
  damp_kernel<<<1, 1024, 0, st>>>(A, K, damp, rowv[0], colv[0]);
  const int64_t total = static_cast<int64_t>(K) * K;
  const int gj_grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, 8LL * sms));
  for (int i = 0; i < K; ++i)
    gj_step_kernel<<<gj_grid, 256, 0, st>>>(A, K, i, rowv[i & 1], colv[i & 1], rowv[(i + 1) & 1],
                                            colv[(i + 1) & 1], status);
  // the inverse is symmetric: row 0 is the first pivot's snapshot
  cudaMemcpyAsync(rowv[0], A, K * sizeof(double), cudaMemcpyDeviceToDevice, st);
  for (int i = 0; i + 1 < K; ++i) {
    const int64_t t = static_cast<int64_t>(K - i - 1) * (K - i - 1);
    const int g = static_cast<int>(std::min<int64_t>(std::max<int64_t>((t + 255) / 256, 1), 8LL * sms));
    downdate_step_kernel<<<g, 256, 0, st>>>(A, K, i, rowv[i & 1], rowv[(i + 1) & 1], status);
  }
  const size_t smem = static_cast<size_t>(K) * sizeof(double);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(sweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  sweep_kernel<<<N, 256, smem, st>>>(W, bf16, ldw, K, group, A, S, Z, packed, status);
  return cudaGetLastError();
}

}  // namespace wq
