// Internal launch interface between the C ABI layer (api.cu) and the kernel files.
// Every launcher validates nothing: api.cu checks shapes, alignment and pointers first.
#pragma once

#include <cuda_runtime.h>
#include <initializer_list>
#include <stdint.h>

namespace wq {

// SM count and device address of the status word for the current device (false if there
// is no usable sm_100 device). Defined in api.cu.
bool current_device(int* sms, unsigned** status);
// Every non-null pointer is memory of the current device (or managed memory). api.cu.
bool pointers_on_current_device(std::initializer_list<const void*> ptrs);

// sym: symmetric INT4 (s' = max|w|/7, Z = 8) in the same storage.
cudaError_t launch_quant_asym(const void* W, bool bf16, int64_t ldw, int N, int K, int group,
                              uint8_t* packed, uint16_t* S, uint16_t* Z, bool sym,
                              unsigned* status, int sms, cudaStream_t st);
cudaError_t launch_quant_sym_int8(const void* W, bool bf16, int64_t ldw, int N, int K,
                                  int8_t* codes, uint16_t* S, unsigned* status, int sms,
                                  cudaStream_t st);
int per_tensor_parts(int sms);
cudaError_t launch_quant_per_tensor(const void* W, bool bf16, int64_t ldw, int N, int K,
                                    uint8_t* packed, uint16_t* S, uint16_t* Z, float2* part,
                                    int nparts, unsigned* status, cudaStream_t st);

cudaError_t launch_pack_int4(const uint8_t* codes, int64_t N, int64_t K, uint8_t* packed,
                             unsigned* status, int sms, cudaStream_t st);
cudaError_t launch_dequant(const uint8_t* packed, const uint16_t* S, const uint16_t* Z,
                           int64_t N, int K, int group, int sz_row, void* out, bool bf16_out,
                           int sms, cudaStream_t st);

// Small-M W4A16 matmul on CUDA cores. sz_row = scales per row (K/group), 0 = per-tensor.
struct GemvArgs {
  const uint16_t* X;
  int64_t ldx;
  const uint8_t* P;
  const uint16_t* S;
  const uint16_t* Z;
  int M, N, K, group, sz_row;
  uint16_t* Y;
  int64_t ldy;
  unsigned* status;
};
int gemv_max_k();
// Streaming TMA-fed decode kernel for M <= 4, g = 128 (decode.cu).
bool gemv_stream_ok(const GemvArgs& a);
bool gemv_stream_fits(const GemvArgs& a);
// Integer-MMA decode kernel for M <= 2, g = 128, short rows: whole-row tiles by bulk copies
// (gemv_imma.cu).
bool gemv_imma_bulk_ok(const GemvArgs& a);
cudaError_t launch_gemv_imma_bulk(const GemvArgs& a, int sms, cudaStream_t st);
// 32-row-tile TMA-fed decode kernel for M <= 4, g = 128, N % 32 == 0 (gemv_tma.cu).
bool gemv_tma_ok(const GemvArgs& a);
cudaError_t launch_gemv_tma(const GemvArgs& a, int sms, cudaStream_t st);
// Largest token block (8, 4, 2 or 1, at most a.M) with a fast decode kernel; 0 if none.
int gemv_fast_block(const GemvArgs& a);
cudaError_t launch_gemv_stream(const GemvArgs& a, int sms, cudaStream_t st);
cudaError_t launch_gemv_w4a16(const GemvArgs& a, int sms, cudaStream_t st);

// Skinny M (up to kSkinnyMaxTokens tokens), g = 128: tcgen05 kind::f16 on the centred codes
// as bf16 and the activations, split-K over a thread-block cluster (tc_skinny.cu). a.M is the
// full M.
constexpr int kSkinnyMaxTokens = 64;
bool tc_skinny_ok(const GemvArgs& a);
cudaError_t launch_tc_skinny(const GemvArgs& a, int sms, cudaStream_t st);
// The same for W8A16: a.P = int8 codes [N, K], a.S = per-row scales [N], a.Z unused.
bool tc_skinny8_ok(const GemvArgs& a);
cudaError_t launch_tc_skinny8(const GemvArgs& a, int sms, cudaStream_t st);

// Small-M W8A16 (symmetric INT8 per output channel) on CUDA cores.
struct Gemv8Args {
  const uint16_t* X;
  int64_t ldx;
  const int8_t* Q;
  const uint16_t* S;
  int M, N, K;
  uint16_t* Y;
  int64_t ldy;
};
cudaError_t launch_gemv_w8a16(const Gemv8Args& a, cudaStream_t st);

// Per-input-channel scale folding (scale_fold.cu). cols % 8 == 0 for channel_stat.
cudaError_t launch_channel_stat(const void* A, bool bf16, int64_t lda, int64_t rows, int cols,
                                bool mean, float* out, int sms, cudaStream_t st);
cudaError_t launch_smooth_scales(const float* xmax, const float* wmax, int K, float alpha,
                                 float* s, int sms, cudaStream_t st);
cudaError_t launch_awq_scales(const float* a_mag, int K, float alpha, float* s,
                              cudaStream_t st);
cudaError_t launch_quant_scaled(const void* W, bool bf16, int64_t ldw, int N, int K, int group,
                                const float* s, uint8_t* packed, uint16_t* S, uint16_t* Z,
                                bool sym, unsigned* status, int sms, cudaStream_t st);
cudaError_t launch_scale_activations(const uint16_t* X, int64_t ldx, int M, int K,
                                     const float* s, uint16_t* Xs, int64_t ldxs, int sms,
                                     cudaStream_t st);

// GPTQ sweep on a fixed grid (gptq.cu): workspace of gptq_workspace_bytes(K) bytes.
size_t gptq_workspace_bytes(int64_t K);
int gptq_max_k();
cudaError_t launch_gptq(const void* W, bool bf16, int64_t ldw, int N, int K, int group,
                        const uint16_t* X, int64_t ldx, int T, double damp, uint8_t* packed,
                        const uint16_t* S, const uint16_t* Z, void* workspace, unsigned* status,
                        int sms, cudaStream_t st);

// One CTA whose single bounded mbarrier wait runs out (selftest.cu).
cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, bool spin, unsigned* status,
                                         cudaStream_t st);

}  // namespace wq
