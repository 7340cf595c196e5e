// Tensor-core (tcgen05/TMEM) W4A16 / W8A16 GEMM for larger M: interface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wq.h"

namespace wq {

struct TcGemmArgs {
  const uint16_t* X;   // bf16 [M, K], row stride ldx
  int64_t ldx;
  const uint8_t* P;    // packed INT4 [N, K/2] (W4A16), or nullptr
  const uint16_t* S;   // binary16 scales
  const uint16_t* Z;   // binary16 zero-points (W4A16) or nullptr
  const int8_t* Q8;    // INT8 codes [N, K] (W8A16), or nullptr
  int M, N, K, group, sz_row;
  uint16_t* Y;         // bf16 [M, N], row stride ldy
  int64_t ldy;
};

wq_status launch_tc_gemm(const TcGemmArgs& a, int sms, unsigned* status, cudaStream_t st);

}  // namespace wq
