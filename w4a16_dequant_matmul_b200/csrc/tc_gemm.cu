// Tensor-core W4A16 / W8A16 GEMM (placeholder until the tcgen05 kernel lands).
#include "tc_gemm.h"

namespace wq {

wq_status launch_tc_gemm(const TcGemmArgs&, int, unsigned*, cudaStream_t) {
  return WQ_ERR_UNSUPPORTED;
}

}  // namespace wq
