// K3: INT4 W4A4 GEMM (placeholder until the tcgen05 kind::i8 kernel lands).
#include "svdq_internal.h"

namespace svdq {
int launch_gemm_int4(const svdq_layer*, int64_t, void*, uint8_t*, const Workspace&, int32_t*, cudaStream_t) {
  return SVDQ_ERR_INVALID_ARG;
}
}  // namespace svdq
