// Few-token forward path (placeholder until the dequant-GEMV kernel lands):
// disabled, so every M runs the tensor-core fused dequant-GEMM.
#include "internal.h"

namespace qlora {

bool gemv_enabled() { return false; }

qlora_status launch_gemv(const GemvArgs &, cudaStream_t) { return QLORA_ERR_UNSUPPORTED_SHAPE; }

}  // namespace qlora
