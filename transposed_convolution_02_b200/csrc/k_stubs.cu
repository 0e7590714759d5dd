// Placeholders for kernel modules not built yet: they serve no plan.
#include "ct_internal.h"

namespace ct {
bool fp32_gemm_supports(const Plan &) { return false; }
size_t fp32_gemm_packed_bytes(const Plan &) { return 0; }
ct_status fp32_gemm_prepack(const Plan &, const void *, void *, cudaStream_t) { return CT_ERR_UNSUPPORTED; }
ct_status fp32_gemm_run(const Plan &, const void *, const void *, const void *, void *, cudaStream_t) { return CT_ERR_UNSUPPORTED; }
}  // namespace ct
