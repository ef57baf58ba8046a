// Fused NF4 doubleDequant + tcgen05 GEMM (placeholder until the sm_100a
// kernel lands: reports every shape as unsupported).
#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

bool nf4_tc_gemm_supported(const qln_nf4_weight *, bool, int64_t, int) { return false; }

cudaError_t launch_nf4_tc_gemm(const qln_nf4_weight *, bool, const uint16_t *, int64_t, const uint16_t *,
                               const uint16_t *, int, uint16_t *, int *, cudaStream_t, int) {
    return cudaErrorNotSupported;
}

}  // namespace qln
