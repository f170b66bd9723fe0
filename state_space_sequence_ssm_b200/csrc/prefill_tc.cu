// prefill_tc.cu -- tcgen05/TMEM/TMA chunked prefill (bf16 I/O, fp32 state).
#include "m3_internal.h"

namespace m3 {

bool prefill_tc_supported(const Problem &, const char **why) {
    *why = "tensor-core prefill not built yet";
    return false;
}

size_t prefill_tc_workspace(const Problem &) { return 0; }

cudaError_t launch_prefill_tc(const Problem &, const char **why) {
    *why = "tensor-core prefill not built yet";
    return cudaErrorNotSupported;
}

}  // namespace m3
