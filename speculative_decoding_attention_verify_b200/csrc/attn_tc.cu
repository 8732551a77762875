// Tensor-core (tcgen05) attention path: not built yet; every problem runs on the CUDA-core
// engine until it is.
#include "sd_internal.h"

namespace sd {

bool tc_supported(int kind, int dtype, int head_dim, int rows) {
    (void)kind; (void)dtype; (void)head_dim; (void)rows;
    return false;
}

cudaError_t launch_attention_tc(const AttnParams &, const AttnPlan &, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace sd
