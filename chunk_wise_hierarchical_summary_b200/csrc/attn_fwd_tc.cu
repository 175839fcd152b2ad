// Tensor-core (tcgen05) prefill attention: placeholder until the sm_100a kernel lands.
#include "internal.h"

namespace hils {
bool attn_fwd_tc_supported(const Dims &, int) { return false; }
size_t attn_fwd_tc_workspace(const Dims &) { return 0; }
cudaError_t launch_attn_fwd_tc(const Dims &, const void *, const void *, const void *, const void *, const void *,
                               const float *, const int *, void *, float *, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace hils
