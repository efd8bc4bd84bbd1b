// Tensor-core path dispatch.
#include "tc.h"

namespace la {

bool tc_supported(const Problem&) { return false; }

cudaError_t tc_kv_partial(const Problem&, const void*, const void*, int, int, float*, cudaStream_t) {
    return cudaErrorNotSupported;
}
cudaError_t tc_readout(const Problem&, const void*, const float*, const float*, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}
cudaError_t tc_causal(const Problem&, int, const void*, const void*, const void*, const float*, int,
                      int, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace la
