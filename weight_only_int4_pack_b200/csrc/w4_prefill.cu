// w4_prefill.cu -- the W4A16 linear layer for large M (placeholder until the
// tcgen05 kernel lands).
#include "w4_internal.cuh"

namespace w4 {
int launch_prefill(const void *, int, int64_t, const uint8_t *, const float *, const float *,
                   int64_t, int64_t, void *, cudaStream_t) {
    return W4_ERR_UNSUPPORTED;
}
}  // namespace w4
