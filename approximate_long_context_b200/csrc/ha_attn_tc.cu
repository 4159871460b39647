// ha_attn_tc.cu -- tensor-core (tcgen05) attention kernels. Placeholder entry points until the
// tensor-core kernels land: they report "unsupported" so that the caller picks the SIMT kernels.
#include "ha_internal.h"

namespace ha {

int launch_attn_tc(const Level &, const void *, const void *, const void *, int, const int32_t *, const int32_t *,
                   const int32_t *, int, int64_t, void *, int, float *, float *, float *, int *, cudaStream_t) {
    return -2;
}

int launch_causal_base_tc(const void *, const void *, const void *, int64_t, int64_t, int, int64_t, int,
                          const float *, const float *, void *, int, int *, cudaStream_t) {
    return -2;
}

}  // namespace ha
