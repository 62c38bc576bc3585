// Fused tcgen05 tensor-core prefill: not built yet; the SIMT path serves every shape.
#include "gdn2_internal.h"

namespace gdn2 {

bool tc_supported(int, int, int, int, int, int, int) { return false; }
size_t tc_workspace_bytes(int, int, int, int, int, int) { return kStatusBytes; }
int launch_chunk_tc(const void *, const void *, const void *, const float *, const void *, const void *,
                    const float *, void *, float *, int, int, int, int, int, int, void *, cudaStream_t) {
    return -4;
}

}  // namespace gdn2
