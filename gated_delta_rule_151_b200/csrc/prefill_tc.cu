// tcgen05 chunked prefill (bf16 I/O, d_k = d_v = 128): not built yet.
#include "internal.h"

namespace gdr {

bool tcgen05_prefill_available() { return false; }

size_t tcgen05_workspace_bytes(int, int, int) { return 0; }

cudaError_t launch_prefill_tcgen05(const void *, const void *, const void *, const float *,
                                   const float *, const float *, const int32_t *, int, int, int,
                                   bool, void *, float *, void *, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace gdr
