// chunked_tc.cu -- tensor-core (tcgen05) chunked kernel: not built yet.
#include "common.cuh"

namespace gdr {

bool chunked_tc_supports(const gdr_desc&) { return false; }

cudaError_t launch_chunked_tc(const gdr_desc&, const void*, const void*, const void*,
                              const void*, const void*, const void*, const float*, void*,
                              float*, int*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace gdr
