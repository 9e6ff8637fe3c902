// gdn_chunked.cu -- chunked WY/UT dual-stream forward on tcgen05 tensor cores (sm_100a).
#include "gdn_internal.cuh"

namespace gdn {

bool chunked_supported(int dtype, int d, int B, int conv_width) {
    (void)dtype; (void)d; (void)B; (void)conv_width;
    return false;
}

cudaError_t launch_chunked(const Params &p, cudaStream_t stream) {
    (void)p; (void)stream;
    return cudaErrorNotSupported;
}

}  // namespace gdn
