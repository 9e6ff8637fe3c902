// gdn_noalloc.cu -- gdn_dual_forward for callers that cannot allocate device memory.
//
// gdn_dual_forward asks its caller for a small device workspace (the kernels' status words).
// Some hosts of this library have no way to provide one: an inference engine that reserved
// all device memory for its own pool up front (a fresh cudaMalloc would fail or fragment that
// pool), or a plugin / FFI host that exposes no device allocator across the C ABI.  This entry
// point serves them: the workspace is a fixed array in the library's own device memory, so
// the caller passes only inputs and outputs and nothing is allocated on any call.
#include <mutex>

#include "gdn_internal.cuh"

namespace {

// Fixed scratch: 4096 bytes.  Every GPU that loads this library holds it until the process
// exits.  The kernels need 256 bytes of it (their status words and work counter); with ShortConv
// the conv then runs in the chunked kernel's prologue (the separate conv pass would need room for
// the convolved inputs).
constexpr size_t kNoAllocScratchBytes = 4096;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};   // device address of the array, per device ordinal

// Device address of the scratch array on the current device.  The first call on a device looks
// it up (host code cannot use the symbol itself, which is only a host-side stand-in for the
// device array) and keeps it for the life of the process: the address belongs to the device's
// primary context, the one the CUDA runtime uses.
gdn_status scratch_address(void **addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return GDN_OK;
}

}  // namespace

extern "C" gdn_status gdn_dual_forward_noalloc(const gdn_dual_desc *desc,
                                               const void *q, const void *k, const void *v,
                                               const float *g, const float *beta,
                                               const void *qn, const void *kn, const void *vn,
                                               const float *gn, const float *betan,
                                               const int32_t *doc_offsets, const int32_t *prompt_len,
                                               const float *conv_w,
                                               void *out, void *out_noisy, float *final_state,
                                               gdn_stream_t stream) {
    if (!desc || !doc_offsets) return GDN_ERR_INVALID_ARG;
    // Route I keeps every block-boundary state in its workspace: far more than the array holds.
    if (desc->algo == GDN_ALGO_ROUTE1) return GDN_ERR_UNSUPPORTED;
    if (gdn_dual_workspace_size(desc, doc_offsets) == 0) return GDN_ERR_INVALID_ARG;
    static_assert(sizeof(gdn::WorkspaceHeader) <= kNoAllocScratchBytes, "the status words fit the array");
    void *scratch = nullptr;
    const gdn_status st = scratch_address(&scratch);
    if (st != GDN_OK) return st;
    // gdn_dual_forward clears the status words at the start of the scratch on `stream` before
    // the launch; the rest of the array is never read before it is written.
    return gdn_dual_forward(desc, q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, conv_w,
                            out, out_noisy, final_state, scratch, kNoAllocScratchBytes, stream);
}

extern "C" gdn_status gdn_dual_noalloc_read_device_status(gdn_stream_t stream) {
    void *scratch = nullptr;
    const gdn_status st = scratch_address(&scratch);
    if (st != GDN_OK) return st;
    return gdn_dual_read_device_status(scratch, stream);
}
