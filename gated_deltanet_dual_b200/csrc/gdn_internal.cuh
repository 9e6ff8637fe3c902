// gdn_internal.cuh -- parameters shared by the host entry points and the kernels of the
// dual-stream Gated DeltaNet forward (sm_100a).  Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/gdn_dual.h"

namespace gdn {

// Documents are passed to the kernels by value (kernel parameter space), so a launch needs no
// host-to-device copy and no allocation.  1024 documents keep the parameter block ~16 KB.
constexpr int kMaxDocs = 1024;

// Iteration bound of every device-side mbarrier wait (each iteration is one try_wait, which
// itself may suspend the thread for a while), and of the drain of outstanding copies and MMAs
// after a wait gave up.  Kernels take the bound of their ordinary waits from their parameters,
// so that a test can make a wait give up on purpose.
constexpr uint32_t kWaitIters = 1u << 22;
constexpr uint32_t kDrainWaitIters = 1u << 22;

// Device-side status words at the start of the workspace.
struct WorkspaceHeader {
    int32_t status;         // GDN_OK or GDN_ERR_TIMEOUT, written by kernels
    int32_t next_unit;      // dynamic work counter of the persistent kernel
    int32_t timeout_where;  // diagnostic: which wait gave up (or, range-checking build, which check failed)
    int32_t pad[61];        // header is 256 bytes
};
static_assert(sizeof(WorkspaceHeader) == 256, "workspace header is 256 bytes");

// Range checks of the debug build (compiled with -DGDN_DEBUG_BOUNDS, libgdn_dual_debug.so): a
// failed check records GDN_ERR_BOUNDS and its site in the workspace status words, and the access
// it guards is skipped.  In the normal build a check is `true` and its condition is not evaluated.
#ifdef GDN_DEBUG_BOUNDS
__device__ __forceinline__ bool bounds_ok(WorkspaceHeader *ws, bool ok, int where) {
    if (!ok) {
        atomicCAS(&ws->status, 0, (int)GDN_ERR_BOUNDS);
        atomicCAS(&ws->timeout_where, 0, where);
    }
    return ok;
}
#define GDN_IN_RANGE(ws, cond, where) ::gdn::bounds_ok((ws), (cond), (where))
#else
#define GDN_IN_RANGE(ws, cond, where) true
#endif

struct Params {
    const void *q, *k, *v;
    const float *g, *beta;
    const void *qn, *kn, *vn;
    const float *gn, *betan;
    const float *conv_w;
    void *out, *out_noisy;
    float *final_state;
    WorkspaceHeader *ws;
    void *states;           // Route I on tensor cores: the block-boundary state blobs (else NULL)
    int64_t T, TR;
    int32_t N, H, dk, dv, V, B, conv_width, num_units;
    int32_t parts;                    // chunked kernel: CTAs per unit (1, or 2 when units are few)
    float scale;                      // 1 / sqrt(d_k)
    uint32_t wait_iters;              // test entry point only: bound of the mbarrier waits, in polls
    uint32_t wait_test;               // 1: launch the kernels' test instantiation (polling waits)
    int32_t doc_start[kMaxDocs + 1];  // token offset of each document (doc_offsets)
    int32_t doc_prompt[kMaxDocs];     // prompt length of each document
    int32_t resp_off[kMaxDocs + 1];   // first packed noisy row of each document
    int32_t unit_doc[kMaxDocs];       // documents in scheduling order (longest first)
};

// Launchers (one per kernel family).  Return a CUDA error code; the caller maps it.
cudaError_t launch_sequential(const Params &p, int dtype, cudaStream_t stream);
// pipelined: the warp-specialised variant (no ShortConv), else the in-order kernel.
cudaError_t launch_chunked(const Params &p, bool pipelined, cudaStream_t stream);
// The warp-specialised pipelined variant of the chunked kernel (no ShortConv, at most two views).
cudaError_t launch_pipe(const Params &p, cudaStream_t stream);
// ShortConv as a pass of its own: the convolved bf16 q, k, v (T H d each, in that order) and
// their noisy twins (V T_R H d each) into `buf` (conv_pass_bytes of them).
size_t conv_pass_bytes(int64_t T, int64_t TR, int H, int d, int V);
cudaError_t launch_conv_pass(const Params &p, void *buf, cudaStream_t stream);
// Route I: clean chain writing block-boundary states into `states`, then block refinement.
cudaError_t launch_route1(const Params &p, int dtype, float *states, cudaStream_t stream);
bool chunked_supported(int dtype, int d, int B, int conv_width);
// Route I on tensor cores (gdn_route1_tc.cu): bf16, d = 128, B = 16 or 32, no ShortConv.  Stage 1
// is launch_chunked with P.states set and no views (the chunked kernel's EXPORT instantiation),
// stage 2 refines every (boundary state, pair of views) from P.states.
bool route1_tc_supported(int dtype, int d, int B, int conv_width);
cudaError_t launch_route1_refine(const Params &p, cudaStream_t stream);
// The backward on validated arguments, inputs and upstream gradients of element type `dtype`;
// the workspace must hold gdn_dual_backward_workspace_size() bytes for the descriptor.
gdn_status run_backward(const gdn_dual_desc *desc, int dtype, const void *q, const void *k, const void *v,
                        const float *g, const float *beta, const void *qn, const void *kn, const void *vn,
                        const float *gn, const float *betan, const int32_t *doc_offsets, const int32_t *prompt_len,
                        const void *d_out, const void *d_out_noisy, const float *d_final_state, float *dq,
                        float *dk, float *dv, float *dg, float *dbeta, float *dqn, float *dkn, float *dvn,
                        float *dgn, float *dbetan, void *workspace, cudaStream_t st);

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

}  // namespace gdn
