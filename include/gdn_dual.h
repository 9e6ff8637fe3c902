/*
 * gdn_dual.h -- C ABI of the B200 (sm_100a) dual-stream Gated DeltaNet forward.
 *
 * The operation is the forward pass of the two streams described in
 * "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes):
 *
 *   Method > Key design 2 -- clean causal stream, the gated delta rule
 *       S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  alpha_t = exp(g_t),
 *       o_t = S_t^T q_t / sqrt(d_k)                  (S is d_k x d_v, read after the update);
 *     and the block-bidirectional noisy stream: for every response block b of B tokens and
 *     every noisy view, S~ starts from the clean state S_{e(b-1)} just before the block, runs
 *     the same rule over the block's noisy tokens, and every position of the block reads the
 *     block-end state: o~_l = S~_{e(b)}^T q~_l / sqrt(d_k).  No per-block state is ever
 *     written to memory by this library.
 *   Method > Key design 3 -- optional width-4 depthwise causal ShortConv on q, k, v whose
 *     noisy taps that reach before the block start read the clean raw input; state reset and
 *     no tap across packed-document boundaries; document boundaries aligned to B.
 *   Method > Overall framework -- prompt tokens are causal context only; the response of
 *     each document is cut into blocks of B tokens; each block has complementary noisy views.
 *
 * Tensor layouts (row-major, contiguous, device memory owned by the caller):
 *   q, k         [T, H, d_k]        dtype = desc->dtype (bf16 or fp32)
 *   v            [T, H, d_v]
 *   g, beta      [T, H]             fp32 (g = log alpha, any real; beta any real)
 *   qn, kn       [V, T_R, H, d_k]   noisy twins, packed over RESPONSE tokens only,
 *   vn           [V, T_R, H, d_v]   documents in order (row r of doc n = its response token r)
 *   gn, betan    [V, T_R, H]        fp32
 *   conv_w       [3, H*d_k, 4]      fp32 weights for q, k, v channels; tap 3 is the current
 *                                   token: x'_p = sum_j w[c][3-j] x_{p-j}; NULL when conv is off
 *   out          [T, H, d_v]        dtype = desc->dtype
 *   out_noisy    [V, T_R, H, d_v]   dtype = desc->dtype
 *   final_state  [N, H, d_k, d_v]   fp32, the state after each document's last token
 * where T = doc_offsets[N] and T_R = sum_n (len_n - prompt_len[n]).
 *
 * Threading / ownership: the library allocates nothing and keeps no state between calls.
 * gdn_dual_forward only validates on the host, then enqueues work on `stream` and returns;
 * results are ready when the stream is.  Calls on different streams that share a workspace
 * race.  All functions are thread-safe.
 *
 * Errors: every entry point returns a gdn_status.  Bad arguments are rejected on the host
 * before anything is enqueued (no partial writes).  CUDA launch failures return
 * GDN_ERR_CUDA.  Device code never traps or asserts; bounded waits inside kernels record
 * GDN_ERR_TIMEOUT in the workspace (see gdn_dual_read_device_status); a kernel whose wait gave
 * up first waits for every copy and MMA it had issued, then leaves.
 */
#ifndef GDN_DUAL_H
#define GDN_DUAL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* inconsistent sizes, offsets, block alignment, NULL pointer */
    GDN_ERR_ALIGNMENT = 2,     /* a tensor pointer is not 16-byte aligned */
    GDN_ERR_UNSUPPORTED = 3,   /* valid but not implemented here (d, dtype, conv width, algo) */
    GDN_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    GDN_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up (reported by the device) */
    GDN_ERR_BOUNDS = 6         /* range-checking build only (libgdn_dual_debug.so, compiled with
                                  GDN_DEBUG_BOUNDS): a device-side index check failed and the
                                  access was skipped; the check's site is the `where` code of
                                  gdn_dual_read_device_status_where (201-209 chunked kernel,
                                  301-304 ShortConv pass) */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_FP32 = 1 } gdn_dtype;

typedef enum {
    GDN_ALGO_AUTO = 0,        /* the in-order chunked kernel when supported, else the sequential one */
    GDN_ALGO_SEQUENTIAL = 1,  /* token-sequential CUDA-core kernel, fp32 state (any dtype) */
    GDN_ALGO_CHUNKED = 2,     /* chunked WY/UT tcgen05 kernel, chunks in order (bf16,
                                 d_k = d_v = 128, B | 32, ShortConv off or width 4) */
    GDN_ALGO_ROUTE1 = 3,      /* chunk-then-refine (Route I of the notes, Key design 2), a measured
                                 comparison: a clean pass writes the state before every response
                                 block into the workspace, then each (view, block) is refined from
                                 its stored state.  bf16, d_k = d_v = 128, B in {16, 32}: tensor
                                 cores (the chunked kernel exports bf16 states from its intra-chunk
                                 products, then a tcgen05 refine kernel takes two views of a block
                                 per item; ShortConv as a pass of its own into the workspace
                                 first).  Otherwise CUDA cores (fp32 states), without ShortConv.
                                 Never chosen by AUTO */
    GDN_ALGO_PIPELINED = 4    /* the chunked WY/UT tcgen05 kernel pipelined across chunks: helper
                                 warps prepare chunk c+1's state-independent products (the
                                 triangular solve among them) while the main warps run chunk c's
                                 state chain (bf16, d_k = d_v = 128, B | 32, no ShortConv); a
                                 measured alternative, slower than GDN_ALGO_CHUNKED on B200, never
                                 chosen by AUTO */
} gdn_algo;

/* Problem descriptor.  num_docs N >= 1; num_heads H >= 1; d_k == d_v in {32, 64, 128};
 * num_views V in [0, 8]; block_size B >= 1 (the chunked kernel needs B | 32); dtype a
 * gdn_dtype; conv_width 0 (off) or 4; algo a gdn_algo; reserved must be 0. */
typedef struct {
    int32_t num_docs;
    int32_t num_heads;
    int32_t d_k;
    int32_t d_v;
    int32_t num_views;
    int32_t block_size;
    int32_t dtype;
    int32_t conv_width;
    int32_t algo;
    int32_t reserved;
} gdn_dual_desc;

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *gdn_stream_t;

/* Bytes of device workspace gdn_dual_forward wants for this problem (>= 256, a multiple of
 * 256).  doc_offsets_host: HOST array [N+1].  Returns 0 if the descriptor or offsets are
 * invalid.  Any workspace of at least 256 bytes is accepted; the size returned here also covers
 * the convolved inputs of a GDN_ALGO_AUTO call with ShortConv on the chunked path (bf16, 3 T H d
 * plus 3 V T H d elements): with that much, the conv runs as a pass of its own over every SM
 * before the chunked kernel; with less, inside the chunked kernel's prologue (same results up to
 * the accumulation order of the chunked products).  For GDN_ALGO_ROUTE1 it adds the materialised block-boundary states, T_R / B x H x
 * d_k x d_v fp32 (all documents' responses, T_R from doc_offsets and the prompt lengths); for
 * that algorithm prompt_len must be known, so use gdn_dual_workspace_size_route1. */
size_t gdn_dual_workspace_size(const gdn_dual_desc *desc, const int32_t *doc_offsets_host);

/* Workspace bytes for GDN_ALGO_ROUTE1: 256 + (T_R / B) * H * d_k * d_v * 4 (rounded up to 256),
 * where T_R is the total response length (doc_offsets_host [N+1] and prompt_len_host [N] are HOST
 * arrays); the tensor-core form stores its bf16 states in the first half of that.  With ShortConv
 * it adds the convolved inputs, 3 (T + V T_R) H d bf16 elements.  Returns 0 if the descriptor,
 * offsets or prompt lengths are invalid. */
size_t gdn_dual_workspace_size_route1(const gdn_dual_desc *desc, const int32_t *doc_offsets_host,
                                      const int32_t *prompt_len_host);

/*
 * Dual-stream GDN forward (Key design 2 and 3 of the FLARE notes; see the file comment).
 *   desc                 problem descriptor (host).
 *   q k v g beta         clean-stream inputs (device), layouts above.
 *   qn kn vn gn betan    noisy-stream inputs (device); may be NULL when V == 0 or T_R == 0.
 *   doc_offsets          HOST int32 [N+1]: doc_offsets[0] == 0, non-decreasing.  Document n
 *                        covers tokens [doc_offsets[n], doc_offsets[n+1]).
 *   prompt_len           HOST int32 [N]: 0 <= prompt_len[n] <= len_n and
 *                        (len_n - prompt_len[n]) % B == 0 (response aligned to B).
 *   conv_w               device fp32 [3, H*d_k, 4], or NULL when desc->conv_width == 0.
 *   out out_noisy final_state   outputs (device), fully overwritten.
 *   workspace            device scratch of at least gdn_dual_workspace_size() bytes,
 *                        16-byte aligned; contents on entry are ignored.
 *   stream               CUDA stream to enqueue on.
 * Every device pointer must be 16-byte aligned.
 */
gdn_status gdn_dual_forward(const gdn_dual_desc *desc,
                            const void *q, const void *k, const void *v,
                            const float *g, const float *beta,
                            const void *qn, const void *kn, const void *vn,
                            const float *gn, const float *betan,
                            const int32_t *doc_offsets, const int32_t *prompt_len,
                            const float *conv_w,
                            void *out, void *out_noisy, float *final_state,
                            void *workspace, size_t workspace_bytes,
                            gdn_stream_t stream);

/*
 * Backward pass of gdn_dual_forward (Method > Key design 2 of the FLARE notes: the noisy
 * blocks' gradients are injected into the causal chain).  Given the forward's inputs and the
 * upstream gradients d_out [T, H, d_v] and d_out_noisy [V, T_R, H, d_v] (dtype = desc->dtype)
 * and d_final_state [N, H, d_k, d_v] fp32 (NULL = zero), writes the gradients of
 *   L = <d_out, out> + <d_out_noisy, out_noisy> + <d_final_state, final_state>
 * with respect to every input, all fp32 in the inputs' layouts: dq dk dv [T, H, d], dg dbeta
 * [T, H], dqn dkn dvn [V, T_R, H, d], dgn dbetan [V, T_R, H] (fully overwritten; the noisy ones
 * may be NULL when there are no noisy rows).  The workspace holds the clean states at every
 * 16th token and the per-slice partial sums below: at least gdn_dual_backward_workspace_size()
 * bytes.  Host validation as for the forward; GDN_ERR_UNSUPPORTED for ShortConv (conv_width != 0:
 * use gdn_dual_backward_conv), d_k != d_v or d not in {32, 64, 128}.  CUDA-core kernel (one CTA
 * per (document, head, 32 state columns)); the column-summed gradients (dq, dk, dg, dbeta and
 * their noisy twins) are stored per 32-column slice and added in slice order by a second kernel,
 * so the results are the same on every call.
 */
size_t gdn_dual_backward_workspace_size(const gdn_dual_desc *desc, const int32_t *doc_offsets_host);
gdn_status gdn_dual_backward(const gdn_dual_desc *desc,
                             const void *q, const void *k, const void *v,
                             const float *g, const float *beta,
                             const void *qn, const void *kn, const void *vn,
                             const float *gn, const float *betan,
                             const int32_t *doc_offsets, const int32_t *prompt_len,
                             const void *d_out, const void *d_out_noisy, const float *d_final_state,
                             float *dq, float *dk, float *dv, float *dg, float *dbeta,
                             float *dqn, float *dkn, float *dvn, float *dgn, float *dbetan,
                             void *workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * Backward pass of gdn_dual_forward with the width-4 ShortConv prologue (desc->conv_width == 4;
 * Method > Key design 3 of the FLARE notes: depthwise causal conv of q, k, v, tap 3 = the current
 * token, the same weights for both streams, a noisy tap before its block start reads the clean raw
 * input, no tap across a document start).  Arguments as gdn_dual_backward, plus:
 *   conv_w    device fp32 [3, H*d_k, 4], the forward's weights;
 *   dconv_w   device fp32 [3, H*d_k, 4] output, the gradient of the weights.
 * dq dk dv (dqn dkn dvn) are the gradients of the RAW (unconvolved) inputs.  The workspace must
 * hold gdn_dual_backward_conv_workspace_size() bytes (the convolved inputs and their gradients in
 * fp32, besides the backward's own checkpoints).  Every sum runs in a fixed order, so the results
 * are the same on every call.  GDN_ERR_UNSUPPORTED unless conv_width == 4, d_k == d_v in
 * {32, 64, 128}.  CUDA cores: the conv, the backward of the recurrence on the convolved fp32
 * inputs, then the transposed taps and the weight sums.
 */
size_t gdn_dual_backward_conv_workspace_size(const gdn_dual_desc *desc, const int32_t *doc_offsets_host);
gdn_status gdn_dual_backward_conv(const gdn_dual_desc *desc,
                                  const void *q, const void *k, const void *v,
                                  const float *g, const float *beta,
                                  const void *qn, const void *kn, const void *vn,
                                  const float *gn, const float *betan,
                                  const int32_t *doc_offsets, const int32_t *prompt_len,
                                  const float *conv_w,
                                  const void *d_out, const void *d_out_noisy, const float *d_final_state,
                                  float *dq, float *dk, float *dv, float *dg, float *dbeta,
                                  float *dqn, float *dkn, float *dvn, float *dgn, float *dbetan,
                                  float *dconv_w, void *workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_dual_forward without a workspace argument, for callers that cannot allocate device
 * memory: e.g. an engine that reserved all device memory for its own pool up front, or a
 * plugin/FFI host with no device allocator reachable through the C ABI.  (The FLARE notes have
 * no counterpart; this is an interface convenience.)  Same inputs, outputs, layouts, stream
 * semantics and host validation as gdn_dual_forward.
 *   Scratch: a fixed 4096-byte array in the library's own device memory (a file-scope
 *     __device__ array; every GPU that loads the library holds it until the process exits).
 *     The kernels need 256 bytes of it; with ShortConv the conv runs in the chunked kernel's
 *     prologue (the separate conv pass needs room for the convolved inputs, which the array does
 *     not have).
 *   Allocation: none, on any call (no cudaMalloc or cudaFree).
 *   Set-up: the first call on a device, with that device current, looks up the array's device
 *     address (cudaGetSymbolAddress); make that first call before any stream capture.
 *   Sharing: all calls on a device share the array, which keeps the last call's contents; the
 *     status words are cleared on `stream` at the start of every call.  Calls whose work
 *     overlaps on the GPU (e.g. on two streams at once) race on the array: serialise them.
 *     The address is kept per device ordinal for the life of the process, so it belongs to the
 *     device's primary context (the CUDA runtime's); do not call this from another context, or
 *     after cudaDeviceReset.
 *   Errors: as gdn_dual_forward, plus GDN_ERR_CUDA if the set-up lookup fails, and
 *     GDN_ERR_UNSUPPORTED for GDN_ALGO_ROUTE1 (its block-boundary states need far more scratch
 *     than the array holds).  A bounded device-side wait that gives up is recorded in the array,
 *     not returned here: read it with gdn_dual_noalloc_read_device_status.
 */
gdn_status gdn_dual_forward_noalloc(const gdn_dual_desc *desc,
                                    const void *q, const void *k, const void *v,
                                    const float *g, const float *beta,
                                    const void *qn, const void *kn, const void *vn,
                                    const float *gn, const float *betan,
                                    const int32_t *doc_offsets, const int32_t *prompt_len,
                                    const float *conv_w,
                                    void *out, void *out_noisy, float *final_state,
                                    gdn_stream_t stream);

/* The device-side status recorded by the last gdn_dual_forward_noalloc on the current device
 * (GDN_OK or GDN_ERR_TIMEOUT): synchronises `stream` and reads the status word at the start of
 * the library's fixed scratch array.  No allocation.  (The FLARE notes have no counterpart.) */
gdn_status gdn_dual_noalloc_read_device_status(gdn_stream_t stream);

/*
 * gdn_dual_forward from and to HOST buffers (same descriptor, layouts and results as
 * gdn_dual_forward; every tensor argument is a host pointer, pinned for the copies to run
 * asynchronously).  The documents are cut into `groups` contiguous groups of about equal token
 * counts (at most min(groups, N, 64)); each group's inputs are copied into one of two device
 * buffers inside `staging`, the group's forward runs on `stream`, and its outputs are copied
 * back, on two streams of the call's own, so that one group's outputs travel to the host while the
 * next group's inputs travel to the device.  Stream-ordered: it starts after the work already on
 * `stream`, and `stream` reaches the outputs in host memory only after every copy has landed
 * (synchronise `stream` before reading them).  Not capturable in a CUDA graph (it creates its two
 * copy streams and destroys them when the work is done).
 *   staging        DEVICE memory of at least gdn_dual_host_staging_size() bytes, 256-byte aligned.
 *   Errors: the whole problem is validated on the host as gdn_dual_forward validates it before
 *   anything is enqueued; GDN_ERR_INVALID_ARG also for groups < 1 or a staging area that is too
 *   small; GDN_ERR_CUDA if a copy or launch fails (work already enqueued then still runs).
 * Device-side status: gdn_dual_host_read_device_status.  (The FLARE notes have no counterpart:
 * this is the library's host interface.) */
size_t gdn_dual_host_staging_size(const gdn_dual_desc *desc, const int32_t *doc_offsets_host,
                                  const int32_t *prompt_len_host, int32_t groups);

gdn_status gdn_dual_forward_host(const gdn_dual_desc *desc,
                                 const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 const void *qn, const void *kn, const void *vn,
                                 const float *gn, const float *betan,
                                 const int32_t *doc_offsets, const int32_t *prompt_len,
                                 const float *conv_w,
                                 void *out, void *out_noisy, float *final_state,
                                 void *staging, size_t staging_bytes, int32_t groups,
                                 gdn_stream_t stream);

/* Synchronises `stream` and returns the first non-OK device-side status that the groups of the
 * last gdn_dual_forward_host on `staging` recorded (GDN_OK or GDN_ERR_TIMEOUT), storing the
 * diagnostic code of the wait that gave up in `where` when it is not NULL. */
gdn_status gdn_dual_host_read_device_status(const void *staging, int32_t *where, gdn_stream_t stream);

/* Synchronises `stream` and returns the device-side status recorded in `workspace` by the
 * last gdn_dual_forward on it (GDN_OK or GDN_ERR_TIMEOUT), or GDN_ERR_CUDA if the sync fails.
 * For debugging and tests; the forward path itself never synchronises. */
gdn_status gdn_dual_read_device_status(const void *workspace, gdn_stream_t stream);

/* As gdn_dual_read_device_status, and, when `where` is not NULL, stores the diagnostic code of
 * the wait that gave up (0 when none did). */
gdn_status gdn_dual_read_device_status_where(const void *workspace, int32_t *where, gdn_stream_t stream);

/* FOR TESTS of the bounded-wait error path only: gdn_dual_forward with every device-side
 * mbarrier wait bounded by `wait_iters` non-blocking polls (>= 1) instead of the library's
 * normal bound.  A tiny bound makes a wait give up while its copy or MMA is still in flight: the
 * kernel then records GDN_ERR_TIMEOUT (and where) in the workspace, waits with the normal bound
 * for every copy and MMA it has issued, and leaves; outputs are unspecified.  The next ordinary
 * call is unaffected.  The tensor-core kernels have this test variant for B = 4 only (other block
 * sizes on them: GDN_ERR_UNSUPPORTED).  (The FLARE notes have no counterpart: this exercises the failure
 * detection of this library.) */
gdn_status gdn_dual_forward_test_wait_limit(const gdn_dual_desc *desc,
                                            const void *q, const void *k, const void *v,
                                            const float *g, const float *beta,
                                            const void *qn, const void *kn, const void *vn,
                                            const float *gn, const float *betan,
                                            const int32_t *doc_offsets, const int32_t *prompt_len,
                                            const float *conv_w,
                                            void *out, void *out_noisy, float *final_state,
                                            void *workspace, size_t workspace_bytes,
                                            uint32_t wait_iters, gdn_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
const char *gdn_status_string(gdn_status status);

/* Library version as 10000*major + 100*minor + patch. */
int32_t gdn_dual_version(void);

/* Which algorithm GDN_ALGO_AUTO selects for this descriptor (a gdn_algo value), or -1 if the
 * descriptor is invalid.  Host only. */
int32_t gdn_dual_select_algo(const gdn_dual_desc *desc);

#ifdef __cplusplus
}
#endif

#endif /* GDN_DUAL_H */
