// gdn_api.cu -- host side of the C ABI declared in include/gdn_dual.h: argument validation,
// per-call kernel parameters, algorithm selection and launch.  Validation happens entirely
// on the host before anything is enqueued; no allocation, no synchronisation on the forward
// path.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

#include "gdn_internal.cuh"

namespace {

constexpr int32_t kVersion = 100;   // 0.1.0

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool desc_ok(const gdn_dual_desc *d) {
    if (!d) return false;
    if (d->num_docs < 1 || d->num_heads < 1) return false;
    if (d->d_k < 1 || d->d_v < 1) return false;
    if (d->num_views < 0 || d->num_views > 8) return false;
    if (d->block_size < 1) return false;
    if (d->dtype != GDN_BF16 && d->dtype != GDN_FP32) return false;
    if (d->conv_width < 0) return false;
    if (d->algo < GDN_ALGO_AUTO || d->algo > GDN_ALGO_PIPELINED) return false;
    if (d->reserved != 0) return false;
    return true;
}

bool desc_supported(const gdn_dual_desc *d) {
    if (d->d_k != d->d_v) return false;
    if (d->d_k != 32 && d->d_k != 64 && d->d_k != 128) return false;
    if (d->conv_width != 0 && d->conv_width != 4) return false;
    if (d->num_docs > gdn::kMaxDocs) return false;
    return true;
}

// GDN_ALGO_ROUTE1 on tensor cores (else the CUDA-core form)
bool route1_tc_form(const gdn_dual_desc *d) {
    return d->d_k == d->d_v && gdn::route1_tc_supported(d->dtype, d->d_k, d->block_size, d->conv_width);
}

// AUTO with ShortConv on the chunked path runs the conv as a pass of its own (into the workspace)
// when the workspace has room for the convolved inputs; else the chunked kernel's fused prologue.
bool conv_pass_wanted(const gdn_dual_desc *d) {
    return d->algo == GDN_ALGO_AUTO && d->conv_width == 4 &&
           gdn::chunked_supported(d->dtype, d->d_k, d->block_size, d->conv_width) && d->d_k == d->d_v;
}

int select_algo(const gdn_dual_desc *d) {
    if (d->algo != GDN_ALGO_AUTO) return d->algo;
    return gdn::chunked_supported(d->dtype, d->d_k, d->block_size, d->conv_width) ? GDN_ALGO_CHUNKED
                                                                                  : GDN_ALGO_SEQUENTIAL;
}

}  // namespace

extern "C" {

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_ALIGNMENT: return "GDN_ERR_ALIGNMENT";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_BOUNDS: return "GDN_ERR_BOUNDS";
    }
    return "GDN_ERR_UNKNOWN";
}

int32_t gdn_dual_version(void) { return kVersion; }

int32_t gdn_dual_select_algo(const gdn_dual_desc *desc) {
    if (!desc_ok(desc)) return -1;
    return select_algo(desc);
}

size_t gdn_dual_workspace_size(const gdn_dual_desc *desc, const int32_t *doc_offsets_host) {
    if (!desc_ok(desc) || !doc_offsets_host) return 0;
    if (doc_offsets_host[0] != 0) return 0;
    for (int n = 0; n < desc->num_docs; ++n)
        if (doc_offsets_host[n + 1] < doc_offsets_host[n]) return 0;
    if (desc->algo == GDN_ALGO_ROUTE1) return 0;   // needs the prompt lengths: the _route1 variant
    if (conv_pass_wanted(desc)) {                  // room for the convolved inputs (T_R <= T)
        const int64_t T = doc_offsets_host[desc->num_docs];
        return sizeof(gdn::WorkspaceHeader) +
               gdn::conv_pass_bytes(T, T, desc->num_heads, desc->d_k, desc->num_views);
    }
    return sizeof(gdn::WorkspaceHeader);
}

size_t gdn_dual_workspace_size_route1(const gdn_dual_desc *desc, const int32_t *doc_offsets_host,
                                      const int32_t *prompt_len_host) {
    if (!desc_ok(desc) || !doc_offsets_host || !prompt_len_host) return 0;
    if (doc_offsets_host[0] != 0) return 0;
    int64_t TR = 0;
    for (int n = 0; n < desc->num_docs; ++n) {
        const int64_t len = (int64_t)doc_offsets_host[n + 1] - doc_offsets_host[n];
        if (len < 0 || prompt_len_host[n] < 0 || prompt_len_host[n] > len) return 0;
        if ((len - prompt_len_host[n]) % desc->block_size != 0) return 0;
        TR += len - prompt_len_host[n];
    }
    const size_t states = (size_t)(TR / desc->block_size) * desc->num_heads * desc->d_k * desc->d_v * sizeof(float);
    size_t bytes = sizeof(gdn::WorkspaceHeader) + ((states + 255) / 256) * 256;
    if (desc->conv_width > 0 && route1_tc_form(desc))   // its conv pass: the convolved copies follow the states
        bytes += gdn::conv_pass_bytes(doc_offsets_host[desc->num_docs], TR, desc->num_heads, desc->d_k,
                                      desc->num_views);
    return bytes;
}

}  // extern "C"

namespace {

gdn_status forward_impl(const gdn_dual_desc *desc,
                        const void *q, const void *k, const void *v,
                        const float *g, const float *beta,
                        const void *qn, const void *kn, const void *vn,
                        const float *gn, const float *betan,
                        const int32_t *doc_offsets, const int32_t *prompt_len,
                        const float *conv_w,
                        void *out, void *out_noisy, float *final_state,
                        void *workspace, size_t workspace_bytes,
                        uint32_t wait_iters, gdn_stream_t stream) {
    if (!desc_ok(desc) || !doc_offsets || !prompt_len) return GDN_ERR_INVALID_ARG;
    const int N = desc->num_docs, H = desc->num_heads, B = desc->block_size, V = desc->num_views;
    // documents: offsets monotone from 0, prompt within the document, response aligned to B
    if (doc_offsets[0] != 0) return GDN_ERR_INVALID_ARG;
    int64_t TR = 0;
    for (int n = 0; n < N; ++n) {
        const int64_t len = (int64_t)doc_offsets[n + 1] - doc_offsets[n];
        if (len < 0) return GDN_ERR_INVALID_ARG;
        if (prompt_len[n] < 0 || prompt_len[n] > len) return GDN_ERR_INVALID_ARG;
        if ((len - prompt_len[n]) % B != 0) return GDN_ERR_INVALID_ARG;
        TR += len - prompt_len[n];
    }
    const int64_t T = doc_offsets[N];
    if (TR > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (desc->conv_width > 0 && !conv_w) return GDN_ERR_INVALID_ARG;
    // pointers: required ones non-NULL, all 16-byte aligned
    if (!final_state) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_INVALID_ARG;
    const bool noisy = V > 0 && TR > 0;
    if (noisy && (!qn || !kn || !vn || !gn || !betan || !out_noisy)) return GDN_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < sizeof(gdn::WorkspaceHeader)) return GDN_ERR_INVALID_ARG;
    const size_t route1_states = (((size_t)(TR / B) * H * desc->d_k * desc->d_v * sizeof(float) + 255) / 256) * 256;
    const size_t route1_conv =
        desc->conv_width > 0 && route1_tc_form(desc) ? gdn::conv_pass_bytes(T, TR, H, desc->d_k, V) : 0;
    if (desc->algo == GDN_ALGO_ROUTE1 && workspace_bytes < sizeof(gdn::WorkspaceHeader) + route1_states + route1_conv)
        return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, qn, kn, vn, gn, betan, conv_w, out, out_noisy, final_state, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    if (!desc_supported(desc)) return GDN_ERR_UNSUPPORTED;
    const int algo = select_algo(desc);
    if ((algo == GDN_ALGO_CHUNKED || algo == GDN_ALGO_PIPELINED) &&
        !gdn::chunked_supported(desc->dtype, desc->d_k, B, desc->conv_width))
        return GDN_ERR_UNSUPPORTED;
    if (algo == GDN_ALGO_PIPELINED && desc->conv_width != 0) return GDN_ERR_UNSUPPORTED;
    // Route I: tensor cores for bf16, d = 128, B in {16, 32} (ShortConv through the conv pass);
    // otherwise CUDA cores, without ShortConv
    const bool route1_tc = algo == GDN_ALGO_ROUTE1 && route1_tc_form(desc);
    if (algo == GDN_ALGO_ROUTE1 && (B > 64 || (desc->conv_width != 0 && (!route1_tc || wait_iters < gdn::kWaitIters))))
        return GDN_ERR_UNSUPPORTED;

    gdn::Params P;
    std::memset(&P, 0, sizeof(P));
    P.q = q; P.k = k; P.v = v; P.g = g; P.beta = beta;
    P.qn = qn; P.kn = kn; P.vn = vn; P.gn = gn; P.betan = betan;
    P.conv_w = desc->conv_width > 0 ? conv_w : nullptr;
    P.out = out; P.out_noisy = out_noisy; P.final_state = final_state;
    P.ws = static_cast<gdn::WorkspaceHeader *>(workspace);
    P.T = T; P.TR = TR;
    P.N = N; P.H = H; P.dk = desc->d_k; P.dv = desc->d_v; P.V = noisy ? V : 0; P.B = B;
    P.conv_width = desc->conv_width;
    P.num_units = N * H;
    P.parts = 1;
    P.scale = (float)(1.0 / std::sqrt((double)desc->d_k));
    P.wait_iters = wait_iters;
    P.wait_test = wait_iters < gdn::kWaitIters ? 1u : 0u;
    int64_t roff = 0;
    for (int n = 0; n <= N; ++n) {
        P.doc_start[n] = doc_offsets[n];
        P.resp_off[n] = (int32_t)roff;
        if (n < N) {
            P.doc_prompt[n] = prompt_len[n];
            roff += (int64_t)doc_offsets[n + 1] - doc_offsets[n] - prompt_len[n];
        }
    }
    // longest documents first, so a dynamic scheduler finishes the long chains early
    std::vector<int32_t> order(N);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
        return doc_offsets[a + 1] - doc_offsets[a] > doc_offsets[b + 1] - doc_offsets[b];
    });
    std::copy(order.begin(), order.end(), P.unit_doc);

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, sizeof(gdn::WorkspaceHeader), st) != cudaSuccess) return GDN_ERR_CUDA;
    cudaError_t err;
    const size_t pass_bytes = gdn::conv_pass_bytes(T, TR, H, desc->d_k, P.V);
    if (algo == GDN_ALGO_CHUNKED && conv_pass_wanted(desc) && !P.wait_test &&
        workspace_bytes >= sizeof(gdn::WorkspaceHeader) + pass_bytes) {
        // the conv pass, then the chunked kernel without its prologue on the convolved inputs
        uint8_t *buf = static_cast<uint8_t *>(workspace) + sizeof(gdn::WorkspaceHeader);
        err = gdn::launch_conv_pass(P, buf, st);
        if (err == cudaSuccess) {
            const int64_t clean = T * H * desc->d_k, nz = (int64_t)P.V * TR * H * desc->d_k;
            const __nv_bfloat16 *y = reinterpret_cast<const __nv_bfloat16 *>(buf);
            gdn::Params Q = P;
            Q.q = y; Q.k = y + clean; Q.v = y + 2 * clean;
            Q.qn = y + 3 * clean; Q.kn = y + 3 * clean + nz; Q.vn = y + 3 * clean + 2 * nz;
            Q.conv_width = 0;
            Q.conv_w = nullptr;
            err = gdn::launch_chunked(Q, false, st);
        }
    } else if (algo == GDN_ALGO_CHUNKED || algo == GDN_ALGO_PIPELINED) {
        err = gdn::launch_chunked(P, algo == GDN_ALGO_PIPELINED, st);
    } else if (route1_tc && (P.V > 0 || desc->conv_width > 0) && !P.wait_test) {
        // Route I on tensor cores: the clean stream exporting the state before every response
        // block (bf16 blobs of 32 KB, in the space the fp32 states take otherwise), then the refine
        // kernel over every (block, head, pair of views).  With ShortConv, the conv pass first
        // writes the convolved inputs after the states, and both stages read those.
        gdn::Params Q = P;
        Q.states = static_cast<uint8_t *>(workspace) + sizeof(gdn::WorkspaceHeader);
        err = cudaSuccess;
        if (desc->conv_width > 0) {
            uint8_t *buf = static_cast<uint8_t *>(workspace) + sizeof(gdn::WorkspaceHeader) + route1_states;
            err = gdn::launch_conv_pass(P, buf, st);
            const int64_t clean = T * H * desc->d_k, nz = (int64_t)P.V * TR * H * desc->d_k;
            const __nv_bfloat16 *y = reinterpret_cast<const __nv_bfloat16 *>(buf);
            Q.q = y; Q.k = y + clean; Q.v = y + 2 * clean;
            Q.qn = y + 3 * clean; Q.kn = y + 3 * clean + nz; Q.vn = y + 3 * clean + 2 * nz;
            Q.conv_width = 0;
            Q.conv_w = nullptr;
        }
        Q.V = 0;
        if (err == cudaSuccess) err = gdn::launch_chunked(Q, false, st);
        if (err == cudaSuccess) {
            cudaMemsetAsync(&static_cast<gdn::WorkspaceHeader *>(workspace)->next_unit, 0, sizeof(int32_t), st);
            Q.V = P.V;
            err = gdn::launch_route1_refine(Q, st);
        }
    } else if (algo == GDN_ALGO_ROUTE1) {
        err = gdn::launch_route1(P, desc->dtype,
                                 reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + sizeof(gdn::WorkspaceHeader)), st);
    } else {
        err = gdn::launch_sequential(P, desc->dtype, st);
    }
    if (err == cudaErrorNotSupported) return GDN_ERR_UNSUPPORTED;
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

extern "C" {

gdn_status gdn_dual_forward(const gdn_dual_desc *desc,
                            const void *q, const void *k, const void *v,
                            const float *g, const float *beta,
                            const void *qn, const void *kn, const void *vn,
                            const float *gn, const float *betan,
                            const int32_t *doc_offsets, const int32_t *prompt_len,
                            const float *conv_w,
                            void *out, void *out_noisy, float *final_state,
                            void *workspace, size_t workspace_bytes,
                            gdn_stream_t stream) {
    return forward_impl(desc, q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, conv_w, out,
                        out_noisy, final_state, workspace, workspace_bytes, gdn::kWaitIters, stream);
}

gdn_status gdn_dual_forward_test_wait_limit(const gdn_dual_desc *desc,
                                            const void *q, const void *k, const void *v,
                                            const float *g, const float *beta,
                                            const void *qn, const void *kn, const void *vn,
                                            const float *gn, const float *betan,
                                            const int32_t *doc_offsets, const int32_t *prompt_len,
                                            const float *conv_w,
                                            void *out, void *out_noisy, float *final_state,
                                            void *workspace, size_t workspace_bytes,
                                            uint32_t wait_iters, gdn_stream_t stream) {
    if (wait_iters < 1) return GDN_ERR_INVALID_ARG;
    return forward_impl(desc, q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, conv_w, out,
                        out_noisy, final_state, workspace, workspace_bytes, wait_iters, stream);
}

gdn_status gdn_dual_read_device_status(const void *workspace, gdn_stream_t stream) {
    return gdn_dual_read_device_status_where(workspace, nullptr, stream);
}

gdn_status gdn_dual_read_device_status_where(const void *workspace, int32_t *where, gdn_stream_t stream) {
    if (!workspace) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    gdn::WorkspaceHeader h;
    if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GDN_ERR_CUDA;
    if (where) *where = h.timeout_where;
    return h.status == 0 ? GDN_OK : static_cast<gdn_status>(h.status);
}

}  // extern "C"
