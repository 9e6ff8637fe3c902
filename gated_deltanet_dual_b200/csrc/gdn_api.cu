// gdn_api.cu -- host side of the C ABI declared in include/gdn_dual.h: argument validation,
// per-call kernel parameters, algorithm selection and launch.  Validation happens entirely
// on the host before anything is enqueued; no allocation, no synchronisation on the forward
// path.
#include <algorithm>
#include <cmath>
#include <cstddef>
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
                        uint32_t wait_iters, gdn_stream_t stream, bool dry_run = false) {
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

    if (dry_run) return GDN_OK;          // validation only (the host-buffer entry point)

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
    } else if (route1_tc && !P.wait_test) {
        // (every eligible problem takes this path, views or not, so that the clean stream's
        // arithmetic never depends on how documents are batched)
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

// ---------------------------------------------------------------------------------------------
// gdn_dual_forward_host: the forward from and to HOST buffers.  The documents are cut into
// contiguous groups of about equal token counts; each group's inputs are copied into one of two
// device buffers of the caller's staging area (stream `in`), the group runs through the forward on
// the caller's stream, and its outputs are copied back (stream `out`).  With two buffers, group
// g+1's inputs and group g-1's outputs cross the host link while group g computes, so
// host-to-device and device-to-host traffic overlap (the link is full duplex).
namespace {

constexpr int kHostMaxGroups = 64;

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

struct HostPlan {
    int G = 0;
    int n0[kHostMaxGroups + 1];                  // group g = documents [n0[g], n0[g+1])
    std::vector<int64_t> roff;                   // response offset of each document, [N+1]
    // byte offsets inside one group buffer, and sizes
    size_t o_q, o_k, o_v, o_g, o_beta, o_qn, o_kn, o_vn, o_gn, o_betan, o_out, o_outn, o_fs, o_ws, ws_bytes, buf;
    size_t o_status, o_convw, o_buf0, o_buf1, total;
};

// The group's sub-problem: its documents' offsets from 0 and prompt lengths.
void sub_layout(const int32_t *offs, const int32_t *pl, int n0, int n1, std::vector<int32_t> &so,
                std::vector<int32_t> &sp) {
    so.assign(n1 - n0 + 1, 0);
    sp.assign(n1 - n0, 0);
    for (int n = n0; n <= n1; ++n) so[n - n0] = offs[n] - offs[n0];
    for (int n = n0; n < n1; ++n) sp[n - n0] = pl[n];
}

bool make_host_plan(const gdn_dual_desc *d, const int32_t *offs, const int32_t *pl, int groups, HostPlan &hp) {
    const int N = d->num_docs;
    const int64_t T = offs[N];
    hp.roff.assign(N + 1, 0);
    for (int n = 0; n < N; ++n) hp.roff[n + 1] = hp.roff[n] + (offs[n + 1] - offs[n]) - pl[n];
    const int G = std::max(1, std::min({groups, N, kHostMaxGroups}));
    hp.G = G;
    hp.n0[0] = 0;
    for (int g = 1; g < G; ++g) {        // first document at or past the g-th share of the tokens
        int n = hp.n0[g - 1] + 1;
        while (n < N - (G - g) && (int64_t)offs[n] * G < T * g) ++n;
        hp.n0[g] = n;
    }
    hp.n0[G] = N;
    int64_t mT = 0, mR = 0;
    int mN = 0;
    size_t mws = 0;
    std::vector<int32_t> so, sp;
    for (int g = 0; g < G; ++g) {
        const int a = hp.n0[g], b = hp.n0[g + 1];
        mT = std::max<int64_t>(mT, offs[b] - offs[a]);
        mR = std::max<int64_t>(mR, hp.roff[b] - hp.roff[a]);
        mN = std::max(mN, b - a);
        gdn_dual_desc sd = *d;
        sd.num_docs = b - a;
        sub_layout(offs, pl, a, b, so, sp);
        const size_t w = d->algo == GDN_ALGO_ROUTE1 ? gdn_dual_workspace_size_route1(&sd, so.data(), sp.data())
                                                    : gdn_dual_workspace_size(&sd, so.data());
        if (w == 0) return false;
        mws = std::max(mws, w);
    }
    const size_t es = d->dtype == GDN_BF16 ? 2 : 4, H = d->num_heads, V = d->num_views;
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o += up256(bytes); return at; };
    hp.o_q = take(mT * H * d->d_k * es);
    hp.o_k = take(mT * H * d->d_k * es);
    hp.o_v = take(mT * H * d->d_v * es);
    hp.o_g = take(mT * H * 4);
    hp.o_beta = take(mT * H * 4);
    hp.o_qn = take(V * mR * H * d->d_k * es);
    hp.o_kn = take(V * mR * H * d->d_k * es);
    hp.o_vn = take(V * mR * H * d->d_v * es);
    hp.o_gn = take(V * mR * H * 4);
    hp.o_betan = take(V * mR * H * 4);
    hp.o_out = take(mT * H * d->d_v * es);
    hp.o_outn = take(V * mR * H * d->d_v * es);
    hp.o_fs = take((size_t)mN * H * d->d_k * d->d_v * 4);
    hp.o_ws = take(mws);
    hp.ws_bytes = mws;
    hp.buf = o;
    hp.o_status = 0;                                    // [G] x {status, where} of each group
    hp.o_convw = up256(kHostMaxGroups * 2 * sizeof(int32_t));
    hp.o_buf0 = hp.o_convw + up256((size_t)3 * H * d->d_k * std::max(d->conv_width, 1) * 4);
    hp.o_buf1 = hp.o_buf0 + hp.buf;
    hp.total = hp.o_buf1 + hp.buf;
    return true;
}

bool host_layout_ok(const gdn_dual_desc *d, const int32_t *offs, const int32_t *pl) {
    if (!desc_ok(d) || !offs || !pl || offs[0] != 0) return false;
    for (int n = 0; n < d->num_docs; ++n) {
        const int64_t len = (int64_t)offs[n + 1] - offs[n];
        if (len < 0 || pl[n] < 0 || pl[n] > len || (len - pl[n]) % d->block_size != 0) return false;
    }
    return true;
}

}  // namespace

extern "C" {

size_t gdn_dual_host_staging_size(const gdn_dual_desc *desc, const int32_t *doc_offsets_host,
                                  const int32_t *prompt_len_host, int32_t groups) {
    if (!host_layout_ok(desc, doc_offsets_host, prompt_len_host) || groups < 1) return 0;
    HostPlan hp;
    if (!make_host_plan(desc, doc_offsets_host, prompt_len_host, groups, hp)) return 0;
    return hp.total;
}

gdn_status gdn_dual_forward_host(const gdn_dual_desc *desc,
                                 const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 const void *qn, const void *kn, const void *vn,
                                 const float *gn, const float *betan,
                                 const int32_t *doc_offsets, const int32_t *prompt_len,
                                 const float *conv_w,
                                 void *out, void *out_noisy, float *final_state,
                                 void *staging, size_t staging_bytes, int32_t groups,
                                 gdn_stream_t stream) {
    if (groups < 1 || !host_layout_ok(desc, doc_offsets, prompt_len)) return GDN_ERR_INVALID_ARG;
    HostPlan hp;
    if (!make_host_plan(desc, doc_offsets, prompt_len, groups, hp)) return GDN_ERR_INVALID_ARG;
    if (!staging || staging_bytes < hp.total || (reinterpret_cast<uintptr_t>(staging) & 255u))
        return GDN_ERR_INVALID_ARG;
    // the whole problem through the forward's own validation, on stand-in device pointers
    // (aligned, never dereferenced): nothing is enqueued unless it passes
    {
        const int N = desc->num_docs;
        const int64_t T = doc_offsets[N], TR = hp.roff[N];
        if ((T > 0 && (!q || !k || !v || !g || !beta || !out)) || !final_state) return GDN_ERR_INVALID_ARG;
        if (desc->num_views > 0 && TR > 0 && (!qn || !kn || !vn || !gn || !betan || !out_noisy))
            return GDN_ERR_INVALID_ARG;
        const void *s = staging;
        const gdn_status vs = forward_impl(desc, s, s, s, (const float *)s, (const float *)s, s, s, s,
                                           (const float *)s, (const float *)s, doc_offsets, prompt_len,
                                           desc->conv_width > 0 && conv_w ? (const float *)s : nullptr,
                                           const_cast<void *>(s), const_cast<void *>(s), (float *)s,
                                           const_cast<void *>(s), SIZE_MAX, gdn::kWaitIters, stream, true);
        if (vs != GDN_OK) return vs;
    }
    const int N = desc->num_docs, H = desc->num_heads, V = desc->num_views;
    const size_t es = desc->dtype == GDN_BF16 ? 2 : 4;
    const size_t rq = (size_t)H * desc->d_k * es, rv = (size_t)H * desc->d_v * es, rs = (size_t)H * 4;
    const int64_t TR = hp.roff[N];
    uint8_t *base = static_cast<uint8_t *>(staging);
    cudaStream_t user = reinterpret_cast<cudaStream_t>(stream), s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_in[2] = {nullptr, nullptr}, ev_comp[2] = {nullptr, nullptr},
                ev_out[2] = {nullptr, nullptr};
    gdn_status st = GDN_OK;
    auto ck = [&](cudaError_t e) {
        if (e != cudaSuccess && st == GDN_OK) st = GDN_ERR_CUDA;
        return st == GDN_OK;
    };
    ck(cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking));
    ck(cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking));
    for (cudaEvent_t *e : {&ev_start, &ev_in[0], &ev_in[1], &ev_comp[0], &ev_comp[1], &ev_out[0], &ev_out[1]})
        ck(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    if (st == GDN_OK) {
        ck(cudaEventRecord(ev_start, user));
        ck(cudaStreamWaitEvent(s_in, ev_start, 0));
        ck(cudaStreamWaitEvent(s_out, ev_start, 0));
        ck(cudaMemsetAsync(base + hp.o_status, 0, kHostMaxGroups * 2 * sizeof(int32_t), user));
        const float *dconv = nullptr;
        if (desc->conv_width > 0) {
            const size_t bytes = (size_t)3 * H * desc->d_k * desc->conv_width * 4;
            ck(cudaMemcpyAsync(base + hp.o_convw, conv_w, bytes, cudaMemcpyHostToDevice, s_in));
            dconv = reinterpret_cast<const float *>(base + hp.o_convw);
        }
        std::vector<int32_t> so, sp;
        for (int gi = 0; gi < hp.G && st == GDN_OK; ++gi) {
            const int b = gi & 1, a0 = hp.n0[gi], a1 = hp.n0[gi + 1];
            uint8_t *buf = base + (b ? hp.o_buf1 : hp.o_buf0);
            const int64_t t0 = doc_offsets[a0], Tg = doc_offsets[a1] - t0;
            const int64_t r0 = hp.roff[a0], Rg = hp.roff[a1] - r0;
            // inputs: the buffer is free once group gi-2's outputs have left
            if (gi >= 2) ck(cudaStreamWaitEvent(s_in, ev_out[b], 0));
            auto h2d = [&](size_t off, const void *src, size_t src_off, size_t bytes) {
                if (bytes) ck(cudaMemcpyAsync(buf + off, static_cast<const uint8_t *>(src) + src_off, bytes,
                                              cudaMemcpyHostToDevice, s_in));
            };
            h2d(hp.o_q, q, t0 * rq, Tg * rq);
            h2d(hp.o_k, k, t0 * rq, Tg * rq);
            h2d(hp.o_v, v, t0 * rv, Tg * rv);
            h2d(hp.o_g, g, t0 * rs, Tg * rs);
            h2d(hp.o_beta, beta, t0 * rs, Tg * rs);
            for (int w = 0; w < V && Rg > 0; ++w) {
                h2d(hp.o_qn + w * Rg * rq, qn, (w * TR + r0) * rq, Rg * rq);
                h2d(hp.o_kn + w * Rg * rq, kn, (w * TR + r0) * rq, Rg * rq);
                h2d(hp.o_vn + w * Rg * rv, vn, (w * TR + r0) * rv, Rg * rv);
                h2d(hp.o_gn + w * Rg * rs, gn, (w * TR + r0) * rs, Rg * rs);
                h2d(hp.o_betan + w * Rg * rs, betan, (w * TR + r0) * rs, Rg * rs);
            }
            ck(cudaEventRecord(ev_in[b], s_in));
            // the group's forward on the caller's stream, then its device status into slot gi
            ck(cudaStreamWaitEvent(user, ev_in[b], 0));
            gdn_dual_desc sd = *desc;
            sd.num_docs = a1 - a0;
            sub_layout(doc_offsets, prompt_len, a0, a1, so, sp);
            if (st == GDN_OK) {
                const gdn_status fs = forward_impl(
                    &sd, buf + hp.o_q, buf + hp.o_k, buf + hp.o_v, reinterpret_cast<const float *>(buf + hp.o_g),
                    reinterpret_cast<const float *>(buf + hp.o_beta), buf + hp.o_qn, buf + hp.o_kn, buf + hp.o_vn,
                    reinterpret_cast<const float *>(buf + hp.o_gn), reinterpret_cast<const float *>(buf + hp.o_betan),
                    so.data(), sp.data(), dconv, buf + hp.o_out, buf + hp.o_outn,
                    reinterpret_cast<float *>(buf + hp.o_fs), buf + hp.o_ws, hp.ws_bytes, gdn::kWaitIters, stream);
                if (fs != GDN_OK) st = fs;
            }
            ck(cudaMemcpyAsync(base + hp.o_status + gi * 2 * sizeof(int32_t), buf + hp.o_ws, sizeof(int32_t),
                               cudaMemcpyDeviceToDevice, user));
            ck(cudaMemcpyAsync(base + hp.o_status + (gi * 2 + 1) * sizeof(int32_t),
                               buf + hp.o_ws + offsetof(gdn::WorkspaceHeader, timeout_where), sizeof(int32_t),
                               cudaMemcpyDeviceToDevice, user));
            ck(cudaEventRecord(ev_comp[b], user));
            // outputs
            ck(cudaStreamWaitEvent(s_out, ev_comp[b], 0));
            auto d2h = [&](void *dst, size_t dst_off, size_t off, size_t bytes) {
                if (bytes) ck(cudaMemcpyAsync(static_cast<uint8_t *>(dst) + dst_off, buf + off, bytes,
                                              cudaMemcpyDeviceToHost, s_out));
            };
            d2h(out, t0 * rv, hp.o_out, Tg * rv);
            for (int w = 0; w < V && Rg > 0; ++w) d2h(out_noisy, (w * TR + r0) * rv, hp.o_outn + w * Rg * rv, Rg * rv);
            d2h(final_state, (size_t)a0 * H * desc->d_k * desc->d_v * 4, hp.o_fs,
                (size_t)(a1 - a0) * H * desc->d_k * desc->d_v * 4);
            ck(cudaEventRecord(ev_out[b], s_out));
        }
        // the caller's stream continues once every copy has landed
        for (int b = 0; b < 2; ++b)
            if (hp.G > b) ck(cudaStreamWaitEvent(user, ev_out[b], 0));
    }
    for (cudaEvent_t e : {ev_start, ev_in[0], ev_in[1], ev_comp[0], ev_comp[1], ev_out[0], ev_out[1]})
        if (e) cudaEventDestroy(e);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
    return st;
}

gdn_status gdn_dual_host_read_device_status(const void *staging, int32_t *where, gdn_stream_t stream) {
    if (!staging) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t words[kHostMaxGroups * 2];
    if (cudaMemcpyAsync(words, staging, sizeof(words), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GDN_ERR_CUDA;
    if (where) *where = 0;
    for (int i = 0; i < kHostMaxGroups; ++i)
        if (words[2 * i] != 0) {
            if (where) *where = words[2 * i + 1];
            return static_cast<gdn_status>(words[2 * i]);
        }
    return GDN_OK;
}

}  // extern "C"
