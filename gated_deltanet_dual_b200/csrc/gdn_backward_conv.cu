// gdn_backward_conv.cu -- backward of the dual-stream forward with the width-4 ShortConv prologue
// (gdn_dual_backward_conv in gdn_dual.h), on sm_100a CUDA cores.
//
// "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes), Method > Key design 3: a
// depthwise causal conv of width W = 4 on q, k and v (tap W-1 is the current token, the same
// weights for both streams); a noisy tap that reaches before its block's start reads the clean raw
// input, and no tap crosses a document start.  The conv is linear, so the backward is
//   1. the conv itself, into fp32 copies of the convolved q, k, v and their noisy twins;
//   2. the backward of the gated delta rule with respect to those inputs (gdn_backward.cu);
//   3. every tap's gradient sent back to its source -- the transposed taps, where a noisy output's
//      taps before its block start feed the clean raw input -- and to its weight.
// Step 3 gives each source element and each weight to one thread or one block, and every sum runs
// in a fixed order, so the results are the same on every call.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kW = 4;                  // conv width
constexpr int kCThreads = 256;

struct ConvParams {
    const void *x[3];                  // raw clean q, k, v          [T, H, d]
    const void *xn[3];                 // raw noisy q~, k~, v~       [V, T_R, H, d]
    const float *w;                    // [3, H d, 4]
    float *y[3], *yn[3];               // convolved (fp32) / their gradients
    float *dx[3], *dxn[3];             // gradients of the raw inputs (fp32 outputs)
    float *dw;                         // [3, H d, 4]
    int64_t T, TR;
    int32_t N, H, d, V, B;
    int32_t doc_start[kMaxDocs + 1];
    int32_t doc_prompt[kMaxDocs];
    int32_t resp_off[kMaxDocs + 1];
};

template <typename T>
__device__ __forceinline__ float ldx(const void *p, int64_t i) {
    return to_f32(static_cast<const T *>(p)[i]);
}

// document of clean token p (the last n with doc_start[n] <= p < doc_start[n + 1]), and of packed
// noisy row r (the same over resp_off)
__device__ __forceinline__ int doc_of(const int32_t *starts, int N, int64_t p) {
    int lo = 0, hi = N;                // starts[lo] <= p < starts[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (starts[mid] <= p) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Source of tap j (0 = the current token) of the noisy output at response index i of document n,
// view vw: the noisy row inside the block, the clean raw token before it, nothing before the
// document.  Returns 1 (noisy, *row = packed noisy row), 0 (clean, *row = token) or -1.
__device__ __forceinline__ int noisy_tap(const ConvParams &P, int n, int vw, int i, int j, int64_t *row) {
    const int s = P.doc_start[n], pr = P.doc_prompt[n];
    const int bs = (i / P.B) * P.B;    // block start (response index)
    const int src = i - j;
    if (src >= bs) {
        *row = (int64_t)vw * P.TR + P.resp_off[n] + src;
        return 1;
    }
    const int64_t tok = (int64_t)s + pr + src;
    if (tok < s) return -1;
    *row = tok;
    return 0;
}

// 1. the conv: clean rows [0, T), then noisy rows [0, V T_R); one thread per (row, head, channel),
//    all three tensors
template <typename TIO>
__global__ void __launch_bounds__(kCThreads) conv_fwd_kernel(const __grid_constant__ ConvParams P) {
    const int64_t hd = (int64_t)P.H * P.d;
    const int64_t total = (P.T + (int64_t)P.V * P.TR) * hd;
    for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < total;
         it += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = it / hd, e = it % hd;        // e = h d + c
        if (row < P.T) {
            const int n = doc_of(P.doc_start, P.N, row);
            const int64_t s = P.doc_start[n];
            for (int X = 0; X < 3; ++X) {
                const float *w = P.w + ((int64_t)X * hd + e) * kW;
                float acc = 0.f;
                for (int j = 0; j < kW; ++j)
                    if (row - j >= s) acc = fmaf(w[kW - 1 - j], ldx<TIO>(P.x[X], (row - j) * hd + e), acc);
                P.y[X][row * hd + e] = acc;
            }
        } else {
            const int64_t r = row - P.T;                  // packed noisy row
            const int vw = (int)(r / P.TR), rr = (int)(r % P.TR);
            const int n = doc_of(P.resp_off, P.N, rr);
            const int i = rr - P.resp_off[n];
            for (int X = 0; X < 3; ++X) {
                const float *w = P.w + ((int64_t)X * hd + e) * kW;
                float acc = 0.f;
                for (int j = 0; j < kW; ++j) {
                    int64_t src;
                    const int kind = noisy_tap(P, n, vw, i, j, &src);
                    if (kind < 0) continue;
                    const float xv = kind ? ldx<TIO>(P.xn[X], src * hd + e) : ldx<TIO>(P.x[X], src * hd + e);
                    acc = fmaf(w[kW - 1 - j], xv, acc);
                }
                P.yn[X][r * hd + e] = acc;
            }
        }
    }
}

// 3a. gradients of the raw inputs: one thread per (source row, head, channel), all three tensors.
//   clean token p:  sum_j w[3-j] dy_{p+j} over the clean outputs of its document, plus, for every view,
//                   w[3-j] dy~ of the noisy output at p+j (j >= 1) when p lies before that output's
//                   block start (the tap read the clean raw input);
//   noisy row:      sum_j w[3-j] dy~ of the outputs j later in the same block and view.
__global__ void __launch_bounds__(kCThreads) conv_bwd_kernel(const __grid_constant__ ConvParams P) {
    const int64_t hd = (int64_t)P.H * P.d;
    const int64_t total = (P.T + (int64_t)P.V * P.TR) * hd;
    for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < total;
         it += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = it / hd, e = it % hd;
        if (row < P.T) {
            const int n = doc_of(P.doc_start, P.N, row);
            const int64_t s = P.doc_start[n], end = P.doc_start[n + 1], rs = s + P.doc_prompt[n];
            for (int X = 0; X < 3; ++X) {
                const float *w = P.w + ((int64_t)X * hd + e) * kW;
                float acc = 0.f;
                for (int j = 0; j < kW; ++j)
                    if (row + j < end) acc = fmaf(w[kW - 1 - j], P.y[X][(row + j) * hd + e], acc);
                for (int j = 1; j < kW; ++j) {
                    const int64_t out = row + j;                     // a noisy output position
                    if (out < rs || out >= end) continue;
                    const int i = (int)(out - rs);
                    if (row >= rs + (i / P.B) * P.B) continue;        // inside the block: read the noisy row
                    for (int vw = 0; vw < P.V; ++vw)
                        acc = fmaf(w[kW - 1 - j], P.yn[X][((int64_t)vw * P.TR + P.resp_off[n] + i) * hd + e], acc);
                }
                P.dx[X][row * hd + e] = acc;
            }
        } else {
            const int64_t r = row - P.T;                  // the view's rows are consecutive
            const int rr = (int)(r % P.TR);
            const int n = doc_of(P.resp_off, P.N, rr);
            const int i = rr - P.resp_off[n];
            const int R = P.doc_start[n + 1] - P.doc_start[n] - P.doc_prompt[n];
            for (int X = 0; X < 3; ++X) {
                const float *w = P.w + ((int64_t)X * hd + e) * kW;
                float acc = 0.f;
                for (int j = 0; j < kW; ++j) {
                    const int io = i + j;
                    if (io < R && io / P.B == i / P.B)
                        acc = fmaf(w[kW - 1 - j], P.yn[X][(r + j) * hd + e], acc);
                }
                P.dxn[X][r * hd + e] = acc;
            }
        }
    }
}

// 3b. the weights: one block per (tensor X, channel e = h d + c); its threads stride over all
//    output rows (clean, then noisy) and sum source x gradient for each tap, then the block adds the
//    threads' sums in a fixed tree.
template <typename TIO>
__global__ void __launch_bounds__(kCThreads) conv_dw_kernel(const __grid_constant__ ConvParams P) {
    __shared__ float red[kW][kCThreads];
    const int64_t hd = (int64_t)P.H * P.d;
    const int X = (int)(blockIdx.x / hd);
    const int64_t e = blockIdx.x % hd;
    float acc[kW] = {0.f, 0.f, 0.f, 0.f};
    const int64_t rows = P.T + (int64_t)P.V * P.TR;
    for (int64_t row = threadIdx.x; row < rows; row += kCThreads) {
        if (row < P.T) {
            const int n = doc_of(P.doc_start, P.N, row);
            const int64_t s = P.doc_start[n];
            const float g = P.y[X][row * hd + e];
            for (int j = 0; j < kW; ++j)
                if (row - j >= s) acc[j] = fmaf(ldx<TIO>(P.x[X], (row - j) * hd + e), g, acc[j]);
        } else {
            const int64_t r = row - P.T;
            const int vw = (int)(r / P.TR), rr = (int)(r % P.TR);
            const int n = doc_of(P.resp_off, P.N, rr);
            const int i = rr - P.resp_off[n];
            const float g = P.yn[X][r * hd + e];
            for (int j = 0; j < kW; ++j) {
                int64_t src;
                const int kind = noisy_tap(P, n, vw, i, j, &src);
                if (kind < 0) continue;
                const float xv = kind ? ldx<TIO>(P.xn[X], src * hd + e) : ldx<TIO>(P.x[X], src * hd + e);
                acc[j] = fmaf(xv, g, acc[j]);
            }
        }
    }
    for (int j = 0; j < kW; ++j) red[j][threadIdx.x] = acc[j];
    __syncthreads();
    for (int step = kCThreads / 2; step > 0; step >>= 1) {
        if (threadIdx.x < step)
            for (int j = 0; j < kW; ++j) red[j][threadIdx.x] += red[j][threadIdx.x + step];
        __syncthreads();
    }
    if (threadIdx.x < kW) P.dw[((int64_t)X * hd + e) * kW + (kW - 1 - threadIdx.x)] = red[threadIdx.x][0];
}

template <typename TIO>
__global__ void to_f32_kernel(const void *src, float *dst, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = ldx<TIO>(src, i);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// fp32 buffers the conv path keeps after the inner backward's workspace: convolved inputs (3 clean,
// 3 noisy), fp32 upstream gradients (clean, noisy), gradients of the convolved inputs (3 + 3).  Noisy
// buffers are sized over V x T rows (T_R <= T: no prompt lengths needed).
int64_t conv_floats(const gdn_dual_desc *d, int64_t T) {
    const int64_t th = T * d->num_heads * d->d_k, V = d->num_views;
    return 3 * th + 3 * V * th + th + V * th + 3 * th + 3 * V * th;
}

int64_t grid_for(int64_t n) { return std::max<int64_t>(1, std::min<int64_t>((n + kCThreads - 1) / kCThreads, 148 * 32)); }

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" size_t gdn_dual_backward_conv_workspace_size(const gdn_dual_desc *desc, const int32_t *doc_offsets_host) {
    gdn_dual_desc inner = desc ? *desc : gdn_dual_desc{};
    inner.conv_width = 0;
    const size_t base = desc ? gdn_dual_backward_workspace_size(&inner, doc_offsets_host) : 0;
    if (base == 0) return 0;
    const size_t extra = (size_t)conv_floats(desc, doc_offsets_host[desc->num_docs]) * sizeof(float);
    return ((base + 255) / 256) * 256 + extra;
}

extern "C" gdn_status gdn_dual_backward_conv(const gdn_dual_desc *desc, const void *q, const void *k, const void *v,
                                             const float *g, const float *beta, const void *qn, const void *kn,
                                             const void *vn, const float *gn, const float *betan,
                                             const int32_t *doc_offsets, const int32_t *prompt_len,
                                             const float *conv_w, const void *d_out, const void *d_out_noisy,
                                             const float *d_final_state, float *dq, float *dk, float *dv, float *dg,
                                             float *dbeta, float *dqn, float *dkn, float *dvn, float *dgn,
                                             float *dbetan, float *dconv_w, void *workspace, size_t workspace_bytes,
                                             gdn_stream_t stream) {
    if (!desc || !doc_offsets || !prompt_len || doc_offsets[0] != 0) return GDN_ERR_INVALID_ARG;
    if (desc->num_docs < 1 || desc->num_heads < 1 || desc->d_k < 1 || desc->d_v < 1 || desc->num_views < 0 ||
        desc->block_size < 1 || (desc->dtype != GDN_BF16 && desc->dtype != GDN_FP32) || desc->reserved != 0)
        return GDN_ERR_INVALID_ARG;
    const int N = desc->num_docs, H = desc->num_heads, B = desc->block_size, D = desc->d_k;
    int64_t TR = 0;
    for (int n = 0; n < N; ++n) {
        const int64_t len = (int64_t)doc_offsets[n + 1] - doc_offsets[n];
        if (len < 0 || prompt_len[n] < 0 || prompt_len[n] > len || (len - prompt_len[n]) % B != 0)
            return GDN_ERR_INVALID_ARG;
        TR += len - prompt_len[n];
    }
    const int64_t T = doc_offsets[N];
    if (TR > INT32_MAX || T > INT32_MAX) return GDN_ERR_INVALID_ARG;
    const bool noisy = desc->num_views > 0 && TR > 0;
    if (T > 0 && (!q || !k || !v || !g || !beta || !d_out || !dq || !dk || !dv || !dg || !dbeta || !conv_w ||
                  !dconv_w))
        return GDN_ERR_INVALID_ARG;
    if (noisy && (!qn || !kn || !vn || !gn || !betan || !d_out_noisy || !dqn || !dkn || !dvn || !dgn || !dbetan))
        return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_dual_backward_conv_workspace_size(desc, doc_offsets);
    if (!workspace || workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, qn, kn, vn, gn, betan, conv_w, d_out, d_out_noisy, d_final_state,
                          dq, dk, dv, dg, dbeta, dqn, dkn, dvn, dgn, dbetan, dconv_w, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    if (desc->d_k != desc->d_v || (D != 32 && D != 64 && D != 128) || desc->conv_width != 4 || N > kMaxDocs)
        return GDN_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return cudaMemsetAsync(dconv_w, 0, (size_t)3 * H * D * kW * sizeof(float), st) == cudaSuccess
                           ? GDN_OK : GDN_ERR_CUDA;

    // workspace: the inner backward's, then the conv path's fp32 buffers
    gdn_dual_desc inner = *desc;
    inner.conv_width = 0;
    const size_t base = ((gdn_dual_backward_workspace_size(&inner, doc_offsets) + 255) / 256) * 256;
    float *f = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + base);
    const int64_t th = T * H * D, V = noisy ? desc->num_views : 0, nth = V * TR * H * D, vth = (int64_t)desc->num_views * th;
    ConvParams C;
    std::memset(&C, 0, sizeof(C));
    const void *xs[3] = {q, k, v}, *xns[3] = {qn, kn, vn};
    float *dxs[3] = {dq, dk, dv}, *dxns[3] = {dqn, dkn, dvn};
    for (int X = 0; X < 3; ++X) {
        C.x[X] = xs[X];
        C.xn[X] = xns[X];
        C.y[X] = f + X * th;                       // convolved clean
        C.yn[X] = f + 3 * th + X * vth;            // convolved noisy
        C.dx[X] = dxs[X];
        C.dxn[X] = dxns[X];
    }
    float *dout32 = f + 3 * th + 3 * vth, *doutn32 = dout32 + th;
    float *gy[3], *gyn[3];                         // gradients of the convolved inputs
    for (int X = 0; X < 3; ++X) {
        gy[X] = doutn32 + vth + X * th;
        gyn[X] = doutn32 + vth + 3 * th + X * vth;
    }
    C.w = conv_w;
    C.dw = dconv_w;
    C.T = T; C.TR = TR; C.N = N; C.H = H; C.d = D; C.V = (int32_t)V; C.B = B;
    int64_t roff = 0;
    for (int n = 0; n <= N; ++n) {
        C.doc_start[n] = doc_offsets[n];
        C.resp_off[n] = (int32_t)roff;
        if (n < N) {
            C.doc_prompt[n] = prompt_len[n];
            roff += (int64_t)doc_offsets[n + 1] - doc_offsets[n] - prompt_len[n];
        }
    }
    const bool bf = desc->dtype == GDN_BF16;
    const int64_t items = (T + V * TR) * H * D;
    // 1. the conv (fp32), and fp32 upstream gradients
    if (bf) conv_fwd_kernel<__nv_bfloat16><<<(unsigned)grid_for(items), kCThreads, 0, st>>>(C);
    else conv_fwd_kernel<float><<<(unsigned)grid_for(items), kCThreads, 0, st>>>(C);
    if (bf) {
        to_f32_kernel<__nv_bfloat16><<<(unsigned)grid_for(th), kCThreads, 0, st>>>(d_out, dout32, th);
        if (noisy) to_f32_kernel<__nv_bfloat16><<<(unsigned)grid_for(nth), kCThreads, 0, st>>>(d_out_noisy, doutn32, nth);
    } else {
        if (cudaMemcpyAsync(dout32, d_out, th * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return GDN_ERR_CUDA;
        if (noisy && cudaMemcpyAsync(doutn32, d_out_noisy, nth * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    // 2. the recurrence's backward with respect to the convolved inputs
    const gdn_status s2 = run_backward(&inner, GDN_FP32, C.y[0], C.y[1], C.y[2], g, beta, C.yn[0], C.yn[1], C.yn[2],
                                       gn, betan, doc_offsets, prompt_len, dout32, noisy ? doutn32 : nullptr,
                                       d_final_state, gy[0], gy[1], gy[2], dg, dbeta, gyn[0], gyn[1], gyn[2], dgn,
                                       dbetan, workspace, st);
    if (s2 != GDN_OK) return s2;
    // 3. back through the conv: sources and weights (C.y / C.yn now carry the gradients)
    for (int X = 0; X < 3; ++X) {
        C.y[X] = gy[X];
        C.yn[X] = gyn[X];
    }
    conv_bwd_kernel<<<(unsigned)grid_for(items), kCThreads, 0, st>>>(C);
    const unsigned wblocks = (unsigned)(3 * (int64_t)H * D);
    if (bf) conv_dw_kernel<__nv_bfloat16><<<wblocks, kCThreads, 0, st>>>(C);
    else conv_dw_kernel<float><<<wblocks, kCThreads, 0, st>>>(C);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
