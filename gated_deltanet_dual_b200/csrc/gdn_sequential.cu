// gdn_sequential.cu -- token-sequential dual-stream Gated DeltaNet forward on CUDA cores.
//
// One CTA per (document, head).  Thread t owns column j = t/2 of the d_k x d_v state and
// half of its rows (i in [ (t%2)*d/2, (t%2+1)*d/2 )), in fp32 registers, so k^T S and S^T q
// need only a pair shuffle.  This is the fp32-I/O path and the independent GPU cross-check of
// the chunked tensor-core kernel.
//
// Method ("FLARE: Diffusion for Hybrid Language Model", papernotes.org notes):
//   Key design 2: S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
//                 o_t = S_t^T q_t / sqrt(d_k); noisy block b restarts from S_{e(b-1)}, runs its
//                 B noisy tokens and every position reads the block-end state.
//   Key design 3: ShortConv taps (width 4) never cross the document start; noisy taps that
//                 reach before the block start read the clean raw input.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kTok = 16;   // clean tokens staged per tile
constexpr int kNTok = 8;   // noisy tokens staged per tile
constexpr int kW = 4;      // ShortConv width

template <typename TIO>
__device__ __forceinline__ float ld(const void *base, int64_t idx) {
    return to_f32(static_cast<const TIO *>(base)[idx]);
}

// Clean-stream value of channel c (of width dch) at document-local position p, with the
// causal ShortConv applied when conv is on (taps before the document start read 0).
template <typename TIO>
__device__ __forceinline__ float clean_in(const Params &P, const void *x, const float *w,
                                          int64_t doc_tok0, int p, int h, int c, int dch) {
    const int64_t rs = (int64_t)P.H * dch;
    const int64_t col = (int64_t)h * dch + c;
    if (!w) return ld<TIO>(x, (doc_tok0 + p) * rs + col);
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < kW; ++j) {
        const int src = p - j;
        if (src >= 0) acc = fmaf(w[col * kW + (kW - 1 - j)], ld<TIO>(x, (doc_tok0 + src) * rs + col), acc);
    }
    return acc;
}

// Noisy-stream value at document-local position p inside the block starting at blk
// (anti-leak rule: taps >= blk read noisy rows, taps in [0, blk) read clean raw rows).
template <typename TIO>
__device__ __forceinline__ float noisy_in(const Params &P, const void *x, const void *xn,
                                          const float *w, int64_t doc_tok0, int64_t nrow0,
                                          int prompt, int blk, int p, int h, int c, int dch) {
    const int64_t rs = (int64_t)P.H * dch;
    const int64_t col = (int64_t)h * dch + c;
    if (!w) return ld<TIO>(xn, (nrow0 + (p - prompt)) * rs + col);
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < kW; ++j) {
        const int src = p - j;
        float val;
        if (src >= blk) val = ld<TIO>(xn, (nrow0 + (src - prompt)) * rs + col);
        else if (src >= 0) val = ld<TIO>(x, (doc_tok0 + src) * rs + col);
        else val = 0.f;
        acc = fmaf(w[col * kW + (kW - 1 - j)], val, acc);
    }
    return acc;
}

template <typename TIO, int D>
__global__ void __launch_bounds__(2 * D)
gdn_sequential_kernel(const __grid_constant__ Params P) {
    constexpr int HALF = D / 2;
    const int tid = threadIdx.x;
    const int j = tid >> 1;           // state column (value dim)
    const int i0 = (tid & 1) * HALF;  // first state row (key dim) owned
    const int unit = blockIdx.x;
    const int n = unit / P.H, h = unit % P.H;
    const int64_t tok0 = P.doc_start[n];
    const int len = P.doc_start[n + 1] - P.doc_start[n];
    const int prompt = P.doc_prompt[n];
    const int B = P.B;
    const float scale = P.scale;
    const bool conv = P.conv_width > 0;
    const float *wq = conv ? P.conv_w : nullptr;
    const float *wk = conv ? P.conv_w + (int64_t)P.H * D * kW : nullptr;
    const float *wv = conv ? P.conv_w + 2 * (int64_t)P.H * D * kW : nullptr;
    const int64_t rs = (int64_t)P.H * D;   // row stride of q/k/v (d_k == d_v == D)

    __shared__ float sq[kTok][D], sk[kTok][D], sv[kTok][D], sg[kTok], sb[kTok];
    __shared__ float nq[kNTok][D], nk[kNTok][D], nv[kNTok][D], ng[kNTok], nb[kNTok];

    float S[HALF];
#pragma unroll
    for (int i = 0; i < HALF; ++i) S[i] = 0.f;

    for (int p0 = 0; p0 < len; p0 += kTok) {
        const int nt = min(kTok, len - p0);
        __syncthreads();
        for (int e = tid; e < nt * D; e += 2 * D) {
            const int t = e / D, c = e % D;
            sq[t][c] = clean_in<TIO>(P, P.q, wq, tok0, p0 + t, h, c, D);
            sk[t][c] = clean_in<TIO>(P, P.k, wk, tok0, p0 + t, h, c, D);
            sv[t][c] = clean_in<TIO>(P, P.v, wv, tok0, p0 + t, h, c, D);
        }
        for (int t = tid; t < nt; t += 2 * D) {
            sg[t] = P.g[(tok0 + p0 + t) * P.H + h];
            sb[t] = P.beta[(tok0 + p0 + t) * P.H + h];
        }
        __syncthreads();

        for (int t = 0; t < nt; ++t) {
            const int p = p0 + t;
            // ---- noisy stream: block starting at p reads S_{e(b-1)} = current S ----
            if (p >= prompt && ((p - prompt) % B) == 0 && P.V > 0) {
                const int blk = p;
                const int64_t nrow0 = P.resp_off[n];
                for (int view = 0; view < P.V; ++view) {
                    const int64_t vrow = (int64_t)view * P.TR + nrow0;   // this view's doc base row
                    const void *qn = P.qn, *kn = P.kn, *vn = P.vn;
                    float St[HALF];
#pragma unroll
                    for (int i = 0; i < HALF; ++i) St[i] = S[i];
                    // B steps of the rule on the noisy tokens
                    for (int l0 = 0; l0 < B; l0 += kNTok) {
                        const int nl = min(kNTok, B - l0);
                        __syncthreads();
                        for (int e = tid; e < nl * D; e += 2 * D) {
                            const int l = e / D, c = e % D;
                            nk[l][c] = noisy_in<TIO>(P, P.k, kn, wk, tok0, vrow, prompt, blk, blk + l0 + l, h, c, D);
                            nv[l][c] = noisy_in<TIO>(P, P.v, vn, wv, tok0, vrow, prompt, blk, blk + l0 + l, h, c, D);
                        }
                        for (int l = tid; l < nl; l += 2 * D) {
                            const int64_t r = vrow + (blk - prompt) + l0 + l;
                            ng[l] = P.gn[r * P.H + h];
                            nb[l] = P.betan[r * P.H + h];
                        }
                        __syncthreads();
                        for (int l = 0; l < nl; ++l) {
                            float u = 0.f;
#pragma unroll
                            for (int i = 0; i < HALF; ++i) u = fmaf(nk[l][i0 + i], St[i], u);
                            u += __shfl_xor_sync(0xffffffffu, u, 1);
                            const float a = expf(ng[l]);
                            const float bt = nb[l];
                            const float vj = nv[l][j];
#pragma unroll
                            for (int i = 0; i < HALF; ++i) {
                                // alpha (S - beta k u^T) + beta k v^T
                                const float ki = nk[l][i0 + i];
                                St[i] = a * (St[i] - bt * ki * u) + bt * ki * vj;
                            }
                        }
                    }
                    // every position of the block reads the block-end state
                    for (int l0 = 0; l0 < B; l0 += kNTok) {
                        const int nl = min(kNTok, B - l0);
                        __syncthreads();
                        for (int e = tid; e < nl * D; e += 2 * D) {
                            const int l = e / D, c = e % D;
                            nq[l][c] = noisy_in<TIO>(P, P.q, qn, wq, tok0, vrow, prompt, blk, blk + l0 + l, h, c, D);
                        }
                        __syncthreads();
                        for (int l = 0; l < nl; ++l) {
                            float o = 0.f;
#pragma unroll
                            for (int i = 0; i < HALF; ++i) o = fmaf(nq[l][i0 + i], St[i], o);
                            o += __shfl_xor_sync(0xffffffffu, o, 1);
                            if ((tid & 1) == 0) {
                                const int64_t r = vrow + (blk - prompt) + l0 + l;
                                static_cast<TIO *>(P.out_noisy)[r * rs + (int64_t)h * D + j] = from_f32<TIO>(o * scale);
                            }
                        }
                    }
                }
            }
            // ---- clean stream, token p ----
            float u = 0.f;
#pragma unroll
            for (int i = 0; i < HALF; ++i) u = fmaf(sk[t][i0 + i], S[i], u);
            u += __shfl_xor_sync(0xffffffffu, u, 1);
            const float a = expf(sg[t]);
            const float bt = sb[t];
            const float vj = sv[t][j];
            float o = 0.f;
#pragma unroll
            for (int i = 0; i < HALF; ++i) {
                const float ki = sk[t][i0 + i];
                S[i] = a * (S[i] - bt * ki * u) + bt * ki * vj;
                o = fmaf(sq[t][i0 + i], S[i], o);
            }
            o += __shfl_xor_sync(0xffffffffu, o, 1);
            if ((tid & 1) == 0)
                static_cast<TIO *>(P.out)[(tok0 + p) * rs + (int64_t)h * D + j] = from_f32<TIO>(o * scale);
        }
    }
    // final state [N, H, d_k, d_v]
    float *fs = P.final_state + ((int64_t)n * P.H + h) * D * D;
#pragma unroll
    for (int i = 0; i < HALF; ++i) fs[(int64_t)(i0 + i) * D + j] = S[i];
}

template <typename TIO, int D>
cudaError_t launch_d(const Params &p, cudaStream_t stream) {
    gdn_sequential_kernel<TIO, D><<<p.N * p.H, 2 * D, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sequential(const Params &p, int dtype, cudaStream_t stream) {
    if (p.N * p.H == 0) return cudaSuccess;
    const bool bf = dtype == GDN_BF16;
    switch (p.dk) {
        case 32: return bf ? launch_d<__nv_bfloat16, 32>(p, stream) : launch_d<float, 32>(p, stream);
        case 64: return bf ? launch_d<__nv_bfloat16, 64>(p, stream) : launch_d<float, 64>(p, stream);
        case 128: return bf ? launch_d<__nv_bfloat16, 128>(p, stream) : launch_d<float, 128>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
