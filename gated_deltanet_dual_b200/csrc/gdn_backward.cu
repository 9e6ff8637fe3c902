// gdn_backward.cu -- backward pass of the dual-stream Gated DeltaNet forward on CUDA cores
// (sm_100a), and its C ABI (gdn_dual_backward in gdn_dual.h).
//
// "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes), Method > Key design 2:
// the backward injects every noisy block's gradient into the causal chain.  With
// Lam_t = dL/dS_t (L = <do, out> + <do~, out_noisy> + <dS, final_state>):
//   Lam_t  = q_t do_t^T / sqrt(d) + A_{t+1}^T Lam_{t+1} + sum_views Lam~_0 of the block starting at t+1,
//   Lam~_B = sum_l q~_l do~_l^T / sqrt(d),  Lam~_{i-1} = A~_i^T Lam~_i   (A = alpha (I - beta k k^T) = A^T)
// and per step (state S_prev before it, Lam after it):
//   dv = beta Lam^T k,  dk = beta Lam v - alpha beta (Lam S_prev^T k + S_prev Lam^T k),
//   dbeta = k^T Lam v - alpha (k^T S_prev)(Lam^T k),  dg = alpha (<Lam, S_prev> - beta (k^T S_prev)(Lam^T k)),
//   dq_t = S_t do_t / sqrt(d).
//
// Every column of S evolves on its own (the rule only mixes rows), and so does every column of
// Lam.  One CTA takes one (document, head, slice of 32 columns); two threads per column hold half
// of its rows of S and of Lam in registers (a pair shuffle completes the k^T S and k^T Lam dot
// products).  Gradients that sum over columns (dq, dk, dg, dbeta) are reduced over the CTA's 32
// columns in shared memory and stored as the slice's partial in the workspace; a second kernel
// adds the d/32 partials of every element in slice order, so the results are the same on every
// call (no atomics).
//   pass 1: the clean chain, writing the state before every 16th token into the workspace
//   pass 2: 16-token segments from the last: the segment's states are rebuilt from its
//           checkpoint, 4 tokens at a time into shared memory, and the adjoint runs backwards
//           through them; where a response block starts right after a token, each view's block
//           is rebuilt from that token's state (token by token, from the start for every step)
//           and run backwards, and its initial-state gradient joins Lam.
// The work per token is a few dot products of length d per column: CUDA cores, not tensor cores.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kBwdThreads = 64;       // 32 columns x 2 row halves
constexpr int kCk = 16;               // checkpoint stride (tokens)
constexpr int kSeg = 4;               // states rebuilt into shared memory at a time

struct BwdParams {
    const void *q, *k, *v, *qn, *kn, *vn, *dout, *doutn;
    const float *g, *beta, *gn, *betan, *dsf;
    float *dq, *dk, *dv, *dg, *dbeta, *dqn, *dkn, *dvn, *dgn, *dbetan;
    float *ck;                        // checkpoints [ck index][H][slice][R2][64]
    int64_t pst_vec, pst_sc, pst_nvec, pst_nsc;   // slice strides of the partial buffers (floats)
    int64_t TR;
    int32_t N, H, V, B;
    float scale;
    int32_t doc_start[kMaxDocs + 1];
    int32_t doc_prompt[kMaxDocs];
    int32_t resp_off[kMaxDocs + 1];
    int32_t ck_off[kMaxDocs + 1];     // first checkpoint of each document
};

template <typename T>
__device__ __forceinline__ float ld(const void *p, int64_t i) {
    return to_f32(static_cast<const T *>(p)[i]);
}

// the two threads of a column (adjacent lanes) hold its two row halves
__device__ __forceinline__ float pair_sum(float x) {
    return x + __shfl_xor_sync(0xffffffffu, x, 1);
}

template <typename TIO, int D>
__global__ void __launch_bounds__(kBwdThreads)
gdn_backward_kernel(const __grid_constant__ BwdParams P) {
    constexpr int R2 = D / 2, NS = D / 32;
    extern __shared__ float smb[];
    float *seg = smb;                                 // [kSeg][R2][64]: states before the tokens
    float *s0b = seg + kSeg * R2 * kBwdThreads;        // [R2][64]: a noisy block's start state
    float *lmb = s0b + R2 * kBwdThreads;              // [R2][64]: the clean Lam while a block runs
    float *red = lmb + R2 * kBwdThreads;              // [32][D + 2]: column reduction
    const int tid = threadIdx.x, c = tid >> 1, hf = tid & 1, rb = hf * R2;
    const int unit = blockIdx.x / NS, js = blockIdx.x % NS, col = js * 32 + c;
    const int n = unit / P.H, h = unit % P.H, H = P.H;
    const int s = P.doc_start[n], len = P.doc_start[n + 1] - s, Pn = P.doc_prompt[n], R = len - Pn;
    const int roff = P.resp_off[n];
    const float sc = P.scale;
    auto at = [&](float *buf, int i) -> float & { return buf[i * kBwdThreads + tid]; };
    // this slice's partial buffers (P.dq ... point at slice 0)
    float *const pdq = P.dq + js * P.pst_vec, *const pdk = P.dk + js * P.pst_vec;
    float *const pdg = P.dg + js * P.pst_sc, *const pdbeta = P.dbeta + js * P.pst_sc;
    float *const pdqn = P.dqn + js * P.pst_nvec, *const pdkn = P.dkn + js * P.pst_nvec;
    float *const pdgn = P.dgn + js * P.pst_nsc, *const pdbetan = P.dbetan + js * P.pst_nsc;

    // this thread's rows of a k or q vector (clean row, or noisy packed row), as 16-byte loads
    // (the rows start 32-byte aligned: D >= 32 and the tensors are 16-byte aligned)
    auto kq = [&](const void *base, int64_t row, float (&x)[R2]) {
        const int64_t o = (row * H + h) * D + rb;
        if constexpr (sizeof(TIO) == 4) {
            const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + o);
#pragma unroll
            for (int i = 0; i < R2 / 4; ++i) {
                const float4 f = __ldg(p + i);
                x[4 * i] = f.x;
                x[4 * i + 1] = f.y;
                x[4 * i + 2] = f.z;
                x[4 * i + 3] = f.w;
            }
        } else {
            const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(base) + o);
#pragma unroll
            for (int i = 0; i < R2 / 8; ++i) {
                const uint4 u = __ldg(p + i);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
                    x[8 * i + 2 * j] = f.x;
                    x[8 * i + 2 * j + 1] = f.y;
                }
            }
        }
    };
    // one forward step of this thread's half column
    auto fwd = [&](float (&st)[R2], const float (&kk)[R2], float vc, float a, float b) {
        float ks = 0.f;
#pragma unroll
        for (int i = 0; i < R2; ++i) ks = fmaf(kk[i], st[i], ks);
        ks = pair_sum(ks);
#pragma unroll
        for (int i = 0; i < R2; ++i) st[i] = a * fmaf(-b * ks, kk[i], st[i]) + b * kk[i] * vc;
    };
    // reduce red[c][0..D+1] over the 32 columns, add into out_vec[0..D) and the two scalars
    auto reduce_add = [&](float *out_vec, float *sc0, float *sc1) {
        __syncthreads();
        for (int r = tid; r < D + 2; r += kBwdThreads) {
            float a4[4] = {0.f, 0.f, 0.f, 0.f};         // four independent chains
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) a4[cc & 3] += red[cc * (D + 2) + r];
            const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
            if (r < D) {
                if (out_vec) out_vec[r] = acc;
            } else if (r == D) {
                if (sc0) *sc0 = acc;
            } else if (sc1) {
                *sc1 = acc;
            }
        }
        __syncthreads();
    };
    // backward of one step: Lam (after the step) -> Lam before it; S_prev in sp.
    // Writes dk rows and the dg, dbeta column terms into red, dv of this column into *dv_out.
    auto bwd = [&](float (&lam)[R2], const float (&sp)[R2], const float (&kk)[R2], float vc, float a, float b,
                   float *dv_out) {
        float kl = 0.f, ks = 0.f, ls = 0.f;
#pragma unroll
        for (int i = 0; i < R2; ++i) {
            kl = fmaf(kk[i], lam[i], kl);
            ks = fmaf(kk[i], sp[i], ks);
            ls = fmaf(lam[i], sp[i], ls);
        }
        kl = pair_sum(kl);
        ks = pair_sum(ks);
        float *rr = red + c * (D + 2);
#pragma unroll
        for (int i = 0; i < R2; ++i) rr[rb + i] = b * vc * lam[i] - a * b * (ks * lam[i] + kl * sp[i]);
        // dalpha = <Lam, S_prev> - beta ks kl ; dg = alpha dalpha ; dbeta = kl v - alpha ks kl
        const float own = a * ls;                             // this half's part of alpha <Lam, S_prev>
        const float other = __shfl_xor_sync(0xffffffffu, own, 1);
        if (hf == 0) {
            rr[D] = own + other - a * b * ks * kl;
            rr[D + 1] = kl * vc - a * ks * kl;
            *dv_out = b * kl;
        }
#pragma unroll
        for (int i = 0; i < R2; ++i) lam[i] = a * fmaf(-b * kl, kk[i], lam[i]);
    };
    // dq rows = S do / sqrt(d) for one token, reduced over the columns
    auto dq_rows = [&](const float (&st)[R2], float doc_, float *out_vec) {
        float *rr = red + c * (D + 2);
#pragma unroll
        for (int i = 0; i < R2; ++i) rr[rb + i] = st[i] * doc_ * sc;
        if (hf == 0) rr[D] = rr[D + 1] = 0.f;
        reduce_add(out_vec, nullptr, nullptr);
    };

    // Backward of every view of the noisy block at packed rows [roff + r0, +B), started from the
    // state in s0b; adds the views' initial-state gradients into lmb.
    auto noisy_block = [&](int r0, float (&sw)[R2], float (&lt)[R2]) {
        for (int w = 0; w < P.V; ++w) {
            const int64_t base = (int64_t)w * P.TR + roff + r0;
            float kk[R2], qq[R2];
            // forward to the block end
#pragma unroll
            for (int i = 0; i < R2; ++i) sw[i] = at(s0b, i);
            for (int j = 0; j < P.B; ++j) {
                const int64_t row = base + j;
                kq(P.kn, row, kk);
                fwd(sw, kk, ld<TIO>(P.vn, (row * H + h) * D + col), expf(P.gn[row * H + h]), P.betan[row * H + h]);
            }
            // Lam~_B and dq~ of every position
#pragma unroll
            for (int i = 0; i < R2; ++i) lt[i] = 0.f;
            for (int j = 0; j < P.B; ++j) {
                const int64_t row = base + j;
                const float dd = ld<TIO>(P.doutn, (row * H + h) * D + col);
                kq(P.qn, row, qq);
#pragma unroll
                for (int i = 0; i < R2; ++i) lt[i] = fmaf(qq[i], dd * sc, lt[i]);
                dq_rows(sw, dd, pdqn + (row * H + h) * D);
            }
            // steps from the last: rebuild the state before step j from the block start
            for (int j = P.B - 1; j >= 0; --j) {
#pragma unroll
                for (int i = 0; i < R2; ++i) sw[i] = at(s0b, i);
                for (int jj = 0; jj < j; ++jj) {
                    const int64_t row = base + jj;
                    kq(P.kn, row, kk);
                    fwd(sw, kk, ld<TIO>(P.vn, (row * H + h) * D + col), expf(P.gn[row * H + h]),
                        P.betan[row * H + h]);
                }
                const int64_t row = base + j;
                kq(P.kn, row, kk);
                float dvc = 0.f;
                bwd(lt, sw, kk, ld<TIO>(P.vn, (row * H + h) * D + col), expf(P.gn[row * H + h]),
                    P.betan[row * H + h], &dvc);
                if (hf == 0) P.dvn[(row * H + h) * D + col] = dvc;
                reduce_add(pdkn + (row * H + h) * D, pdgn + row * H + h, pdbetan + row * H + h);
            }
#pragma unroll
            for (int i = 0; i < R2; ++i) at(lmb, i) += lt[i];
        }
    };

    float st[R2], lam[R2], kk[R2];
    // ---------------- pass 1: clean chain with checkpoints every kCk tokens
#pragma unroll
    for (int i = 0; i < R2; ++i) st[i] = 0.f;
    auto ckp = [&](int ci) -> float * {
        return P.ck + (((int64_t)(P.ck_off[n] + ci) * H + h) * NS + js) * (R2 * kBwdThreads);
    };
    for (int t = 0; t < len; ++t) {
        if (t % kCk == 0) {
            float *cp = ckp(t / kCk);
#pragma unroll
            for (int i = 0; i < R2; ++i) cp[i * kBwdThreads + tid] = st[i];
        }
        const int64_t row = s + t;
        kq(P.k, row, kk);
        fwd(st, kk, ld<TIO>(P.v, (row * H + h) * D + col), expf(P.g[row * H + h]), P.beta[row * H + h]);
    }
    // st = final state; Lam starts at the final-state gradient
#pragma unroll
    for (int i = 0; i < R2; ++i)
        lam[i] = P.dsf ? P.dsf[(((int64_t)n * H + h) * D + rb + i) * D + col] : 0.f;

    // ---------------- pass 2: backwards over the segments
    float sp[R2];
    const int nseg = (len + kCk - 1) / kCk;
    for (int sgi = nseg - 1; sgi >= 0; --sgi) {
        const int t0 = sgi * kCk, t1 = min(len, t0 + kCk);
        for (int u0 = t1 - ((t1 - t0 - 1) % kSeg) - 1; u0 >= t0; u0 -= kSeg) {
            // rebuild the states before tokens u0 .. u1-1 (u0 >= t0 on a kSeg grid from t0)
            const int u1 = min(t1, u0 + kSeg);
            const float *cp = ckp(sgi);
#pragma unroll
            for (int i = 0; i < R2; ++i) sp[i] = cp[i * kBwdThreads + tid];
            for (int t = t0; t < u1; ++t) {
                if (t >= u0) {
#pragma unroll
                    for (int i = 0; i < R2; ++i) at(seg, (t - u0) * R2 + i) = sp[i];
                }
                const int64_t row = s + t;
                kq(P.k, row, kk);
                fwd(sp, kk, ld<TIO>(P.v, (row * H + h) * D + col), expf(P.g[row * H + h]), P.beta[row * H + h]);
            }
            // sp = the state after token u1 - 1
            for (int t = u1 - 1; t >= u0; --t) {
                const int64_t row = s + t;
                const float dd = ld<TIO>(P.dout, (row * H + h) * D + col);
                float qq[R2];
                kq(P.q, row, qq);
#pragma unroll
                for (int i = 0; i < R2; ++i) lam[i] = fmaf(qq[i], dd * sc, lam[i]);
                // a response block starts right after this token: its views start from S_t
                const int rel = t + 1 - Pn;
                if (rel >= 0 && rel < R && rel % P.B == 0 && P.V > 0) {
#pragma unroll
                    for (int i = 0; i < R2; ++i) {
                        at(s0b, i) = sp[i];
                        at(lmb, i) = lam[i];
                    }
                    noisy_block(rel, sp, lam);
#pragma unroll
                    for (int i = 0; i < R2; ++i) {
                        sp[i] = at(s0b, i);
                        lam[i] = at(lmb, i);
                    }
                }
                dq_rows(sp, dd, pdq + (row * H + h) * D);
                // the state before token t
#pragma unroll
                for (int i = 0; i < R2; ++i) sp[i] = at(seg, (t - u0) * R2 + i);
                kq(P.k, row, kk);
                float dvc = 0.f;
                bwd(lam, sp, kk, ld<TIO>(P.v, (row * H + h) * D + col), expf(P.g[row * H + h]),
                    P.beta[row * H + h], &dvc);
                if (hf == 0) P.dv[(row * H + h) * D + col] = dvc;
                reduce_add(pdk + (row * H + h) * D, pdg + row * H + h, pdbeta + row * H + h);
            }
        }
    }
    // first block of a document without prompt: it starts from the hard zero state
    if (Pn == 0 && R > 0 && P.V > 0) {
#pragma unroll
        for (int i = 0; i < R2; ++i) {
            at(s0b, i) = 0.f;
            at(lmb, i) = 0.f;
        }
        noisy_block(0, sp, lam);
    }
}

// out[i] = sum over the ns slice partials part[s * stride + i], in slice order.
__global__ void reduce_slices_kernel(const float *__restrict__ part, float *__restrict__ out, int64_t n,
                                     int64_t stride, int ns) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float acc = part[i];
        for (int s = 1; s < ns; ++s) acc += part[s * stride + i];
        out[i] = acc;
    }
}

cudaError_t reduce_slices(const float *part, float *out, int64_t n, int64_t stride, int ns, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
    reduce_slices_kernel<<<(unsigned)blocks, 256, 0, st>>>(part, out, n, stride, ns);
    return cudaGetLastError();
}

template <typename TIO, int D>
cudaError_t launch_bwd(const BwdParams &p, cudaStream_t st) {
    constexpr int R2 = D / 2;
    const size_t smem = (size_t)(kSeg + 2) * R2 * kBwdThreads * 4 + 32 * (D + 2) * 4;
    cudaError_t e = cudaFuncSetAttribute(gdn_backward_kernel<TIO, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)p.N * p.H * (D / 32);
    gdn_backward_kernel<TIO, D><<<(unsigned)grid, kBwdThreads, smem, st>>>(p);
    return cudaGetLastError();
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t bwd_checkpoints(const gdn_dual_desc *d, const int32_t *offs) {
    int64_t nck = 0;
    for (int n = 0; n < d->num_docs; ++n) nck += ((int64_t)offs[n + 1] - offs[n] + kCk - 1) / kCk;
    return nck;
}

// Partial buffers of the column-summed gradients: per slice, [dq | dk] (T H d each), [dg | dbeta]
// (T H each), and for the noisy stream the same over V T rows (T_R <= T: the size needs no prompt
// lengths).  Returns floats per slice; *strides gets the four per-slice offsets and strides.
int64_t bwd_partial_floats(const gdn_dual_desc *d, int64_t T) {
    const int64_t th = T * d->num_heads, V = d->num_views;
    return 2 * th * d->d_k + 2 * th + (V > 0 ? 2 * V * th * d->d_k + 2 * V * th : 0);
}

bool bwd_desc_ok(const gdn_dual_desc *d) {
    return d && d->num_docs >= 1 && d->num_heads >= 1 && d->d_k >= 1 && d->d_v >= 1 &&
           d->num_views >= 0 && d->block_size >= 1 && (d->dtype == GDN_BF16 || d->dtype == GDN_FP32) &&
           d->conv_width >= 0 && d->reserved == 0;
}

}  // namespace
}  // namespace gdn


namespace gdn {

// The backward on validated arguments: dtype is the element type of q, k, v, their noisy twins
// and the upstream gradients (the ShortConv entry point passes fp32 copies).  The workspace holds
// the checkpoints, then the slice partials.
gdn_status run_backward(const gdn_dual_desc *desc, int dtype, const void *q, const void *k, const void *v,
                        const float *g, const float *beta, const void *qn, const void *kn, const void *vn,
                        const float *gn, const float *betan, const int32_t *doc_offsets, const int32_t *prompt_len,
                        const void *d_out, const void *d_out_noisy, const float *d_final_state, float *dq,
                        float *dk, float *dv, float *dg, float *dbeta, float *dqn, float *dkn, float *dvn,
                        float *dgn, float *dbetan, void *workspace, cudaStream_t st) {
    const int N = desc->num_docs, H = desc->num_heads, B = desc->block_size, D = desc->d_k;
    int64_t TR = 0;
    for (int n = 0; n < N; ++n) TR += (int64_t)doc_offsets[n + 1] - doc_offsets[n] - prompt_len[n];
    const int64_t T = doc_offsets[N];
    const bool noisy = desc->num_views > 0 && TR > 0;
    const int ns = D / 32;
    const int64_t nck = bwd_checkpoints(desc, doc_offsets);
    float *ck = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + 256);
    float *part = ck + nck * H * D * D;
    const int64_t th = T * H, V = desc->num_views;
    // slice-0 bases and slice strides of the partials (bwd_partial_floats layout)
    const int64_t per_slice = bwd_partial_floats(desc, T);
    float *p_dq = part, *p_dk = part + th * D, *p_dg = part + 2 * th * D, *p_dbeta = p_dg + th;
    float *p_dqn = p_dbeta + th, *p_dkn = p_dqn + V * th * D, *p_dgn = p_dkn + V * th * D, *p_dbetan = p_dgn + V * th;

    BwdParams P;
    std::memset(&P, 0, sizeof(P));
    P.q = q; P.k = k; P.v = v; P.qn = qn; P.kn = kn; P.vn = vn; P.dout = d_out; P.doutn = d_out_noisy;
    P.g = g; P.beta = beta; P.gn = gn; P.betan = betan; P.dsf = d_final_state;
    P.dq = p_dq; P.dk = p_dk; P.dv = dv; P.dg = p_dg; P.dbeta = p_dbeta;
    P.dqn = p_dqn; P.dkn = p_dkn; P.dvn = dvn; P.dgn = p_dgn; P.dbetan = p_dbetan;
    P.pst_vec = P.pst_sc = P.pst_nvec = P.pst_nsc = per_slice;
    P.ck = ck;
    P.TR = TR; P.N = N; P.H = H; P.V = noisy ? desc->num_views : 0; P.B = B;
    P.scale = (float)(1.0 / std::sqrt((double)D));
    int64_t roff = 0, ckn = 0;
    for (int n = 0; n <= N; ++n) {
        P.doc_start[n] = doc_offsets[n];
        P.resp_off[n] = (int32_t)roff;
        P.ck_off[n] = (int32_t)ckn;
        if (n < N) {
            P.doc_prompt[n] = prompt_len[n];
            roff += (int64_t)doc_offsets[n + 1] - doc_offsets[n] - prompt_len[n];
            ckn += ((int64_t)doc_offsets[n + 1] - doc_offsets[n] + kCk - 1) / kCk;
        }
    }
    cudaError_t e;
    const bool bf = dtype == GDN_BF16;
    switch (D) {
        case 32: e = bf ? launch_bwd<__nv_bfloat16, 32>(P, st) : launch_bwd<float, 32>(P, st); break;
        case 64: e = bf ? launch_bwd<__nv_bfloat16, 64>(P, st) : launch_bwd<float, 64>(P, st); break;
        default: e = bf ? launch_bwd<__nv_bfloat16, 128>(P, st) : launch_bwd<float, 128>(P, st); break;
    }
    // the slice partials, added in slice order
    const int64_t nn = (noisy ? V * TR : 0) * H;
    if (e == cudaSuccess) e = reduce_slices(p_dq, dq, th * D, per_slice, ns, st);
    if (e == cudaSuccess) e = reduce_slices(p_dk, dk, th * D, per_slice, ns, st);
    if (e == cudaSuccess) e = reduce_slices(p_dg, dg, th, per_slice, ns, st);
    if (e == cudaSuccess) e = reduce_slices(p_dbeta, dbeta, th, per_slice, ns, st);
    if (noisy) {
        // the noisy partials are laid out over V x T_R rows inside their V x T row sections
        if (e == cudaSuccess) e = reduce_slices(p_dqn, dqn, nn * D, per_slice, ns, st);
        if (e == cudaSuccess) e = reduce_slices(p_dkn, dkn, nn * D, per_slice, ns, st);
        if (e == cudaSuccess) e = reduce_slices(p_dgn, dgn, nn, per_slice, ns, st);
        if (e == cudaSuccess) e = reduce_slices(p_dbetan, dbetan, nn, per_slice, ns, st);
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn

using namespace gdn;

extern "C" size_t gdn_dual_backward_workspace_size(const gdn_dual_desc *desc, const int32_t *doc_offsets_host) {
    if (!bwd_desc_ok(desc) || !doc_offsets_host || doc_offsets_host[0] != 0) return 0;
    for (int n = 0; n < desc->num_docs; ++n)
        if (doc_offsets_host[n + 1] < doc_offsets_host[n]) return 0;
    const int64_t nck = bwd_checkpoints(desc, doc_offsets_host);
    const int ns = desc->d_k >= 32 ? desc->d_k / 32 : 1;
    const int64_t part = (int64_t)ns * bwd_partial_floats(desc, doc_offsets_host[desc->num_docs]);
    return ((size_t)nck * desc->num_heads * desc->d_k * desc->d_v + (size_t)part) * sizeof(float) + 256;
}

extern "C" gdn_status gdn_dual_backward(const gdn_dual_desc *desc, const void *q, const void *k, const void *v,
                                        const float *g, const float *beta, const void *qn, const void *kn,
                                        const void *vn, const float *gn, const float *betan,
                                        const int32_t *doc_offsets, const int32_t *prompt_len,
                                        const void *d_out, const void *d_out_noisy, const float *d_final_state,
                                        float *dq, float *dk, float *dv, float *dg, float *dbeta,
                                        float *dqn, float *dkn, float *dvn, float *dgn, float *dbetan,
                                        void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    if (!bwd_desc_ok(desc) || !doc_offsets || !prompt_len || doc_offsets[0] != 0) return GDN_ERR_INVALID_ARG;
    const int N = desc->num_docs, B = desc->block_size, D = desc->d_k;
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
    if (T > 0 && (!q || !k || !v || !g || !beta || !d_out || !dq || !dk || !dv || !dg || !dbeta))
        return GDN_ERR_INVALID_ARG;
    if (noisy && (!qn || !kn || !vn || !gn || !betan || !d_out_noisy || !dqn || !dkn || !dvn || !dgn || !dbetan))
        return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_dual_backward_workspace_size(desc, doc_offsets);
    if (!workspace || workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, qn, kn, vn, gn, betan, d_out, d_out_noisy, d_final_state,
                          dq, dk, dv, dg, dbeta, dqn, dkn, dvn, dgn, dbetan, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    if (desc->d_k != desc->d_v || (D != 32 && D != 64 && D != 128) || desc->conv_width != 0 || N > kMaxDocs)
        return GDN_ERR_UNSUPPORTED;
    if (T == 0) return GDN_OK;

    return gdn::run_backward(desc, desc->dtype, q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len,
                             d_out, d_out_noisy, d_final_state, dq, dk, dv, dg, dbeta, dqn, dkn, dvn, dgn, dbetan,
                             workspace, reinterpret_cast<cudaStream_t>(stream));
}
