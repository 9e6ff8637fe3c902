// gdn_decode.cu -- decode-side state kernels of the Gated DeltaNet layer (include/gdn_decode.h).
//
// From the serving paragraph of "FLARE: Diffusion for Hybrid Language Model" (papernotes.org
// notes): Diffusion-Trust commits a finished block with one causal replay that writes the final
// state into the state pool; AR-Trust verifies K drafted candidates with one clean forward that
// also stores the state after every candidate step, and commits the first r accepted ones by a
// gather-scatter of state r (no recomputation).  The recurrence is that of Method > Key design 2:
// S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t / sqrt(d_k).
//
// Decode work is small and bound by moving states (d_k x d_v fp32 per sequence and head), so the
// kernels are CUDA-core kernels sized for bandwidth: a (sequence, head) is split into items of 32
// state columns, persistent CTAs prefetch the next item's state slice and tokens with cp.async
// while they step the current one, the columns live in registers (thread t owns column t/2 and
// half of its rows, so k^T S and S^T q need only a pair shuffle), and every state row segment is
// read or written as whole 32-byte sectors.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "gdn_internal.cuh"
#include "gdn_decode.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

// kReplay / kVerify: the serving kernels.  kBlockEnd: Route I's refinement of one noisy block from
// its stored boundary state (pool row n % nb), every position reading the block-end state.
enum DecodeMode { kReplay = 0, kVerify = 1, kBlockEnd = 2 };

struct DecodeParams {
    float *pool;              // [P, H, D, D]
    const int32_t *slots;     // [N]
    const void *q, *k, *v;    // [N, L, H, D]
    const float *g, *beta;    // [N, L, H]
    void *out;                // [N, L, H, D]
    float *cache;             // [N, L, H, D, D] (verify)
    int32_t *status;          // optional
    int N, H, L, P;
    int nb;                   // kBlockEnd: number of blocks per view (pool row of item n = n % nb)
    float scale;
};

__device__ __forceinline__ void flag_bad(int32_t *status) {
    if (status) atomicExch(status, (int32_t)GDN_ERR_INVALID_ARG);
}

// Columns of S per work item.  Every column of the state evolves on its own (u_j = k^T S[:, j], and
// the update and the readout of column j read only column j), so a (sequence, head) is split into
// D / kCols items of kCols columns.
constexpr int kCols = 32;

__host__ __device__ constexpr int round16(int x) { return (x + 15) & ~15; }

// Shared-memory bytes of one item buffer: state slice [D][kCols] fp32, q, k, v [L][D] as stored,
// g and beta [L] fp32.
template <typename TIO, int D>
__host__ __device__ constexpr int decode_buf_bytes(int L) {
    return D * kCols * 4 + 3 * round16(L * D * (int)sizeof(TIO)) + 2 * round16(L * 4);
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

// Persistent: each CTA walks work items (sequence, head, column slice) with a stride of gridDim.x
// and prefetches the next item's state slice and tokens into the other shared-memory buffer with
// cp.async while it runs the current one, so the state reads of one item overlap the steps and
// the stores of the previous one.
template <typename TIO, int D, int MODE>
__global__ void __launch_bounds__(2 * kCols) gdn_decode_kernel(const DecodeParams p) {
    constexpr int R = D / 2, NCB = D / kCols;
    extern __shared__ float4 sh4[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(sh4);
    const int tid = threadIdx.x, jl = tid >> 1, half = tid & 1;
    const int L = p.L;
    const int tok_bytes = round16(L * D * (int)sizeof(TIO)), sc_bytes = round16(L * 4);
    const int buf_bytes = decode_buf_bytes<TIO, D>(L);
    const int total = p.N * p.H * NCB;

    // cp.async the inputs of item w into buffer b; false (and nothing loaded) for a bad slot
    auto issue_load = [&](int w, int b) -> bool {
        const int unit = w / NCB, cb = w % NCB;
        const int n = unit / p.H, h = unit % p.H;
        const int slot = MODE == kBlockEnd ? n % p.nb : p.slots[n];
        if (slot < 0 || slot >= p.P) {
            if (tid == 0 && cb == 0) flag_bad(p.status);
            return false;
        }
        uint8_t *buf = smem + b * buf_bytes;
        const float *st = p.pool + ((int64_t)slot * p.H + h) * D * D + cb * kCols;
        for (int i = tid; i < D * (kCols / 4); i += 2 * kCols) {
            const int r = i / (kCols / 4), c4 = i % (kCols / 4);
            cp_async16(buf + (r * kCols + 4 * c4) * 4, st + (int64_t)r * D + 4 * c4);
        }
        constexpr int CPR = D * (int)sizeof(TIO) / 16;   // 16-byte pieces per token row
        const void *src[3] = {p.q, p.k, p.v};
        for (int x = 0; x < 3; ++x) {
            uint8_t *dst = buf + D * kCols * 4 + x * tok_bytes;
            const uint8_t *s0 = static_cast<const uint8_t *>(src[x]);
            for (int i = tid; i < L * CPR; i += 2 * kCols) {
                const int t = i / CPR, c = i % CPR;
                cp_async16(dst + t * D * (int)sizeof(TIO) + 16 * c,
                           s0 + (((int64_t)(n * L + t) * p.H + h) * D) * (int64_t)sizeof(TIO) + 16 * c);
            }
        }
        float *sg = reinterpret_cast<float *>(buf + D * kCols * 4 + 3 * tok_bytes);
        float *sb = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(sg) + sc_bytes);
        for (int t = tid; t < L; t += 2 * kCols) {
            const int64_t row = (int64_t)(n * L + t) * p.H + h;
            cp_async4(sg + t, p.g + row, 4);
            cp_async4(sb + t, p.beta + row, 4);
        }
        return true;
    };

    int w = blockIdx.x, b = 0;
    bool valid = w < total ? issue_load(w, 0) : false;
    cp_async_commit();
    while (w < total) {
        const int wn = w + gridDim.x;
        const bool vnext = wn < total ? issue_load(wn, b ^ 1) : false;
        cp_async_commit();
        cp_async_wait_group1();               // this item's group has landed (the next may not)
        __syncthreads();
        if (valid) {
            const int unit = w / NCB, cb = w % NCB;
            const int n = unit / p.H, h = unit % p.H;
            const int j = cb * kCols + jl;
            const uint8_t *buf = smem + b * buf_bytes;
            const float *st = reinterpret_cast<const float *>(buf);
            const TIO *sq = reinterpret_cast<const TIO *>(buf + D * kCols * 4);
            const TIO *sk = reinterpret_cast<const TIO *>(buf + D * kCols * 4 + tok_bytes);
            const TIO *sv = reinterpret_cast<const TIO *>(buf + D * kCols * 4 + 2 * tok_bytes);
            const float *sg = reinterpret_cast<const float *>(buf + D * kCols * 4 + 3 * tok_bytes);
            const float *sb = reinterpret_cast<const float *>(buf + D * kCols * 4 + 3 * tok_bytes + sc_bytes);
            float S[R];
#pragma unroll
            for (int r = 0; r < R; ++r) S[r] = st[(half * R + r) * kCols + jl];
            for (int t = 0; t < L; ++t) {
                const TIO *kt = sk + t * D + half * R, *qt = sq + t * D + half * R;
                const float alpha = expf(sg[t]), bt = sb[t];
                // u_j = (k^T S)_j: four partial sums shorten the dependent chain
                float pu[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int r4 = 0; r4 < R / 4; ++r4) {
                    const float4 kk = ld4(kt + 4 * r4);
                    pu[0] = fmaf(kk.x, S[4 * r4], pu[0]);
                    pu[1] = fmaf(kk.y, S[4 * r4 + 1], pu[1]);
                    pu[2] = fmaf(kk.z, S[4 * r4 + 2], pu[2]);
                    pu[3] = fmaf(kk.w, S[4 * r4 + 3], pu[3]);
                }
                float u = (pu[0] + pu[1]) + (pu[2] + pu[3]);
                u += __shfl_xor_sync(0xffffffffu, u, 1);
                // S <- alpha S + beta k (v - alpha u)^T   ( = alpha (I - beta k k^T) S + beta k v^T )
                const float wgt = bt * (to_f32(sv[t * D + j]) - alpha * u);
                float po[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int r4 = 0; r4 < R / 4; ++r4) {
                    const float4 kk = ld4(kt + 4 * r4), qq = ld4(qt + 4 * r4);
                    S[4 * r4] = fmaf(alpha, S[4 * r4], kk.x * wgt);
                    S[4 * r4 + 1] = fmaf(alpha, S[4 * r4 + 1], kk.y * wgt);
                    S[4 * r4 + 2] = fmaf(alpha, S[4 * r4 + 2], kk.z * wgt);
                    S[4 * r4 + 3] = fmaf(alpha, S[4 * r4 + 3], kk.w * wgt);
                    po[0] = fmaf(qq.x, S[4 * r4], po[0]);
                    po[1] = fmaf(qq.y, S[4 * r4 + 1], po[1]);
                    po[2] = fmaf(qq.z, S[4 * r4 + 2], po[2]);
                    po[3] = fmaf(qq.w, S[4 * r4 + 3], po[3]);
                }
                const int64_t row = (int64_t)(n * L + t) * p.H + h;
                if (MODE != kBlockEnd) {
                    float o = (po[0] + po[1]) + (po[2] + po[3]);
                    o += __shfl_xor_sync(0xffffffffu, o, 1);
                    if (half == 0) static_cast<TIO *>(p.out)[row * D + j] = from_f32<TIO>(o * p.scale);
                }
                if (MODE == kVerify) {
                    float *c = p.cache + row * D * D + (int64_t)(half * R) * D + j;
#pragma unroll
                    for (int r = 0; r < R; ++r) c[(int64_t)r * D] = S[r];
                }
            }
            if (MODE == kBlockEnd) {          // every position of the block reads the block-end state
                for (int t = 0; t < L; ++t) {
                    const TIO *qt = sq + t * D + half * R;
                    float po[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int r4 = 0; r4 < R / 4; ++r4) {
                        const float4 qq = ld4(qt + 4 * r4);
                        po[0] = fmaf(qq.x, S[4 * r4], po[0]);
                        po[1] = fmaf(qq.y, S[4 * r4 + 1], po[1]);
                        po[2] = fmaf(qq.z, S[4 * r4 + 2], po[2]);
                        po[3] = fmaf(qq.w, S[4 * r4 + 3], po[3]);
                    }
                    float o = (po[0] + po[1]) + (po[2] + po[3]);
                    o += __shfl_xor_sync(0xffffffffu, o, 1);
                    const int64_t row = (int64_t)(n * L + t) * p.H + h;
                    if (half == 0) static_cast<TIO *>(p.out)[row * D + j] = from_f32<TIO>(o * p.scale);
                }
            }
            if (MODE == kReplay) {
                const int slot = p.slots[n];
                float *s1 = p.pool + ((int64_t)slot * p.H + h) * D * D + (int64_t)(half * R) * D + j;
#pragma unroll
                for (int r = 0; r < R; ++r) s1[(int64_t)r * D] = S[r];
            }
        }
        __syncthreads();                      // buffer b is free for the load two items ahead
        w = wn;
        b ^= 1;
        valid = vnext;
    }
    cp_async_wait_all();
}

// Gather-scatter of accepted states: CTA (x, n*H + h) copies its share of state_cache[n, r-1, h]
// into state_pool[slots[n], h] as 16-byte words.
__global__ void __launch_bounds__(256) gdn_decode_commit_kernel(float *pool, const int32_t *slots,
                                                                const float *cache, const int32_t *accepted,
                                                                int32_t *status, int H, int L, int P, int DD) {
    const int unit = blockIdx.y, n = unit / H, h = unit % H;
    const int r = accepted[n], slot = slots[n];
    if (r < 0 || r > L || slot < 0 || slot >= P) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_bad(status);
        return;
    }
    if (r == 0) return;
    const float4 *src = reinterpret_cast<const float4 *>(cache + ((int64_t)(n * L + r - 1) * H + h) * DD);
    float4 *dst = reinterpret_cast<float4 *>(pool + ((int64_t)slot * H + h) * DD);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < DD / 4; i += gridDim.x * blockDim.x) dst[i] = src[i];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

gdn_status check_desc(const gdn_decode_desc *d) {
    if (!d || d->num_seqs < 1 || d->num_heads < 1 || d->d_k < 1 || d->d_v < 1 || d->num_tokens < 1 ||
        d->pool_slots < 1 || d->reserved != 0)
        return GDN_ERR_INVALID_ARG;
    if (d->dtype != GDN_BF16 && d->dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (d->d_k != d->d_v || (d->d_k != 32 && d->d_k != 64 && d->d_k != 128)) return GDN_ERR_UNSUPPORTED;
    if (d->num_tokens > 64) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

int num_sms() {
    static int n = 0;
    static std::once_flag once;
    std::call_once(once, [] {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            n = 148;
    });
    return n > 0 ? n : 148;
}

template <typename TIO, int D, int MODE>
gdn_status launch_steps(const DecodeParams &p, cudaStream_t s) {
    auto fn = gdn_decode_kernel<TIO, D, MODE>;
    const size_t smem = 2 * (size_t)decode_buf_bytes<TIO, D>(p.L);   // double buffer
    if (smem > 48 * 1024 && cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    const int items = p.N * p.H * (D / kCols);
    const int per_sm = std::max(1, std::min(6, (int)((200 * 1024) / smem)));
    const int grid = std::min(items, num_sms() * per_sm);
    fn<<<grid, 2 * kCols, smem, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <int MODE>
gdn_status run_steps(const gdn_decode_desc *d, float *pool, const int32_t *slots, const void *q, const void *k,
                     const void *v, const float *g, const float *beta, void *out, float *cache, int32_t *status,
                     gdn_stream_t stream) {
    gdn_status st = check_desc(d);
    if (st != GDN_OK) return st;
    if (!pool || !slots || !q || !k || !v || !g || !beta || !out || (MODE == kVerify && !cache))
        return GDN_ERR_INVALID_ARG;
    for (const void *t : {(const void *)pool, q, k, v, (const void *)g, (const void *)beta, (const void *)out,
                          (const void *)cache})
        if (t && !aligned16(t)) return GDN_ERR_ALIGNMENT;
    if (!aligned4(slots) || (status && !aligned4(status))) return GDN_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (status && cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return GDN_ERR_CUDA;
    DecodeParams p{pool, slots, q, k, v, g, beta, out, cache, status, d->num_seqs, d->num_heads, d->num_tokens,
                   d->pool_slots, 0, 1.0f / std::sqrt((float)d->d_k)};
    const bool bf = d->dtype == GDN_BF16;
    switch (d->d_k) {
    case 32: return bf ? launch_steps<__nv_bfloat16, 32, MODE>(p, s) : launch_steps<float, 32, MODE>(p, s);
    case 64: return bf ? launch_steps<__nv_bfloat16, 64, MODE>(p, s) : launch_steps<float, 64, MODE>(p, s);
    default: return bf ? launch_steps<__nv_bfloat16, 128, MODE>(p, s) : launch_steps<float, 128, MODE>(p, s);
    }
}

// ----------------------------------------------------------------------------- Route I
// Stage 1 of chunk-then-refine (Route I of the notes): the clean chain of every (document, head)
// token by token, split into items of kCols state columns, writing the clean outputs, the final
// state and, before every response block, the state S_{e(b-1)} into `states` [T_R / B, H, D, D]
// (block index = (first response row of the document + position in the response) / B).
constexpr int kTile = 32;                  // tokens staged per tile

template <typename TIO, int D>
__host__ __device__ constexpr int chain_buf_bytes() {
    return 3 * round16(kTile * D * (int)sizeof(TIO)) + 2 * round16(kTile * 4);
}

template <typename TIO, int D>
__global__ void __launch_bounds__(2 * kCols) gdn_route1_chain_kernel(const __grid_constant__ Params P, float *states) {
    constexpr int R = D / 2, NCB = D / kCols;
    constexpr int tok_bytes = round16(kTile * D * (int)sizeof(TIO)), sc_bytes = round16(kTile * 4);
    constexpr int buf_bytes = chain_buf_bytes<TIO, D>();
    constexpr int CPR = D * (int)sizeof(TIO) / 16;
    extern __shared__ float4 sh4[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(sh4);
    const int tid = threadIdx.x, jl = tid >> 1, half = tid & 1;
    const int H = P.H, B = P.B;
    const int total = P.num_units * NCB;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
        const int unit = w / NCB, cb = w % NCB;
        const int n = P.unit_doc[unit / H], h = unit % H;
        const int s0 = P.doc_start[n], len = P.doc_start[n + 1] - s0, prompt = P.doc_prompt[n];
        const int roff = P.resp_off[n];
        const int j = cb * kCols + jl;
        const int ntiles = (len + kTile - 1) / kTile;
        auto issue = [&](int ti, int b) {
            uint8_t *buf = smem + b * buf_bytes;
            const int t0 = ti * kTile, nt = min(kTile, len - t0);
            const void *src[3] = {P.q, P.k, P.v};
            for (int x = 0; x < 3; ++x) {
                const uint8_t *sx = static_cast<const uint8_t *>(src[x]);
                for (int i = tid; i < nt * CPR; i += 2 * kCols) {
                    const int t = i / CPR, c = i % CPR;
                    cp_async16(buf + x * tok_bytes + t * D * (int)sizeof(TIO) + 16 * c,
                               sx + (((int64_t)(s0 + t0 + t) * H + h) * D) * (int64_t)sizeof(TIO) + 16 * c);
                }
            }
            float *sg = reinterpret_cast<float *>(buf + 3 * tok_bytes), *sb = sg + sc_bytes / 4;
            for (int t = tid; t < nt; t += 2 * kCols) {
                const int64_t row = (int64_t)(s0 + t0 + t) * H + h;
                cp_async4(sg + t, P.g + row, 4);
                cp_async4(sb + t, P.beta + row, 4);
            }
        };
        float S[R];
#pragma unroll
        for (int r = 0; r < R; ++r) S[r] = 0.f;
        if (ntiles > 0) issue(0, 0);
        cp_async_commit();
        for (int ti = 0; ti < ntiles; ++ti) {
            const int b = ti & 1;
            if (ti + 1 < ntiles) issue(ti + 1, b ^ 1);
            cp_async_commit();
            cp_async_wait_group1();
            __syncthreads();
            const uint8_t *buf = smem + b * buf_bytes;
            const TIO *sq = reinterpret_cast<const TIO *>(buf), *sk = reinterpret_cast<const TIO *>(buf + tok_bytes);
            const TIO *sv = reinterpret_cast<const TIO *>(buf + 2 * tok_bytes);
            const float *sg = reinterpret_cast<const float *>(buf + 3 * tok_bytes), *sb = sg + sc_bytes / 4;
            const int t0 = ti * kTile, nt = min(kTile, len - t0);
            for (int t = 0; t < nt; ++t) {
                const int pos = t0 + t;
                if (pos >= prompt && (pos - prompt) % B == 0) {   // state before response block
                    const int64_t gb = (roff + pos - prompt) / B;
                    float *dst = states + (gb * H + h) * D * D + (int64_t)(half * R) * D + j;
#pragma unroll
                    for (int r = 0; r < R; ++r) dst[(int64_t)r * D] = S[r];
                }
                const TIO *kt = sk + t * D + half * R, *qt = sq + t * D + half * R;
                const float alpha = expf(sg[t]), bt = sb[t];
                float pu[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int r4 = 0; r4 < R / 4; ++r4) {
                    const float4 kk = ld4(kt + 4 * r4);
                    pu[0] = fmaf(kk.x, S[4 * r4], pu[0]);
                    pu[1] = fmaf(kk.y, S[4 * r4 + 1], pu[1]);
                    pu[2] = fmaf(kk.z, S[4 * r4 + 2], pu[2]);
                    pu[3] = fmaf(kk.w, S[4 * r4 + 3], pu[3]);
                }
                float u = (pu[0] + pu[1]) + (pu[2] + pu[3]);
                u += __shfl_xor_sync(0xffffffffu, u, 1);
                const float wgt = bt * (to_f32(sv[t * D + j]) - alpha * u);
                float po[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int r4 = 0; r4 < R / 4; ++r4) {
                    const float4 kk = ld4(kt + 4 * r4), qq = ld4(qt + 4 * r4);
                    S[4 * r4] = fmaf(alpha, S[4 * r4], kk.x * wgt);
                    S[4 * r4 + 1] = fmaf(alpha, S[4 * r4 + 1], kk.y * wgt);
                    S[4 * r4 + 2] = fmaf(alpha, S[4 * r4 + 2], kk.z * wgt);
                    S[4 * r4 + 3] = fmaf(alpha, S[4 * r4 + 3], kk.w * wgt);
                    po[0] = fmaf(qq.x, S[4 * r4], po[0]);
                    po[1] = fmaf(qq.y, S[4 * r4 + 1], po[1]);
                    po[2] = fmaf(qq.z, S[4 * r4 + 2], po[2]);
                    po[3] = fmaf(qq.w, S[4 * r4 + 3], po[3]);
                }
                float o = (po[0] + po[1]) + (po[2] + po[3]);
                o += __shfl_xor_sync(0xffffffffu, o, 1);
                if (half == 0)
                    static_cast<TIO *>(P.out)[((int64_t)(s0 + pos) * H + h) * D + j] = from_f32<TIO>(o * P.scale);
            }
            __syncthreads();                  // buffer b is free for tile ti + 2
        }
        cp_async_wait_all();
        float *fs = P.final_state + ((int64_t)n * H + h) * D * D + (int64_t)(half * R) * D + j;
#pragma unroll
        for (int r = 0; r < R; ++r) fs[(int64_t)r * D] = S[r];
    }
}

template <typename TIO, int D>
cudaError_t route1(const Params &p, float *states, cudaStream_t s) {
    auto chain = gdn_route1_chain_kernel<TIO, D>;
    const size_t smem1 = 2 * (size_t)chain_buf_bytes<TIO, D>();
    cudaError_t e = cudaSuccess;
    if (smem1 > 48 * 1024) e = cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e != cudaSuccess) return e;
    const int items1 = p.num_units * (D / kCols);
    const int grid1 = std::min(items1, num_sms() * std::max(1, std::min(6, (int)((200 * 1024) / smem1))));
    if (items1 > 0) chain<<<grid1, 2 * kCols, smem1, s>>>(p, states);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (p.V == 0 || p.TR == 0) return cudaSuccess;
    const int nb = (int)(p.TR / p.B);
    DecodeParams d{states, nullptr, p.qn, p.kn, p.vn, p.gn, p.betan, p.out_noisy, nullptr, nullptr,
                   p.V * nb, p.H, p.B, nb, nb, p.scale};
    auto refine = gdn_decode_kernel<TIO, D, kBlockEnd>;
    const size_t smem2 = 2 * (size_t)decode_buf_bytes<TIO, D>(p.B);
    if (smem2 > 48 * 1024 && (e = cudaFuncSetAttribute(refine, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2)) != cudaSuccess)
        return e;
    const int items2 = d.N * d.H * (D / kCols);
    const int grid2 = std::min(items2, num_sms() * std::max(1, std::min(6, (int)((200 * 1024) / smem2))));
    refine<<<grid2, 2 * kCols, smem2, s>>>(d);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route1(const Params &p, int dtype, float *states, cudaStream_t stream) {
    const bool bf = dtype == GDN_BF16;
    switch (p.dk) {
    case 32: return bf ? route1<__nv_bfloat16, 32>(p, states, stream) : route1<float, 32>(p, states, stream);
    case 64: return bf ? route1<__nv_bfloat16, 64>(p, states, stream) : route1<float, 64>(p, states, stream);
    case 128: return bf ? route1<__nv_bfloat16, 128>(p, states, stream) : route1<float, 128>(p, states, stream);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace gdn

extern "C" gdn_status gdn_decode_replay(const gdn_decode_desc *desc, float *state_pool, const int32_t *slots,
                                        const void *q, const void *k, const void *v, const float *g,
                                        const float *beta, void *out, int32_t *device_status, gdn_stream_t stream) {
    return gdn::run_steps<gdn::kReplay>(desc, state_pool, slots, q, k, v, g, beta, out, nullptr, device_status,
                                        stream);
}

extern "C" gdn_status gdn_decode_verify(const gdn_decode_desc *desc, const float *state_pool, const int32_t *slots,
                                        const void *q, const void *k, const void *v, const float *g,
                                        const float *beta, void *out, float *state_cache, int32_t *device_status,
                                        gdn_stream_t stream) {
    return gdn::run_steps<gdn::kVerify>(desc, const_cast<float *>(state_pool), slots, q, k, v, g, beta, out,
                                        state_cache, device_status, stream);
}

extern "C" gdn_status gdn_decode_commit(const gdn_decode_desc *desc, float *state_pool, const int32_t *slots,
                                        const float *state_cache, const int32_t *accepted, int32_t *device_status,
                                        gdn_stream_t stream) {
    gdn_status st = gdn::check_desc(desc);
    if (st != GDN_OK) return st;
    if (!state_pool || !slots || !state_cache || !accepted) return GDN_ERR_INVALID_ARG;
    if (!gdn::aligned16(state_pool) || !gdn::aligned16(state_cache)) return GDN_ERR_ALIGNMENT;
    if (!gdn::aligned4(slots) || !gdn::aligned4(accepted) || (device_status && !gdn::aligned4(device_status)))
        return GDN_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (device_status && cudaMemsetAsync(device_status, 0, sizeof(int32_t), s) != cudaSuccess) return GDN_ERR_CUDA;
    if ((int64_t)desc->num_seqs * desc->num_heads > 65535) return GDN_ERR_UNSUPPORTED;
    const int DD = desc->d_k * desc->d_v;
    const int blocks_x = std::max(1, std::min(8, DD / 4 / 256));
    dim3 grid(blocks_x, desc->num_seqs * desc->num_heads);
    gdn::gdn_decode_commit_kernel<<<grid, 256, 0, s>>>(state_pool, slots, state_cache, accepted, device_status,
                                                       desc->num_heads, desc->num_tokens, desc->pool_slots, DD);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
