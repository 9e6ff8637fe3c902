// gdn_route1_tc.cu -- Route I on tensor cores, second stage: every noisy block refined from its
// stored boundary state (sm_100a, bf16, d = 128, B = 16 or 32).
//
// "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes), Method > Key design 2: Route
// I (chunk-then-refine) writes the clean state before every response block to memory, then runs
// each view's block from it; the notes report it ahead of their fused schedule at B >= 16.  The
// first stage is the chunked kernel's EXPORT instantiation (gdn_chunked.cu): the clean stream,
// plus the state S_e before every response block as a 32 KB blob in the bf16 S0 tile layout.
//
// Here one item is (boundary state, pair of views).  With Gamma~_i = e^{gamma~_i} the cumulative
// decays inside the block (gamma~ the inclusive cumulative sum of g~), the block in WY/UT form:
//   A~_il = beta~_i e^{gamma~_i - gamma~_l} k~_i.k~_l (l < i),  (I + A~) U~ = R~,
//   R~ = diag(beta~) V~ - diag(beta~ Gamma~) K~ S_e,
//   S_end = Gamma~_B S_e + sum_i e^{gamma~_B - gamma~_i} k~_i u~_i^T,  o~_j = S_end^T q~_j / sqrt(d)
//         = [Gamma~_B (Q~ S_e)_j + sum_i e^{gamma~_B - gamma~_i} (q~_j.k~_i) u~_i] / sqrt(d)
// (gamma~_B the last row's).  The tensor cores form [K~0; K~1; Q~0; Q~1] S_e and
// [K~0; K~1; Q~0; Q~1] [K~0; K~1]^T in one 128-row tile (the state blob loaded as it was stored,
// the MMA's B operand); the rest is per row (tensor memory to shared memory) and per column
// (forward substitution for U~, then the block-end read-out) on CUDA cores in fp32.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int RD = 128;                      // head dim
constexpr int kRThreads = 256;
// Two stages (the next item's loads arrive while this one is computed), each a 32 KB state blob
// (MN-major B operand) and a 32 KB [K~0; K~1; Q~0; Q~1] tile (K-major, 128B swizzle).
constexpr int R_STAGE = 65536;
constexpr int R_OFF_S = 0, R_OFF_A = 32768;
constexpr int R_OFF_X = 2 * R_STAGE;         // fp32 scratch (see below)

template <int B>
struct RLayout {
    // fp32 scratch after the tiles: R~ (then read by columns) and Q~S_e rows per view, A~ and the
    // decayed Q~K~^T per view, the block's log2-decays and betas per view.  Rows are written by
    // one thread each, so R~ and Q~S_e strides are padded by one word (no bank conflicts); A~ and
    // Q~K~^T rows by four, so the column phase reads them as 16-byte broadcasts.
    static constexpr int RS = RD + 1, BS = B + 4;             // row strides
    static constexpr int R = 0;                               // [2][B][RS]
    static constexpr int QS = R + 2 * B * RS;                 // [2][B][RS]
    static constexpr int AT = QS + 2 * B * RS;                // [2][B][BS]
    static constexpr int MQ = AT + 2 * B * BS;                // [2][B][BS]
    static constexpr int GAM = MQ + 2 * B * BS;               // [2][B]
    static constexpr int BETA = GAM + 2 * B;                  // [2][B]
    static constexpr int FLOATS = BETA + 2 * B;
    static constexpr int SMEM = R_OFF_X + FLOATS * 4 + 1024;  // + alignment slack
};

struct R1Params {
    const float *gn, *betan;                 // [V, T_R, H]
    const __nv_bfloat16 *vn;                 // [V, T_R, H, d]
    __nv_bfloat16 *out_noisy;                // [V, T_R, H, d]
    const uint8_t *states;                   // [T_R / B][H] blobs of 32 KB
    WorkspaceHeader *ws;
    int64_t TR;
    int32_t H, V, pairs;
    int64_t items;                           // (T_R / B) * H * pairs
    float scale;                             // 1 / sqrt(d)
};

struct R1Maps {
    CUtensorMap qn, kn;                      // box: 64 columns x 1 head x B rows
};

// Column l of view w's [K~0; K~1]^T block in a 32-column tensor-memory load (B = 16: both views in
// one load; B = 32: one view each): constant indices, so the loaded values stay in registers.
template <int B>
__device__ __forceinline__ float col_of(const float (&xr)[32], int w, int l) {
    if constexpr (B == 16) return w ? xr[16 + l] : xr[l];
    else return xr[l];
}

template <int B>
__global__ void __launch_bounds__(kRThreads, 1)
gdn_route1_refine_kernel(const __grid_constant__ R1Params P, const __grid_constant__ R1Maps M) {
    using L = RLayout<B>;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    float *X = reinterpret_cast<float *>(sm + R_OFF_X);
    __shared__ uint64_t bar_ld[2], bar_mma, bar_drain;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5;
    constexpr float kLog2e = 1.4426950408889634f;

    if (tid == 0) {
        mbar_init(&bar_ld[0], 1);
        mbar_init(&bar_ld[1], 1);
        mbar_init(&bar_mma, 1);
        mbar_init(&bar_drain, 1);
        fence_mbar_init();
        s_abort = 0;
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = s_tmem;
    auto fail = [&](int where) {
        if (atomicExch(&s_abort, 1) == 0) {
            atomicExch(&P.ws->status, (int)GDN_ERR_TIMEOUT);
            atomicExch(&P.ws->timeout_where, where);
        }
    };
    auto wait_ok = [&](uint64_t *bar, uint32_t parity, int where) {
        const bool ok = mbar_wait(bar, parity, kWaitIters);
        if (!ok) fail(where);
        return ok;
    };
    // (thread 0) the loads of `item` into stage st: the state blob and the views' k~, q~ rows
    // (rows 0..4B of the A tile)
    uint32_t iss[2] = {0, 0};
    auto issue_loads = [&](int64_t item, int st) {
        const int64_t sidx = item / P.pairs;
        const int pair = (int)(item - sidx * P.pairs);
        const int h = (int)(sidx % P.H);
        const int64_t row0 = (sidx / P.H) * B;
        const int v0 = 2 * pair, nv = min(2, P.V - v0);
        uint8_t *stg = sm + st * R_STAGE;
        ++iss[st];
        mbar_arrive_expect_tx(&bar_ld[st], 32768u + (uint32_t)(nv * 2 * 2 * B * 128));
        bulk_load(stg + R_OFF_S, P.states + sidx * 32768, 32768u, &bar_ld[st]);
        for (int w = 0; w < nv; ++w) {
            const int row = (int)((int64_t)(v0 + w) * P.TR + row0);
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_3d(stg + R_OFF_A + hf * 16384 + (w * B) * 128, &M.kn, &bar_ld[st], hf * 64, h, row);
                tma_load_3d(stg + R_OFF_A + hf * 16384 + (2 * B + w * B) * 128, &M.qn, &bar_ld[st], hf * 64, h, row);
            }
        }
    };
    uint32_t k = 0;                                  // items done by this CTA (mbarrier phases)
    bool issued = false, stop = false;
    if (tid == 0 && (int64_t)blockIdx.x < P.items) issue_loads(blockIdx.x, 0);
    for (int64_t item = blockIdx.x; item < P.items; item += gridDim.x, ++k) {
        const int st = k & 1;
        const int64_t sidx = item / P.pairs;         // boundary state: (block, head)
        const int pair = (int)(item - sidx * P.pairs);
        const int h = (int)(sidx % P.H);
        const int64_t row0 = (sidx / P.H) * B;       // the block's first packed response row
        const int v0 = 2 * pair, nv = min(2, P.V - v0);
        const uint64_t dA = make_sdesc(smem_u32(sm + st * R_STAGE + R_OFF_A), 16, 1024);
        const uint64_t dS = make_sdesc(smem_u32(sm + st * R_STAGE + R_OFF_S), 16384, 1024);
        // the next item's loads go to the other stage, whose last MMAs completed an item ago
        if (tid == 0 && item + gridDim.x < P.items) issue_loads(item + gridDim.x, st ^ 1);
        // ---- the block's decays and betas (log2 units): one lane per (view, row), the inclusive
        //      cumulative sum by a shuffle scan over each view's B lanes
        if (tid < 2 * B) {
            const int w = tid / B, i = tid - w * B;
            float gl = 0.f, bt = 0.f;
            if (w < nv) {
                const int64_t idx = ((int64_t)(v0 + w) * P.TR + row0 + i) * P.H + h;
                gl = __ldg(P.gn + idx) * kLog2e;
                bt = __ldg(P.betan + idx);
            }
#pragma unroll
            for (int o = 1; o < B; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, gl, o, B);
                if (i >= o) gl += up;
            }
            X[L::GAM + w * B + i] = gl;
            X[L::BETA + w * B + i] = bt;
        }
        if (!wait_ok(&bar_ld[st], (k >> 1) & 1, 101)) stop = true;
        __syncwarp();
        if (tid == 0 && !stop) {
            tc_fence_after();
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(tb, dA + (off >> 4), dS + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 0, 1), kk > 0);
            }
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(tb + 128, dA + (off >> 4), dA + (off >> 4), make_idesc_bf16(128, 2 * B, 0, 0), kk > 0);
            }
            mma_commit(&bar_mma);
            issued = true;
        }
        __syncwarp();
        if (!stop && !wait_ok(&bar_mma, k & 1, 102)) stop = true;
        __syncwarp();
        tc_fence_after();
        if ((stop = __syncthreads_or(stop))) break;
        // ---- rows (warps 0-3, TMEM lane t = tile row t): K~ rows give R~ and A~, Q~ rows Q~S_e and
        //      the decayed Q~K~^T.  A warp's role (K~ rows, Q~ rows, none) is uniform because 2B and 4B
        //      are multiples of 32, so every lane of a warp runs the same tensor-memory loads; a row
        //      of a view that this item does not have only skips its reads and writes.
        if (warp < 4) {
            const int t = tid, kind = t / B, i = t - kind * B, w = kind & 1;
            const bool active = kind < 4 && w < nv;
            const int role = t < 2 * B ? 0 : (t < 4 * B ? 1 : 2);      // uniform over the warp
            const float *gam = X + L::GAM + w * B, *beta = X + L::BETA + w * B;
            float xr[32];
            if (role == 0) {
                const float bi = active ? beta[i] : 0.f, bg = active ? bi * exp2f(gam[i]) : 0.f;
                const __nv_bfloat16 *vrow = P.vn + (((int64_t)(v0 + w) * P.TR + row0 + i) * P.H + h) * RD;
                float *R = X + L::R + (w * B + i) * L::RS;
                uint4 vv[16];                                 // the row of v~, all loads in flight at once
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    vv[q] = active ? __ldg(reinterpret_cast<const uint4 *>(vrow) + q) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int c0 = 0; c0 < RD; c0 += 32) {
                    tmem_ld32(tmem_addr(tb, warp * 32, c0), xr);
                    tmem_wait_ld();
                    if (active) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            const uint4 u = vv[(c0 + e) / 8];
                            const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int p = 0; p < 4; ++p) {
                                const float va = __uint_as_float(wv[p] << 16), vb = __uint_as_float(wv[p] & 0xffff0000u);
                                R[c0 + e + 2 * p] = bi * va - bg * xr[e + 2 * p];
                                R[c0 + e + 2 * p + 1] = bi * vb - bg * xr[e + 2 * p + 1];
                            }
                        }
                    }
                }
                tmem_ld32(tmem_addr(tb, warp * 32, 128 + 32 * ((w * B) / 32)), xr);    // k~_i . k~_l
                tmem_wait_ld();
                if (active) {
                    float *A = X + L::AT + (w * B + i) * L::BS;
#pragma unroll
                    for (int l = 0; l < B; ++l) {
                        const float kk = col_of<B>(xr, w, l);
                        A[l] = l < i ? bi * exp2f(gam[i] - gam[l]) * kk : 0.f;
                    }
                }
            } else if (role == 1) {
                float *Q = X + L::QS + (w * B + i) * L::RS;
#pragma unroll 1
                for (int c0 = 0; c0 < RD; c0 += 32) {
                    tmem_ld32(tmem_addr(tb, warp * 32, c0), xr);
                    tmem_wait_ld();
                    if (active) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) Q[c0 + e] = xr[e];
                    }
                }
                tmem_ld32(tmem_addr(tb, warp * 32, 128 + 32 * ((w * B) / 32)), xr);    // q~_i . k~_l
                tmem_wait_ld();
                if (active) {
                    float *Mq = X + L::MQ + (w * B + i) * L::BS;
                    const float gB = gam[B - 1];
#pragma unroll
                    for (int l = 0; l < B; ++l) Mq[l] = exp2f(gB - gam[l]) * col_of<B>(xr, w, l);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        // ---- columns (thread = (view, column)): U~ by forward substitution, then the read-out
        {
            const int w = tid >> 7, c = tid & 127;
            if (w < nv) {
                const float *R = X + L::R + w * B * L::RS, *A = X + L::AT + w * B * L::BS;
                const float *Q = X + L::QS + w * B * L::RS, *Mq = X + L::MQ + w * B * L::BS;
                float u[B];
#pragma unroll
                for (int i = 0; i < B; ++i) {
                    // two partial sums (even and odd groups of four) halve the dependent FMA chain
                    float acc0 = R[i * L::RS + c], acc1 = 0.f;
#pragma unroll
                    for (int l4 = 0; l4 < i; l4 += 4) {
                        const float4 a = *reinterpret_cast<const float4 *>(A + i * L::BS + l4);   // broadcast
                        float &acc = (l4 & 4) ? acc1 : acc0;
                        acc = fmaf(-a.x, u[l4], acc);
                        if (l4 + 1 < i) acc = fmaf(-a.y, u[l4 + 1], acc);
                        if (l4 + 2 < i) acc = fmaf(-a.z, u[l4 + 2], acc);
                        if (l4 + 3 < i) acc = fmaf(-a.w, u[l4 + 3], acc);
                    }
                    u[i] = acc0 + acc1;
                }
                const float GB = exp2f(X[L::GAM + w * B + B - 1]);
                __nv_bfloat16 *orow = P.out_noisy + (((int64_t)(v0 + w) * P.TR + row0) * P.H + h) * RD + c;
#pragma unroll 1
                for (int j = 0; j < B; ++j) {
                    float o[4] = {GB * Q[j * L::RS + c], 0.f, 0.f, 0.f};   // four independent chains
#pragma unroll
                    for (int i4 = 0; i4 < B; i4 += 4) {
                        const float4 m = *reinterpret_cast<const float4 *>(Mq + j * L::BS + i4);  // broadcast
                        o[0] = fmaf(m.x, u[i4], o[0]);
                        o[1] = fmaf(m.y, u[i4 + 1], o[1]);
                        o[2] = fmaf(m.z, u[i4 + 2], o[2]);
                        o[3] = fmaf(m.w, u[i4 + 3], o[3]);
                    }
                    orow[(int64_t)j * P.H * RD] = __float2bfloat16_rn(((o[0] + o[1]) + (o[2] + o[3])) * P.scale);
                }
            }
        }
        __syncthreads();          // tiles, tensor memory and scratch are free for the next item
    }
    // drain (only when a wait gave up): the last load and the MMAs
    if (stop && tid == 0) {
        for (int st = 0; st < 2; ++st)                // the last load issued on each stage
            if (iss[st]) mbar_wait(&bar_ld[st], (iss[st] - 1) & 1, kDrainWaitIters);
        if (issued) {
            mma_commit(&bar_drain);
            mbar_wait(&bar_drain, 0, kDrainWaitIters);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 256);
}

PFN_cuTensorMapEncodeTiled_v12000 r1_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [rows, H, 128] bf16; box = 64 columns x 1 head x `box_rows` rows, 128B swizzle
bool r1_map(CUtensorMap *m, const void *ptr, int H, int64_t rows, int box_rows) {
    auto enc = r1_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)RD, (cuuint64_t)H, (cuuint64_t)std::max<int64_t>(rows, 1)};
    cuuint64_t strides[2] = {(cuuint64_t)RD * 2, (cuuint64_t)H * RD * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int B>
cudaError_t launch_refine(const Params &p, cudaStream_t stream) {
    R1Params R;
    std::memset(&R, 0, sizeof(R));
    R.gn = p.gn;
    R.betan = p.betan;
    R.vn = static_cast<const __nv_bfloat16 *>(p.vn);
    R.out_noisy = static_cast<__nv_bfloat16 *>(p.out_noisy);
    R.states = static_cast<const uint8_t *>(p.states);
    R.ws = p.ws;
    R.TR = p.TR;
    R.H = p.H;
    R.V = p.V;
    R.pairs = (p.V + 1) / 2;
    R.items = (p.TR / B) * p.H * R.pairs;
    R.scale = p.scale;
    if (R.items == 0) return cudaSuccess;
    R1Maps maps;
    if (!r1_map(&maps.qn, p.qn, p.H, (int64_t)p.V * p.TR, B) || !r1_map(&maps.kn, p.kn, p.H, (int64_t)p.V * p.TR, B))
        return cudaErrorInvalidValue;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    static int sms = 148;
    std::call_once(once, [] {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        attr_err = cudaFuncSetAttribute(gdn_route1_refine_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        RLayout<B>::SMEM);
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int64_t grid = std::min<int64_t>(R.items, sms);
    gdn_route1_refine_kernel<B><<<(unsigned)grid, kRThreads, RLayout<B>::SMEM, stream>>>(R, maps);
    return cudaGetLastError();
}

}  // namespace

bool route1_tc_supported(int dtype, int d, int B, int conv_width) {
    return dtype == GDN_BF16 && d == RD && (B == 16 || B == 32) && conv_width == 0;
}

size_t route1_tc_state_bytes(int64_t TR, int H, int B) { return (size_t)(TR / B) * H * 32768; }

cudaError_t launch_route1_refine(const Params &p, cudaStream_t stream) {
    if (p.V == 0 || p.TR == 0) return cudaSuccess;
    switch (p.B) {
        case 16: return launch_refine<16>(p, stream);
        case 32: return launch_refine<32>(p, stream);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace gdn
