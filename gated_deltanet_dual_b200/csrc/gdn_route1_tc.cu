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
// (gamma~_B the last row's).  With M~_jl = e^{gamma~_B - gamma~_l} q~_j.k~_l and Y = M~ (I + A~)^-1,
// the sum over i is (Y R~)_j, so U~ itself is never formed.  The tensor cores form
// [K~0; K~1; Q~0; Q~1] S_e and [K~0; K~1; Q~0; Q~1] [K~0; K~1]^T in one 128-row tile (the state
// blob loaded as it was stored, the MMA's B operand), and Y R~ (Y block-diagonal over the two
// views); CUDA cores take the rows in fp32 (R~, A~, M~) and Y, one back substitution per Q~ row.
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
constexpr int kRThreads = 128;               // four warps: one per tensor-memory lane quadrant
// Two CTAs per SM, each with one item in flight: while one waits on its loads or its chain of
// dependent phases, the other computes.  Shared memory of a CTA: a 32 KB state blob (MN-major B
// operand), a 32 KB [K~0; K~1; Q~0; Q~1] tile (K-major, 128B swizzle; once the products have read
// it, the R~ and Y tiles live there), the views' v~ rows (two 64-column halves of [2B rows x
// 128 B], 8 KB apart) and the fp32 scratch.  The next item's state blob is loaded as soon as the
// state product has read this one; its other tiles once Y R~ is done.
constexpr int R_OFF_S = 0, R_OFF_A = 32768, R_OFF_V = 65536;
constexpr int R_OFF_RT = R_OFF_A;            // R~ bf16, MN-major B operand: two N-halves of [2B x 128 B]
constexpr int R_OFF_Y = R_OFF_A + 16384;     // Y bf16, K-major A operand: 128 rows x 128 B
constexpr int R_OFF_X = 81920;               // fp32 scratch (see below)
// tensor memory: [0,128) [K~;Q~] S_e; [128,128+2B) [K~;Q~] K~^T, then (once read) [128,256) Y R~
constexpr uint32_t kTmemCols = 256;

struct R1Params {
    const float *gn, *betan;                 // [V, T_R, H]
    __nv_bfloat16 *out_noisy;                // [V, T_R, H, d]
    const uint8_t *states;                   // [T_R / B][H] blobs of 32 KB
    WorkspaceHeader *ws;
    int64_t TR;
    int32_t H, V, pairs;
    int32_t items;                           // (T_R / B) * H * pairs (< 2^31, checked on the host)
    float scale;                             // 1 / sqrt(d)
};

struct R1Maps {
    CUtensorMap qn, kn, vn;                  // box: 64 columns x 1 head x B rows
};

// One item: boundary state sidx = (block, head), and the pair of views v0, v0 + 1 (nv of them).
// 32-bit unsigned divisions (a 64-bit one is a long software sequence, paid three times per item).
struct RItem {
    uint32_t sidx;
    int h, v0, nv;
    int64_t row0;                            // the block's first packed response row
};

template <int B>
__device__ __forceinline__ RItem r1_item(uint32_t item, const R1Params &P) {
    RItem r;
    r.sidx = P.pairs == 1 ? item : item / (uint32_t)P.pairs;
    const uint32_t blk = r.sidx / (uint32_t)P.H;
    r.h = (int)(r.sidx - blk * (uint32_t)P.H);
    r.row0 = (int64_t)blk * B;
    r.v0 = 2 * (int)(item - r.sidx * (uint32_t)P.pairs);
    r.nv = min(2, P.V - r.v0);
    return r;
}

template <int B>
struct RLayout {
    // fp32 scratch after the tiles: A~ per view (row i written by row i's lane, read back as
    // 16-byte broadcasts by the back substitution), the block's log2-decays and betas per view.
    static constexpr int BS = B + 4;                          // row stride (16-byte aligned rows)
    static constexpr int AM = 0;                              // [2][B][BS]
    static constexpr int GAM = AM + 2 * B * BS;               // [2][B]
    static constexpr int BETA = GAM + 2 * B;                  // [2][B]
    static constexpr int FLOATS = BETA + 2 * B;
    static constexpr int RT_LBO = 2 * B * 128;                // R~: bytes between its two N-halves
    static constexpr int SMEM = R_OFF_X + FLOATS * 4 + 1024;  // + alignment slack
};

// Column l of view w's [K~0; K~1]^T block in a 32-column tensor-memory load (B = 16: both views in
// one load; B = 32: one view each): constant indices, so the loaded values stay in registers.
template <int B>
__device__ __forceinline__ float col_of(const float (&xr)[32], int w, int l) {
    if constexpr (B == 16) return w ? xr[16 + l] : xr[l];
    else return xr[l];
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Per item the chain is: loads -> [K~;Q~] K~^T, then [K~;Q~] S_e, on the tensor cores -> rows on
// CUDA cores (A~ rows to fp32 scratch; the decayed Q~K~^T rows M~_j = e^{gamma~_B - gamma~_l}
// q~_j.k~_l in registers; R~ to a bf16 operand tile) -> per Q~ row the coefficients
// Y_j = M~_j (I + A~)^-1 by back substitution (so that sum_i M~_ji u~_i = Y_j R~) into a bf16
// operand tile, block-diagonal over the two views -> Y R~ on the tensor cores -> the next item's
// loads -> o~_j = (Gamma~_B (Q~ S_e)_j + (Y R~)_j) / sqrt(d) from tensor memory to the output rows.
template <int B>
__global__ void __launch_bounds__(kRThreads, 2)
gdn_route1_refine_kernel(const __grid_constant__ R1Params P, const __grid_constant__ R1Maps M) {
    using L = RLayout<B>;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    float *X = reinterpret_cast<float *>(sm + R_OFF_X);
    __shared__ uint64_t bar_lds, bar_ld, bar_mma, bar_mma1, bar_mma2, bar_drain;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5;
    constexpr float kLog2e = 1.4426950408889634f;

    if (tid == 0) {
        mbar_init(&bar_lds, 1);
        mbar_init(&bar_ld, 1);
        mbar_init(&bar_mma, 1);
        mbar_init(&bar_mma1, 1);
        mbar_init(&bar_mma2, 1);
        mbar_init(&bar_drain, 1);
        fence_mbar_init();
        s_abort = 0;
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(&s_tmem, kTmemCols);
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
    // (thread 0) an item's loads: the state blob (bar_lds), the views' k~, q~ rows (rows 0..4B of the
    // A tile) and v~ rows (bar_ld)
    uint32_t loads_s = 0, loads = 0;                 // loads issued (mbarrier phases)
    auto issue_state = [&](const RItem &it) {
        ++loads_s;
        mbar_arrive_expect_tx(&bar_lds, 32768u);
        bulk_load(sm + R_OFF_S, P.states + (int64_t)it.sidx * 32768, 32768u, &bar_lds);
    };
    auto issue_loads = [&](const RItem &it) {
        ++loads;
        mbar_arrive_expect_tx(&bar_ld, (uint32_t)(it.nv * 6 * B * 128));
        for (int w = 0; w < it.nv; ++w) {
            const int row = (int)((int64_t)(it.v0 + w) * P.TR + it.row0);
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_3d(sm + R_OFF_A + hf * 16384 + (w * B) * 128, &M.kn, &bar_ld, hf * 64, it.h, row);
                tma_load_3d(sm + R_OFF_A + hf * 16384 + (2 * B + w * B) * 128, &M.qn, &bar_ld, hf * 64, it.h, row);
                tma_load_3d(sm + R_OFF_V + hf * 8192 + (w * B) * 128, &M.vn, &bar_ld, hf * 64, it.h, row);
            }
        }
    };
    // (threads < 2B) the block's g~ and beta~ of an item for lane (view, row), zeros for an absent view
    auto load_gb = [&](const RItem &it, bool valid, float &gl, float &bt) {
        gl = 0.f;
        bt = 0.f;
        const int w = tid / B, i = tid - w * B;
        if (tid < 2 * B && valid && w < it.nv) {
            const int64_t idx = ((int64_t)(it.v0 + w) * P.TR + it.row0 + i) * P.H + it.h;
            gl = __ldg(P.gn + idx) * kLog2e;
            bt = __ldg(P.betan + idx);
        }
    };
    // this thread's tile row t (TMEM lane t); its role (K~ rows, Q~ rows, none) is uniform over the
    // warp because 2B and 4B are multiples of 32, so every lane of a warp runs the same
    // tensor-memory loads
    const int t = tid, kind = t / B, i = t - kind * B, w = kind & 1;
    const int role = t < 2 * B ? 0 : (t < 4 * B ? 1 : 2);
    uint32_t k = 0;                                  // items done by this CTA (mbarrier phases)
    bool issued = false, stop = false;
    RItem nxt = r1_item<B>(blockIdx.x, P);
    if (tid == 0 && (int)blockIdx.x < P.items) {
        issue_state(nxt);
        issue_loads(nxt);
    }
    float gl_next, bt_next;
    load_gb(nxt, (int)blockIdx.x < P.items, gl_next, bt_next);
    for (int item = blockIdx.x; item < P.items; item += gridDim.x, ++k) {
        const RItem cur = nxt;
        const bool more = item + (int)gridDim.x < P.items;
        if (more) nxt = r1_item<B>(item + gridDim.x, P);
        const bool active = kind < 4 && w < cur.nv;
        // ---- the block's decays and betas (log2 units, loaded an item ahead): one lane per (view,
        //      row), the inclusive cumulative sum by a shuffle scan over each view's B lanes
        float gl = gl_next, bt = bt_next;
        load_gb(nxt, more, gl_next, bt_next);
        if (tid < 2 * B) {
#pragma unroll
            for (int o = 1; o < B; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, gl, o, B);
                if (i >= o) gl += up;
            }
            X[L::GAM + w * B + i] = gl;
            X[L::BETA + w * B + i] = bt;
        }
        if (!wait_ok(&bar_ld, k & 1, 101) || !wait_ok(&bar_lds, k & 1, 105)) stop = true;
        __syncwarp();
        if (tid == 0 && !stop) {
            tc_fence_after();
            const uint64_t dA = make_sdesc(smem_u32(sm + R_OFF_A), 16, 1024);
            const uint64_t dS = make_sdesc(smem_u32(sm + R_OFF_S), 16384, 1024);
            // [K~;Q~] K~^T first (the rows' coefficients wait for it alone), then [K~;Q~] S_e
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(tb + 128, dA + (off >> 4), dA + (off >> 4), make_idesc_bf16(128, 2 * B, 0, 0), kk > 0);
            }
            mma_commit(&bar_mma);
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(tb, dA + (off >> 4), dS + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 0, 1), kk > 0);
            }
            mma_commit(&bar_mma1);
            issued = true;
        }
        __syncwarp();
        if (!stop && !wait_ok(&bar_mma, k & 1, 102)) stop = true;
        __syncwarp();
        tc_fence_after();
        if ((stop = __syncthreads_or(stop))) break;
        // ---- rows.  A row of a view this item does not have writes zeros (K~ rows: its A~ row and
        //      R~ row, so that the other view's products stay finite) or nothing (Q~ rows).  The K~
        //      rows' warps write A~, release the Q~ rows' back substitution by a producer/consumer
        //      barrier, then form R~ once the state product is done.
        const float *gam = X + L::GAM + w * B, *beta = X + L::BETA + w * B;
        float *Am = X + L::AM + w * B * L::BS;
        float xr[32];
        bool ok = true;
        if (role == 0) {
            // row i of A~: A~_il = beta~_i e^{gamma~_i - gamma~_l} k~_i.k~_l (l < i)
            const float bi = active ? beta[i] : 0.f;
            tmem_ld32(tmem_addr(tb, warp * 32, 128 + 32 * ((w * B) / 32)), xr);
            tmem_wait_ld();
            {
                float ar[B];
#pragma unroll
                for (int l = 0; l < B; ++l)
                    ar[l] = (active && l < i) ? bi * exp2f(gam[i] - gam[l]) * col_of<B>(xr, w, l) : 0.f;
#pragma unroll
                for (int c4 = 0; c4 < B / 4; ++c4)
                    *reinterpret_cast<float4 *>(Am + i * L::BS + 4 * c4) =
                        make_float4(ar[4 * c4], ar[4 * c4 + 1], ar[4 * c4 + 2], ar[4 * c4 + 3]);
            }
            asm volatile("bar.arrive 1, 128;" ::: "memory");
            // R~_i = beta~_i v~_i - beta~_i Gamma~_i (K~ S_e)_i -> row i of the R~ tile (bf16), over
            // the state blob that the state product has finished reading
            if (!wait_ok(&bar_mma1, k & 1, 104)) ok = false;
            __syncwarp();
            tc_fence_after();
            // the state product has read the blob (and the A tile): the next item's blob can come
            if (tid == 0 && ok && more) issue_state(nxt);
            const float bg = active ? bi * exp2f(gam[i]) : 0.f;
#pragma unroll
            for (int c0 = 0; c0 < RD; c0 += 32) {
                tmem_ld32(tmem_addr(tb, warp * 32, c0), xr);
                tmem_wait_ld();
                const int hf = c0 >> 6;
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    const int c8 = ((c0 & 63) >> 3) + e8;
                    uint4 o = make_uint4(0u, 0u, 0u, 0u);
                    if (active && ok) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(sm + R_OFF_V + hf * 8192 + sw128_off(t, c8));
                        const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
                        uint32_t r[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const float va = __uint_as_float(wv[p] << 16), vb = __uint_as_float(wv[p] & 0xffff0000u);
                            r[p] = bf16x2(bi * va - bg * xr[8 * e8 + 2 * p], bi * vb - bg * xr[8 * e8 + 2 * p + 1]);
                        }
                        o = make_uint4(r[0], r[1], r[2], r[3]);
                    }
                    if (ok) *reinterpret_cast<uint4 *>(sm + R_OFF_RT + hf * L::RT_LBO + sw128_off(t, c8)) = o;
                }
            }
        } else if (role == 1) {
            float mq[B];                                     // M~_j
            tmem_ld32(tmem_addr(tb, warp * 32, 128 + 32 * ((w * B) / 32)), xr);    // q~_j . k~_l
            tmem_wait_ld();
            const float gB = gam[B - 1];
#pragma unroll
            for (int l = 0; l < B; ++l) mq[l] = exp2f(gB - gam[l]) * col_of<B>(xr, w, l);
            asm volatile("bar.sync 1, 128;" ::: "memory");   // A~ complete
            if (active) {
                // the Y tile overlays the A tile: the state product must have read it
                if (!wait_ok(&bar_mma1, k & 1, 106)) ok = false;
                // Y (I + A~) = M~ by right-looking back substitution: y_m = (what is left of) m_m is
                // final once rows m+1.. are taken out, then y_m A~_ml leaves every l < m at once.  Row
                // m's loads do not depend on y, and entry m-1 is updated first, so the dependent
                // chain is about one FMA per row.
                float *y = mq;                               // in place
#pragma unroll
                for (int m = B - 1; m >= 1; --m) {
                    const float *row = Am + m * L::BS;       // A~_ml, l < m (broadcast loads)
                    const int cm = (m - 1) >> 2;             // the 16-byte group holding l = m - 1
#pragma unroll
                    for (int g = 0; g <= cm; ++g) {
                        const int c4 = g == 0 ? cm : g - 1;
                        const float4 a = *reinterpret_cast<const float4 *>(row + 4 * c4);
                        const float av[4] = {a.x, a.y, a.z, a.w};
                        if (g == 0) y[m - 1] = fmaf(-y[m], av[(m - 1) & 3], y[m - 1]);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (4 * c4 + e < m - 1) y[4 * c4 + e] = fmaf(-y[m], av[e], y[4 * c4 + e]);
                    }
                }
                // row t of the Y tile: this view's B coefficients, zeros in the other view's columns
#pragma unroll
                for (int c8 = 0; c8 < 2 * B / 8 && ok; ++c8) {
                    uint4 o = make_uint4(0u, 0u, 0u, 0u);
                    if ((c8 * 8) / B == w) {
                        const int l0 = (c8 * 8) % B;
                        o = make_uint4(bf16x2(y[l0], y[l0 + 1]), bf16x2(y[l0 + 2], y[l0 + 3]),
                                       bf16x2(y[l0 + 4], y[l0 + 5]), bf16x2(y[l0 + 6], y[l0 + 7]));
                    }
                    *reinterpret_cast<uint4 *>(sm + R_OFF_Y + sw128_off(t, c8)) = o;
                }
            }
        } else {
            asm volatile("bar.arrive 1, 128;" ::: "memory");
        }
        fence_async_smem();                                  // R~ and Y tiles -> tensor cores
        tc_fence_before();
        if ((stop = __syncthreads_or(!ok))) break;
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dY = make_sdesc(smem_u32(sm + R_OFF_Y), 16, 1024);
            const uint64_t dRT = make_sdesc(smem_u32(sm + R_OFF_RT), L::RT_LBO, 1024);
            // Y R~ into the columns of [K~;Q~] K~^T, read by now
            for (int kk = 0; kk < 2 * B / 16; ++kk)
                mma_bf16(tb + 128, dY + ((kk * 32) >> 4), dRT + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 0, 1),
                         kk > 0);
            mma_commit(&bar_mma2);
        }
        __syncwarp();
        if (!wait_ok(&bar_mma2, k & 1, 103)) stop = true;
        __syncwarp();
        tc_fence_after();
        if ((stop = __syncthreads_or(stop))) break;
        // every tile has been read: the next item's loads overlap this read-out
        if (tid == 0 && more) issue_loads(nxt);
        // ---- read-out: the Q~ rows' warps
        if (role == 1) {
            const int j = i;
            const float GB = exp2f(gam[B - 1]);
            __nv_bfloat16 *orow = P.out_noisy + (((int64_t)(cur.v0 + w) * P.TR + cur.row0 + j) * P.H + cur.h) * RD;
            float qs[32], yr[32];
#pragma unroll
            for (int c0 = 0; c0 < RD; c0 += 32) {
                tmem_ld32(tmem_addr(tb, warp * 32, c0), qs);
                tmem_ld32(tmem_addr(tb, warp * 32, 128 + c0), yr);
                tmem_wait_ld();
                if (active) {
#pragma unroll
                    for (int e8 = 0; e8 < 32; e8 += 8) {
                        uint32_t r[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const int e = e8 + 2 * p;
                            r[p] = bf16x2(fmaf(GB, qs[e], yr[e]) * P.scale, fmaf(GB, qs[e + 1], yr[e + 1]) * P.scale);
                        }
                        *reinterpret_cast<uint4 *>(orow + c0 + e8) = make_uint4(r[0], r[1], r[2], r[3]);
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();          // tensor memory and scratch are free for the next item
    }
    // drain (only when a wait gave up): the last load and the MMAs
    if (stop && tid == 0) {
        if (loads_s) mbar_wait(&bar_lds, (loads_s - 1) & 1, kDrainWaitIters);
        if (loads) mbar_wait(&bar_ld, (loads - 1) & 1, kDrainWaitIters);
        if (issued) {
            mma_commit(&bar_drain);
            mbar_wait(&bar_drain, 0, kDrainWaitIters);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, kTmemCols);
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
    R.out_noisy = static_cast<__nv_bfloat16 *>(p.out_noisy);
    R.states = static_cast<const uint8_t *>(p.states);
    R.ws = p.ws;
    R.TR = p.TR;
    R.H = p.H;
    R.V = p.V;
    R.pairs = (p.V + 1) / 2;
    const int64_t items = (p.TR / B) * p.H * R.pairs;
    if (items >= (int64_t(1) << 31) - 1024) return cudaErrorNotSupported;
    R.items = (int32_t)items;
    R.scale = p.scale;
    if (R.items == 0) return cudaSuccess;
    R1Maps maps;
    if (!r1_map(&maps.qn, p.qn, p.H, (int64_t)p.V * p.TR, B) || !r1_map(&maps.kn, p.kn, p.H, (int64_t)p.V * p.TR, B) ||
        !r1_map(&maps.vn, p.vn, p.H, (int64_t)p.V * p.TR, B))
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
    const int64_t grid = std::min<int64_t>(R.items, 2 * (int64_t)sms);     // two CTAs per SM
    gdn_route1_refine_kernel<B><<<(unsigned)grid, kRThreads, RLayout<B>::SMEM, stream>>>(R, maps);
    return cudaGetLastError();
}

}  // namespace

// (ShortConv runs as a pass of its own before both stages, so the kernels never see it)
bool route1_tc_supported(int dtype, int d, int B, int conv_width) {
    return dtype == GDN_BF16 && d == RD && (B == 16 || B == 32) && (conv_width == 0 || conv_width == 4);
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
