// gdn_pipe.cu -- dual-stream Gated DeltaNet forward without the ShortConv prologue: the chunked
// WY/UT form on tcgen05 tensor cores (sm_100a), pipelined across chunks by warp specialisation.
// bf16 I/O, fp32 state and accumulation, d_k = d_v = 128, chunks of C = 64 tokens.
//
// Method ("FLARE: Diffusion for Hybrid Language Model", papernotes.org notes, Method > Key
// design 2): clean causal gated delta rule
//     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t / sqrt(d),
// and a block-bidirectional noisy stream in which block b of every view restarts from the clean
// state S_{e(b-1)}, runs its B noisy tokens and every position reads the block-end state.  The
// algebra is the one of gdn_chunked.cu (the in-order kernel, which also carries the ShortConv
// prologue): per chunk, with gamma the inclusive cumulative log2-decay,
//   A = strictly lower (beta_t 2^{gamma_t-gamma_i} k_t.k_i),  T = (I + A)^{-1},
//   P = lower (2^{gamma_t-gamma_i} q_t.k_i),  R = beta V - beta Gamma K S0,
//   [P U ; U] = [P T ; T] R,  O = Gamma Q S0 + P U,  S_C = Gamma_C S0 + Khat^T U,
// and each noisy row j (block boundary e) is one more row against the chunk:
//   o~_j = Gamma_e Z_j S0 + M'_Z,j U + W~V~_j,   M'_Z,ji = (Gamma_e Z_j . k_i) 2^{-gamma_i} [i <= e].
//
// Schedule.  Only R, [P U; U], S_C and the noisy rows' S0 / U products depend on the state; the
// triangular solve and everything else of the clean stream depends on the chunk's inputs alone.
// So the CTA runs two groups of warps one chunk apart:
//   main warps 0-7 (chunk c): the noisy rows' block coefficients, Z rows and M'_Z, and the state
//       chain  [Q;K] S0 -> R -> [P T;T] R -> O, U -> Khat^T U -> S_C,  fp32 state in registers;
//   helper warps 8-11 (chunk c+1): the chunk's scalars (cumulative decays), [Q;K] K^T, the A and P
//       rows, T = (I + A)^{-1}, P T, [P T; T] and Khat, handed to the main warps through shared
//       memory.
// The helpers own 64 columns of tensor memory and their own MMA-issuing thread; the groups meet
// only at mbarriers (each side waits for the other's products, or for the MMA that frees a buffer).
// Registers are split by setmaxnreg: 176 per main thread, 152 per helper thread.
//
// Persistent CTAs (one per SM) take (document, head) work items longest first from a counter in the
// workspace; the helpers fetch the items and publish one chunk descriptor per chunk.  Every wait
// is bounded; a wait that gives up records GDN_ERR_TIMEOUT, and before the CTA frees its tensor
// memory each issuing thread waits for the copies and MMAs it has issued.
#include <algorithm>

#include "gdn_chunk_common.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kMainThreads = 256;             // warps 0-7
constexpr int kHelpThreads = 128;             // warps 8-11 (one warpgroup)
constexpr int kPipeThreads = kMainThreads + kHelpThreads;
constexpr int kLaunchRegs = 168;              // per thread at launch (65536 / 384, rounded to 8)
constexpr int kMainRegs = 176, kHelpRegs = 152;
static_assert(kMainThreads * kMainRegs + kHelpThreads * kHelpRegs <= kPipeThreads * kLaunchRegs,
              "the register split must fit the registers the block is launched with");

// Shared memory (offsets from a 1024-byte aligned base)
constexpr int Q_S0 = 0;          // 32 KB  S0 bf16, MN-major B: 2 v-halves x [128 k-rows x 128 B]
constexpr int Q_QK = 32768;      // 32 KB  [Q;K] K-major: 2 d-halves x [Q 64 rows | K 64 rows]
constexpr int Q_V = 65536;       // 16 KB  V -> R -> U, MN-major: 2 v-halves x [64 rows x 128 B]
constexpr int Q_KH = 81920;      // 16 KB  Khat: MN-major A (Khat^T U) and K-major B (Z Khat^T)
constexpr int Q_Y = 98304;       // 16 KB  helpers: fp32 solve scratch -> [P;T] -> [P T;T] (K-major A)
constexpr int Q_NQ = 114688;     // 32 KB  [q~0;q~1] -> Gamma_e Z, K-major
constexpr int Q_NK = 147456;     // 32 KB  [k~0;k~1] K-major (and MN-major B)
constexpr int Q_NV = 180224;     // 32 KB  [v~0;v~1] per v-half; v-half 0 later holds M'_Z (K-major)
constexpr int Q_W = 212992;      //  4 KB  helpers: the 32-merge's result (32x32 fp32)
constexpr int Q_SMEM_BYTES = 217088 + 1024;

// Tensor memory columns (512): main warps R0, R1, N, ZK; helpers H.
constexpr uint32_t P_R0 = 0;     // q~k~^T | W~ (A) [0,64) and -Y~ (A) [64,128) | -Y~K~ d-half 0 | [P U; U]
constexpr uint32_t P_R1 = 128;   // k~k~^T | [Q;K] S0 | dS
constexpr uint32_t P_N = 256;    // noisy accumulator: W~V~ + Gamma_e Z S0 + M'_Z U
constexpr uint32_t P_ZK = 384;   // -Y~K~ d-half 1 | Z Khat^T
constexpr uint32_t P_H = 448;    // helpers: [Q;K] K^T | P T

__device__ __forceinline__ void bar_main() { asm volatile("bar.sync 1, %0;" ::"n"(kMainThreads) : "memory"); }
__device__ __forceinline__ void bar_help() { asm volatile("bar.sync 2, %0;" ::"n"(kHelpThreads) : "memory"); }
// The same barriers, returning whether any thread of the group saw the CTA abort (uniform result).
__device__ __forceinline__ bool bar_main_abort(const int *s_abort) {
    return bar_sync_or(1, kMainThreads, *reinterpret_cast<const volatile int *>(s_abort) != 0);
}
__device__ __forceinline__ bool bar_help_abort(const int *s_abort) {
    return bar_sync_or(2, kHelpThreads, *reinterpret_cast<const volatile int *>(s_abort) != 0);
}

// Chunk descriptor published by the helpers: unit (-1: no more work), chunk index m (relative to
// the response start; negative in the prompt), and whether the chunk's decays factorise.
struct ChunkDesc {
    int unit, m, fact;
};

// Clean and noisy per-chunk scalars: [gamma | beta | E = 2^gamma | F = 2^-gamma] for the 64 clean
// rows, then [gamma~ | beta~ (| E~ | F~ for B >= 16)] for the 128 noisy rows of both views.
constexpr int SC_GAM = 0, SC_BETA = CH, SC_E = 2 * CH, SC_F = 3 * CH, SC_NGAM = 4 * CH, SC_NBETA = 6 * CH;
constexpr int SC_NE = 8 * CH, SC_NF = 10 * CH;

// T = (I + A)^{-1} for the strictly lower 64x64 A in the fp32 scratch, by the four helper warps:
// warps 0-1 invert the eight 8x8 diagonal blocks (one thread per column, right-looking forward
// substitution), each warp runs one 8-merge, two warps each 16-merge (in place, a barrier between
// their reads and writes), and all four the 32-merge, 8 columns per warp, whose lower-left block
// goes to the 32 x 32 staging block `wb` (rows 32..63, columns 0..31 of T) so that no warp
// overwrites A while another still reads it.
__device__ void solve_T_help(float *sa, float *wb, int ht, int hw, int lane) {
    if (ht < 64) {
        const int o = (ht >> 3) * 8, c = ht & 7;
        float a[8][8], x[8];
#pragma unroll
        for (int jj = 1; jj < 8; ++jj) {
#pragma unroll
            for (int l = 0; l < jj; ++l) a[jj][l] = sa[sidx(o + jj, o + l)];
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) x[jj] = (jj == c) ? 1.f : 0.f;
#pragma unroll
        for (int l = 0; l < 8; ++l) {
#pragma unroll
            for (int jj = l + 1; jj < 8; ++jj) x[jj] = fmaf(-a[jj][l], x[l], x[jj]);
        }
        __syncwarp();
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) sa[sidx(o + jj, o + c)] = x[jj];
    }
    bar_help();
    auto in_place = [sa](int o, int S) {
        return [sa, o, S](int r, int c, float v) { sa[sidx(o + S + r, o + c)] = v; };
    };
    {
        const int o = 16 * hw;
        warp_merge<8, 8>(sa, o, 0, lane, in_place(o, 8), [] {});
    }
    bar_help();
    {
        const int o = 32 * (hw >> 1), cb = 8 * (hw & 1);
        warp_merge<16, 8>(sa, o, cb, lane, in_place(o, 16), [] { bar_help(); });
    }
    bar_help();
    warp_merge<32, 8>(sa, 0, 8 * hw, lane, [&](int r, int c, float v) { wb[widx(r, c)] = v; }, [] {});
    bar_help();
}

// TW: the test instantiation, whose waits poll with the caller's bound (gdn_dual_forward_test_wait_limit).
template <int B, bool TW = false>
__global__ void __launch_bounds__(kPipeThreads, 1)
gdn_pipe_kernel(const __grid_constant__ Params P, const __grid_constant__ Maps M) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    // TMA barriers (issued by thread 0): [Q;K], V, q~, k~, v~.
    __shared__ uint64_t bar_qk, bar_v, bar_nq, bar_nk, bar_nv;
    // MMA commit barriers of the main issuer (thread 0) and of the helper issuer (thread 256).
    __shared__ uint64_t bar_pk1n, bar_b1, bar_b2, bar_pk2n, bar_s2, bar_s3, bar_pk1c, bar_pk2c;
    // Helper -> main hand-offs: descriptor and scalars (two barriers, by chunk parity), [P T;T] in
    // Y, Khat in KH.
    __shared__ uint64_t bar_hs[2], bar_hy, bar_hk;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ ChunkDesc s_desc[2];
    __shared__ float s_sc[2][(B >= 16 ? 12 : 8) * CH];
    __shared__ int s_okn[2][4];               // every |gamma~| of a 32-row noisy group below 100
    __shared__ float s_g[CH];                 // helpers: scan scratch
    __shared__ float s_raw[2][3 * CH];        // helpers: [gate, beta][row] staged by cp.async
    __shared__ int s_next;
    __shared__ int s_fact[2];
    // Timeout drain: per issuing thread and mbarrier, phases issued and phases seen complete.
    // [0..4] TMA (qk, v, nq, nk, nv), [5..10] main MMA (pk1n, b1, b2, pk2n, s2, s3), [11, 12] helper MMA.
    __shared__ uint32_t s_iss[13], s_ok[13];

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const bool is_main = tid < kMainThreads;
    const int H = P.H, V = P.V;
    const int64_t TR = P.TR;
    const float scale = P.scale;
    constexpr float kLog2e = 1.4426950408889634f;

    if (tid == 0) {
        for (uint64_t *b : {&bar_qk, &bar_v, &bar_nq, &bar_nk, &bar_nv, &bar_pk1n, &bar_b1, &bar_b2, &bar_pk2n,
                            &bar_s2, &bar_s3, &bar_pk1c, &bar_pk2c, &bar_hy, &bar_hk, &bar_hs[0], &bar_hs[1]})
            mbar_init(b, 1);
        fence_mbar_init();
        s_abort = 0;
        for (int i = 0; i < 13; ++i) s_iss[i] = s_ok[i] = 0;
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
        if (lane == 0) {
            prefetch_tmap(&M.q); prefetch_tmap(&M.k); prefetch_tmap(&M.v);
            prefetch_tmap(&M.qn); prefetch_tmap(&M.kn); prefetch_tmap(&M.vn);
        }
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
    // Error path: once one of this thread's waits has given up, or the CTA is aborting, the thread
    // waits on nothing more; its group leaves at its next abort check.  `cnt` >= 0 counts the
    // completion for the drain (issuing threads only).
    bool dead = false;
    auto wait_bar = [&](uint64_t *bar, uint32_t parity, int cnt, int where) {
        if (!dead && *reinterpret_cast<volatile int *>(&s_abort)) dead = true;
        if (dead) return;
        if (kwait<TW>(bar, parity, kWaitIters, P.wait_iters)) {
            if (cnt >= 0) ++s_ok[cnt];
        } else {
            dead = true;
            fail(where);
        }
    };

    const uint32_t a_s0 = smem_u32(sm + Q_S0), a_qk = smem_u32(sm + Q_QK), a_v = smem_u32(sm + Q_V);
    const uint32_t a_kh = smem_u32(sm + Q_KH), a_y = smem_u32(sm + Q_Y), a_nq = smem_u32(sm + Q_NQ);
    const uint32_t a_nk = smem_u32(sm + Q_NK), a_nv = smem_u32(sm + Q_NV);

    if (is_main) {
        // =========================================================================== main warps
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kMainRegs));
        const int q = warp & 3, ch = (warp >> 2) & 1, rho = q * 32 + lane;   // TMEM lane and column half
        // Shared-memory matrix descriptors (built where the MMAs are issued, so that they hold no
        // registers across the loop): K-major [Q;K] (A; its K rows as B), [q~;.] / Z, [k~0;k~1],
        // Khat as B, [P T;T] and M'_Z; MN-major S0, R / U, Khat (A), [v~0;v~1], [k~0;k~1].
#define dK_qk make_sdesc(a_qk, 16, 1024)
#define dK_nq make_sdesc(a_nq, 16, 1024)
#define dK_nk make_sdesc(a_nk, 16, 1024)
#define dK_kh make_sdesc(a_kh, 16, 1024)
#define dK_y make_sdesc(a_y, 16, 1024)
#define dK_mz make_sdesc(a_nv, 16, 1024)
#define dM_s0 make_sdesc(a_s0, 16384, 1024)
#define dM_v make_sdesc(a_v, 8192, 1024)
#define dM_kh make_sdesc(a_kh, 8192, 1024)
#define dM_nv make_sdesc(a_nv, 16384, 1024)

        // TMA loads of chunk (U, m), issued by thread 0.
        auto load = [&](int which, const Unit &U, int m) {
            const int cstart = U.s + U.prompt + CH * m;
            ++s_iss[which];
            if (which == 0) {            // [Q;K]
                mbar_arrive_expect_tx(&bar_qk, 32768u);
                for (int hf = 0; hf < 2; ++hf) {
                    tma_load_3d(sm + Q_QK + hf * 16384, &M.q, &bar_qk, hf * 64, U.h, cstart);
                    tma_load_3d(sm + Q_QK + hf * 16384 + 8192, &M.k, &bar_qk, hf * 64, U.h, cstart);
                }
            } else if (which == 1) {     // V
                mbar_arrive_expect_tx(&bar_v, 16384u);
                for (int hf = 0; hf < 2; ++hf) tma_load_3d(sm + Q_V + hf * 8192, &M.v, &bar_v, hf * 64, U.h, cstart);
            } else {                     // q~, k~ or v~ of both views
                uint64_t *bar = which == 2 ? &bar_nq : (which == 3 ? &bar_nk : &bar_nv);
                const CUtensorMap *map = which == 2 ? &M.qn : (which == 3 ? &M.kn : &M.vn);
                uint8_t *dst = sm + (which == 2 ? Q_NQ : (which == 3 ? Q_NK : Q_NV));
                mbar_arrive_expect_tx(bar, 32768u);
                for (int vw = 0; vw < 2; ++vw) {
                    const int row = vw * (int)TR + U.roff + CH * m;
                    for (int hf = 0; hf < 2; ++hf) tma_load_3d(dst + hf * 16384 + vw * 8192, map, bar, hf * 64, U.h, row);
                }
            }
        };
        auto commit = [&](uint64_t *bar, int which) {
            mma_commit(bar);
            ++s_iss[which];
        };

        float S[64];
        uint32_t gc = 0, gnc = 0;     // chunks, and chunks with noisy rows, processed by this CTA
        Unit U{};
        int cur_unit = -1;
        for (;;) {
            // ---- the helpers' descriptor and scalars for chunk gc ----
            wait_bar(&bar_hs[gc & 1], (gc >> 1) & 1, -1, 60);
            if (bar_main_abort(&s_abort)) break;
            const ChunkDesc cd = s_desc[gc & 1];
            if (cd.unit < 0) break;
            if (cd.unit != cur_unit) {
                U = make_unit(P, cd.unit);
                cur_unit = cd.unit;
            }
            const int m = cd.m;
            const bool noisy = m >= 0 && V > 0;
            const bool first = m == U.m_first, last = m == U.m_first + U.nchunks - 1;
            const bool fact = cd.fact != 0;
            const int cstart = U.s + U.prompt + CH * m;
            const float *sc = s_sc[gc & 1];
            const float *s_beta = sc + SC_BETA, *s_E = sc + SC_E, *s_F = sc + SC_F, *s_gam = sc + SC_GAM;
            // read now: once S3 of this chunk completes, the helpers may overwrite this scalar buffer
            const float GC = s_E[CH - 1];
            if (gc == 0 && tid == 0) {           // the very first chunk: nothing was prefetched
                load(0, U, m);
                load(1, U, m);
                if (noisy) {
                    load(2, U, m);
                    load(3, U, m);
                    load(4, U, m);
                }
            }
            if (first) {
#pragma unroll
                for (int c = 0; c < 64; ++c) S[c] = 0.f;
                uint8_t *s0 = sm + Q_S0 + ch * 16384;
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) *reinterpret_cast<uint4 *>(s0 + sw128_off(rho, c8)) = z;
                fence_async_smem();
            }

            // ---- noisy rows: block products, then the block coefficients as A operands ----
            float gend = 0.f;
            if (noisy) {
                wait_bar(&bar_nq, gnc & 1, tid == 0 ? 2 : -1, 61);
                wait_bar(&bar_nk, gnc & 1, tid == 0 ? 3 : -1, 62);
                if (tid == 0) {
                    tc_fence_after();
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_bf16(tb + P_R0, dK_nq + (off >> 4), dK_nk + (off >> 4), make_idesc_bf16(128, 128, 0, 0), kk > 0);
                        mma_bf16(tb + P_R1, dK_nk + (off >> 4), dK_nk + (off >> 4), make_idesc_bf16(128, 128, 0, 0), kk > 0);
                    }
                    commit(&bar_pk1n, 5);
                }
                __syncwarp();
                wait_bar(&bar_pk1n, gnc & 1, tid == 0 ? 5 : -1, 63);
                __syncwarp();
                tc_fence_after();
                {
                    float wq[32], wk[32];
                    tmem_ld32(tmem_addr(tb, q * 32, P_R0 + 32 * q), wq);
                    tmem_ld32(tmem_addr(tb, q * 32, P_R1 + 32 * q), wk);
                    tmem_wait_ld();
                    const int vw = rho >> 6, j = rho & 63;
                    const bool nfact = B >= 16 && s_okn[gc & 1][0] && s_okn[gc & 1][1] && s_okn[gc & 1][2] &&
                                       s_okn[gc & 1][3];
                    float ycoef[B], wcoef[B];
                    const float *nE = sc + (B >= 16 ? SC_NE : 0), *nF = sc + (B >= 16 ? SC_NF : 0);
                    // the block rows travel by warp shuffles (no shared memory is free to stage them)
                    noisy_coeffs<B, false>(wq, wk, lane, j, sc + SC_NGAM + 64 * vw, sc + SC_NBETA + 64 * vw,
                                           nE + 64 * vw, nF + 64 * vw, nfact, nullptr, ycoef, wcoef, gend);
                    tc_fence_before();
                    bar_main();          // every thread has read R0 and R1 before R0 is overwritten
                    tc_fence_after();
                    const int bs = (j / B) * B;
                    store_block_row<B>(tmem_addr(tb, q * 32, P_R0 + 32 * ch), ch, vw, bs, wcoef, 1.f);
                    store_block_row<B>(tmem_addr(tb, q * 32, P_R0 + 64 + 32 * ch), ch, vw, bs, ycoef, -1.f);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            if (bar_main_abort(&s_abort)) break;

            // ---- batch 1: [Q;K] S0 -> R1 and W~V~ -> N; batch 2: -Y~ K~ -> (R0, ZK) ----
            if (tid == 0) {
                wait_bar(&bar_qk, gc & 1, 0, 64);
                if (noisy) wait_bar(&bar_nv, gnc & 1, 4, 65);
                tc_fence_after();
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tb + P_R1, dK_qk + (off >> 4), dM_s0 + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 0, 1), kk > 0);
                }
                if (noisy)
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tb + P_N, tb + P_R0 + kk * 8, dM_nv + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 0, 1), kk > 0);
                commit(&bar_b1, 6);
            }
            __syncwarp();
            wait_bar(&bar_b1, gc & 1, tid == 0 ? 6 : -1, 66);
            __syncwarp();
            tc_fence_after();
            // the next chunk, once its descriptor is out
            ChunkDesc nd{-1, 0, 0};
            if (tid == 0) {
                if (noisy) {             // W~ (columns [0,64) of R0) is consumed: -Y~ K~ may overwrite it
                    for (int hf = 0; hf < 2; ++hf)
                        for (int kk = 0; kk < 8; ++kk)
                            mma_bf16_ts(tb + (hf == 0 ? P_R0 : P_ZK), tb + P_R0 + 64 + kk * 8,
                                        make_sdesc(a_nk + hf * 16384, 16384, 1024) + ((kk * 2048) >> 4),
                                        make_idesc_bf16(128, 64, 0, 1), kk > 0);
                    commit(&bar_b2, 7);
                }
                wait_bar(&bar_hs[(gc + 1) & 1], ((gc + 1) >> 1) & 1, -1, 67);
                nd = s_desc[(gc + 1) & 1];
                // [Q;K] of the next chunk: once the helpers have built this chunk's Khat from K, and,
                // when Z K^T reads K itself (decays that do not factorise), after that product
                wait_bar(&bar_hk, gc & 1, -1, 68);
                if (nd.unit >= 0 && !(noisy && !fact) && !dead) {
                    const Unit Un = nd.unit == cur_unit ? U : make_unit(P, nd.unit);
                    load(0, Un, nd.m);
                    if (!noisy && nd.m >= 0 && V > 0) {   // this chunk used no noisy tiles
                        load(2, Un, nd.m);
                        load(3, Un, nd.m);
                        load(4, Un, nd.m);
                    }
                }
            }
            __syncwarp();
            // ---- R = beta V - beta Gamma (K S0) over V (K S0: rows 64..127 of R1) ----
            wait_bar(&bar_v, gc & 1, tid == 0 ? 1 : -1, 69);
            if (rho >= 64) {
                const int t = rho - 64;
                const float bt = s_beta[t], bg = bt * s_E[t];
                uint8_t *vrow = sm + Q_V + ch * 8192;
                float ksb[2][32];
                tmem_ld32(tmem_addr(tb, q * 32, P_R1 + 64 * ch), ksb[0]);
                tmem_ld32(tmem_addr(tb, q * 32, P_R1 + 64 * ch + 32), ksb[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        float f[8];
                        const uint32_t o = sw128_off(t, 4 * hf + c4);
                        unpack8(*reinterpret_cast<const uint4 *>(vrow + o), f);
#pragma unroll
                        for (int x = 0; x < 8; ++x) f[x] = bt * f[x] - bg * ksb[hf][8 * c4 + x];
                        *reinterpret_cast<uint4 *>(vrow + o) = pack8(f);
                    }
                }
            }
            // ---- Z rows: Z_j = Gammatil_B q~_j + (-Y~K~)_j, written scaled by Gamma_e when the decays factorise ----
            if (noisy) {
                __syncwarp();
                wait_bar(&bar_b2, gnc & 1, tid == 0 ? 7 : -1, 70);
                __syncwarp();
                tc_fence_after();
                if (tid == 0 && nd.unit >= 0 && nd.m >= 0 && V > 0 && !dead)
                    load(3, nd.unit == cur_unit ? U : make_unit(P, nd.unit), nd.m);   // k~ is consumed
                __syncwarp();
                const int eb = ((rho & 63) / B) * B - 1;       // the row's block boundary (-1: S0)
                const float zs = (fact && eb >= 0) ? s_E[eb] : 1.f;
                const float Gend = exp2f(gend) * zs;
                uint8_t *nq = sm + Q_NQ + ch * 16384;
                float ykb[2][32];
                tmem_ld32(tmem_addr(tb, q * 32, (ch == 0 ? P_R0 : P_ZK)), ykb[0]);
                tmem_ld32(tmem_addr(tb, q * 32, (ch == 0 ? P_R0 : P_ZK) + 32), ykb[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const uint32_t o = sw128_off(rho, 4 * hf + c4);
                        float z[8];
                        unpack8(*reinterpret_cast<const uint4 *>(nq + o), z);
#pragma unroll
                        for (int e = 0; e < 8; ++e) z[e] = fmaf(Gend, z[e], zs * ykb[hf][8 * c4 + e]);
                        *reinterpret_cast<uint4 *>(nq + o) = pack8(z);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            if (bar_main_abort(&s_abort)) break;

            // ---- noisy: Z K^T (Khat when the decays factorise, else K) -> ZK, then M'_Z -> NV ----
            if (noisy) {
                if (tid == 0) {
                    tc_fence_after();
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        const uint64_t bdesc = fact ? dK_kh + ((((kk >> 2) * 8192) + (kk & 3) * 32) >> 4)
                                                    : dK_qk + ((8192 + off) >> 4);
                        mma_bf16(tb + P_ZK, dK_nq + (off >> 4), bdesc, make_idesc_bf16(128, 64, 0, 0), kk > 0);
                    }
                    commit(&bar_pk2n, 8);
                }
                __syncwarp();
                wait_bar(&bar_pk2n, gnc & 1, tid == 0 ? 8 : -1, 71);
                __syncwarp();
                tc_fence_after();
                if (tid == 0 && !fact && nd.unit >= 0 && !dead)     // Z K^T has read K
                    load(0, nd.unit == cur_unit ? U : make_unit(P, nd.unit), nd.m);
                __syncwarp();            // reconverge before warp-collective tcgen05.ld
                const int e = ((rho & 63) / B) * B - 1;      // chunk-local boundary row (-1: S0)
                if (fact) {
                    // Z K^T over Khat = 2^{gamma_C - gamma_i} k_i: M'_Z = (Gamma_e Z Khat^T) 2^{-gamma_C} [i <= e]
                    float zk[32];
                    tmem_ld32(tmem_addr(tb, q * 32, P_ZK + 32 * ch), zk);
                    tmem_wait_ld();
                    const float FC = s_F[CH - 1];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int i = 32 * ch + c;
                        zk[c] = (i <= e) ? zk[c] * FC : 0.f;
                    }
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        *reinterpret_cast<uint4 *>(sm + Q_NV + sw128_off(rho, 4 * ch + c4)) = pack8(zk + 8 * c4);
                } else {
                    mz_rows_exact(sm + Q_NV, sm + Q_NQ, tmem_addr(tb, q * 32, P_ZK + 32 * ch), rho, ch, e, s_gam, s_E);
                }
                fence_async_smem();
                tc_fence_before();
                if (bar_main_abort(&s_abort)) break;
            }

            // ---- S2: [P T;T] R -> R0, Gamma_e Z S0 -> N ----
            if (tid == 0) {
                wait_bar(&bar_hy, gc & 1, -1, 72);
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tb + P_R0, dK_y + ((kk * 32) >> 4), dM_v + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 0, 1), kk > 0);
                if (noisy)
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_bf16(tb + P_N, dK_nq + (off >> 4), dM_s0 + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 0, 1), 1u);
                    }
                commit(&bar_s2, 9);
            }
            __syncwarp();
            wait_bar(&bar_s2, gc & 1, tid == 0 ? 9 : -1, 73);
            __syncwarp();
            tc_fence_after();
            if (tid == 0 && noisy && nd.unit >= 0 && nd.m >= 0 && !dead)    // q~ (Z) is consumed
                load(2, nd.unit == cur_unit ? U : make_unit(P, nd.unit), nd.m);
            __syncwarp();
            // ---- E2: O = Gamma Q S0 + P U -> out; U -> V ----
            if (rho < 64) {
                const int t = rho;
                const int tok = cstart + t;
                const bool ok = tok >= U.s && tok < U.s + U.len;
                const float Gt = s_E[t];
                __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(P.out) + ((int64_t)tok * H + U.h) * D + 64 * ch;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float qs[32], pu[32];
                    tmem_ld32(tmem_addr(tb, q * 32, P_R1 + 64 * ch + 32 * hf), qs);
                    tmem_ld32(tmem_addr(tb, q * 32, P_R0 + 64 * ch + 32 * hf), pu);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) qs[x] = (Gt * qs[x] + pu[x]) * scale;
                    if (ok) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            *reinterpret_cast<uint4 *>(orow + 32 * hf + 8 * c4) = pack8(qs + 8 * c4);
                    }
                }
            } else {
                const int t = rho - 64;
                uint8_t *vrow = sm + Q_V + ch * 8192;
                float uub[2][32];
                tmem_ld32(tmem_addr(tb, q * 32, P_R0 + 64 * ch), uub[0]);
                tmem_ld32(tmem_addr(tb, q * 32, P_R0 + 64 * ch + 32), uub[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        *reinterpret_cast<uint4 *>(vrow + sw128_off(t, 4 * hf + c4)) = pack8(uub[hf] + 8 * c4);
                }
            }
            fence_async_smem();
            tc_fence_before();
            if (bar_main_abort(&s_abort)) break;

            // ---- S3: Khat^T U -> R1 (dS), M'_Z U -> N ----
            if (tid == 0) {
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tb + P_R1, dM_kh + ((kk * 2048) >> 4), dM_v + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 1, 1), kk > 0);
                if (noisy)
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tb + P_N, dK_mz + ((kk * 32) >> 4), dM_v + ((kk * 2048) >> 4), make_idesc_bf16(128, 128, 0, 1), 1u);
                commit(&bar_s3, 10);
            }
            __syncwarp();
            wait_bar(&bar_s3, gc & 1, tid == 0 ? 10 : -1, 74);
            __syncwarp();
            tc_fence_after();
            if (tid == 0 && nd.unit >= 0 && !dead) {       // U, Khat and M'_Z are consumed
                const Unit Un = nd.unit == cur_unit ? U : make_unit(P, nd.unit);
                load(1, Un, nd.m);
                if (noisy && nd.m >= 0 && V > 0) load(4, Un, nd.m);
            }
            __syncwarp();
            // ---- E3: S <- Gamma_C S + dS, S0 for the next chunk, noisy outputs ----
            {
                uint8_t *srow = sm + Q_S0 + ch * 16384;
                float ds0[32], ds1[32];
                tmem_ld32(tmem_addr(tb, q * 32, P_R1 + 64 * ch), ds0);
                tmem_ld32(tmem_addr(tb, q * 32, P_R1 + 64 * ch + 32), ds1);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    S[x] = fmaf(GC, S[x], ds0[x]);
                    S[32 + x] = fmaf(GC, S[32 + x], ds1[x]);
                }
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8)
                    *reinterpret_cast<uint4 *>(srow + sw128_off(rho, c8)) = pack8(S + 8 * c8);
                if (last) {
                    float *fs = P.final_state + ((int64_t)U.n * H + U.h) * D * D + (int64_t)rho * D + 64 * ch;
#pragma unroll
                    for (int c = 0; c < 64; c += 4)
                        *reinterpret_cast<float4 *>(fs + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
                }
            }
            if (noisy) {
                const int vw = rho >> 6, jj = rho & 63;
                const int rr = CH * m + jj;
                const bool ok = vw < V && rr < U.R;
                __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(P.out_noisy) +
                                      (((int64_t)vw * TR + U.roff + rr) * H + U.h) * D + 64 * ch;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float on[32];
                    tmem_ld32(tmem_addr(tb, q * 32, P_N + 64 * ch + 32 * hf), on);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) on[x] *= scale;
                    if (ok) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            *reinterpret_cast<uint4 *>(orow + 32 * hf + 8 * c4) = pack8(on + 8 * c4);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            ++gc;
            if (noisy) ++gnc;
            if (bar_main_abort(&s_abort)) break;
        }
#undef dK_qk
#undef dK_nq
#undef dK_nk
#undef dK_kh
#undef dK_y
#undef dK_mz
#undef dM_s0
#undef dM_v
#undef dM_kh
#undef dM_nv
        // drain (a no-op unless a wait gave up): thread 0's TMA loads and MMA commits, in order
        if (tid == 0) {
            uint64_t *bars[11] = {&bar_qk, &bar_v, &bar_nq, &bar_nk, &bar_nv, &bar_pk1n,
                                  &bar_b1, &bar_b2, &bar_pk2n, &bar_s2, &bar_s3};
            for (int i = 0; i < 11; ++i)
                for (uint32_t p = s_ok[i]; p < s_iss[i]; ++p) mbar_wait(bars[i], p & 1, kDrainWaitIters);
        }
    } else {
        // ========================================================================= helper warps
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHelpRegs));
        const int ht = tid - kMainThreads, hw = ht >> 5, hrho = ht;   // TMEM lane = ht (warps 8-11: quadrants 0-3)
        const uint64_t dK_qk = make_sdesc(a_qk, 16, 1024);
        const uint64_t dK_y = make_sdesc(a_y, 16, 1024);             // [P;T], K-major A
        const uint64_t dM_t = make_sdesc(a_y + 8192, 8192, 1024);    // T rows as MN-major B
        float *scratch = reinterpret_cast<float *>(sm + Q_Y);
        float *wstage = reinterpret_cast<float *>(sm + Q_W);
        const bool issuer = ht == 0;

        int u = blockIdx.x;           // current unit (first: blockIdx.x; then from the counter)
        int m_next = 0;               // next chunk index of unit u (set when u is opened)
        bool open = false;            // unit u opened (its first chunk not yet published)
        uint32_t hc = 0;              // chunks published
        Unit U{};
        for (;;) {
            // ---- next chunk: the next one of the current unit, else the next non-empty unit ----
            int cu = -1, cm = 0;
            for (;;) {
                if (!open) {
                    if (u >= P.num_units) break;
                    U = make_unit(P, u);
                    if (U.nchunks == 0) {       // empty document: its final state is zero
                        float *fs = P.final_state + ((int64_t)U.n * H + U.h) * D * D;
                        for (int i = ht * 4; i < D * D; i += kHelpThreads * 4)
                            *reinterpret_cast<float4 *>(fs + i) = make_float4(0.f, 0.f, 0.f, 0.f);
                    } else {
                        open = true;
                        m_next = U.m_first;
                    }
                    if (!open) {
                        if (issuer) s_next = (int)gridDim.x + atomicAdd(&P.ws->next_unit, 1);
                        bar_help();
                        u = s_next;
                        bar_help();
                        continue;
                    }
                }
                cu = u;
                cm = m_next;
                if (++m_next == U.m_first + U.nchunks) {    // last chunk of the unit: fetch the next unit
                    open = false;
                    if (issuer) s_next = (int)gridDim.x + atomicAdd(&P.ws->next_unit, 1);
                    bar_help();
                    u = s_next;
                    bar_help();
                }
                break;
            }
            // ---- scalars of chunk (cu, cm): cp.async, then the scans ----
            float *sc = s_sc[hc & 1];
            if (cu >= 0) {
                const Unit Uc = make_unit(P, cu);
                // warps 0-1: clean row ht and noisy view-0 row ht; warps 2-3: noisy view-1 row ht-64
                const int row = ht & 63;
                const float *gp = P.g, *bp = P.beta;
                uint32_t nb = 0;
                if (ht < CH) {
                    const int tok = Uc.s + Uc.prompt + CH * cm + row;
                    if (tok >= Uc.s && tok < Uc.s + Uc.len) {
                        gp = P.g + (int64_t)tok * H + Uc.h;
                        bp = P.beta + (int64_t)tok * H + Uc.h;
                        nb = 4;
                    }
                    cp_async4(&s_raw[0][ht], gp, nb);
                    cp_async4(&s_raw[1][ht], bp, nb);
                }
                for (int vw = ht < CH ? 0 : 1; vw < 2; vw += 2) {
                    const int rr = CH * cm + row;
                    const float *gq = P.g, *bq = P.beta;
                    uint32_t nbn = 0;
                    if (cm >= 0 && vw < V && rr < Uc.R) {
                        const int64_t r = (int64_t)vw * TR + Uc.roff + rr;
                        gq = P.gn + r * H + Uc.h;
                        bq = P.betan + r * H + Uc.h;
                        nbn = 4;
                    }
                    cp_async4(&s_raw[0][CH + 64 * vw + row], gq, nbn);
                    cp_async4(&s_raw[1][CH + 64 * vw + row], bq, nbn);
                }
                cp_async_commit();
                cp_async_wait_all();
                __syncwarp();
                // clean: inclusive scan over the chunk (warps 0, 1)
                if (ht < CH) {
                    float gv = s_raw[0][ht] * kLog2e;
                    sc[SC_BETA + ht] = s_raw[1][ht];
#pragma unroll
                    for (int d = 1; d < 32; d <<= 1) {
                        const float o2 = __shfl_up_sync(0xffffffffu, gv, d);
                        if (lane >= d) gv += o2;
                    }
                    s_g[ht] = gv;
                }
                // noisy: inclusive scan inside each block
                for (int vw = ht < CH ? 0 : 1; vw < 2; vw += 2) {
                    const int idx = 64 * vw + row;
                    float gv = s_raw[0][CH + idx] * kLog2e;
                    sc[SC_NBETA + idx] = s_raw[1][CH + idx];
                    const int jl = row % B;
#pragma unroll
                    for (int d = 1; d < 32; d <<= 1) {
                        const float o2 = __shfl_up_sync(0xffffffffu, gv, d);
                        if (d < B && jl >= d) gv += o2;
                    }
                    sc[SC_NGAM + idx] = gv;
                    if constexpr (B >= 16) {
                        sc[SC_NE + idx] = exp2f(gv);
                        sc[SC_NF + idx] = exp2f(-gv);
                        const bool okn = __all_sync(0xffffffffu, fabsf(gv) < 100.f);
                        if (lane == 0) s_okn[hc & 1][idx >> 5] = okn;
                    }
                }
                bar_help();
                if (ht < CH) {
                    const float gm = s_g[ht] + (ht >= 32 ? s_g[31] : 0.f);
                    sc[SC_GAM + ht] = gm;
                    sc[SC_E + ht] = exp2f(gm);
                    sc[SC_F + ht] = exp2f(-gm);
                    // e^{gamma_t - gamma_i} = E_t F_i only while every |gamma| of the chunk is far from
                    // the fp32 exponent range; the two scan warps vote
                    const bool okf = __all_sync(0xffffffffu, fabsf(gm) < 100.f);
                    if (lane == 0) s_fact[ht >> 5] = okf;
                }
                bar_help();
                if (issuer) s_desc[hc & 1] = ChunkDesc{cu, cm, s_fact[0] && s_fact[1]};
            } else if (issuer) {
                s_desc[hc & 1] = ChunkDesc{-1, 0, 0};
            }
            const bool stop = bar_help_abort(&s_abort);
            if (issuer) mbar_arrive(&bar_hs[hc & 1]);
            if (cu < 0 || stop) break;

            // ---- [Q;K] K^T -> H ----
            const ChunkDesc cd = s_desc[hc & 1];
            const bool fact = cd.fact != 0;
            const float *s_gam = sc + SC_GAM, *s_beta = sc + SC_BETA, *s_E = sc + SC_E, *s_F = sc + SC_F;
            wait_bar(&bar_qk, hc & 1, -1, 80);
            if (issuer) {
                tc_fence_after();
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tb + P_H, dK_qk + (off >> 4), dK_qk + ((8192 + off) >> 4), make_idesc_bf16(128, 64, 0, 0), kk > 0);
                }
                mma_commit(&bar_pk1c);
                ++s_iss[11];
            }
            __syncwarp();
            wait_bar(&bar_pk1c, hc & 1, issuer ? 11 : -1, 81);
            __syncwarp();
            tc_fence_after();
            // ---- A rows (lanes 64-127) into the fp32 scratch; the P rows stay in tensor memory ----
            if (hrho >= CH) {
                if (hc > 0) wait_bar(&bar_s2, (hc - 1) & 1, -1, 82);   // Y is free once S2 of the previous chunk is done
                if (fact) {
                    const int t = hrho - CH;
                    const float bEt = s_beta[t] * s_E[t];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        float tk[32];
                        tmem_ld32(tmem_addr(tb, hw * 32, P_H + 32 * h2), tk);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int i = 32 * h2 + c;
                            tk[c] = (i < t) ? (bEt * s_F[i]) * tk[c] : 0.f;
                        }
#pragma unroll
                        for (int g4 = 0; g4 < 8; ++g4)
                            *srow4(scratch, t, 32 * h2 + 4 * g4) =
                                make_float4(tk[4 * g4], tk[4 * g4 + 1], tk[4 * g4 + 2], tk[4 * g4 + 3]);
                    }
                } else {
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2)
                        pa_rows_exact(tmem_addr(tb, hw * 32, P_H + 32 * h2), hrho, h2, s_gam, s_beta, scratch);
                }
            }
            if (bar_help_abort(&s_abort)) break;
            // ---- T = (I + A)^{-1} ----
            solve_T_help(scratch, wstage, ht, hw, lane);
            // ---- [P ; T] as bf16 K-major A (128 rows x 64): row hrho (P from tensor memory, T from the scratch) ----
            uint4 ppk[8];
            if (hrho < CH) {
                const int t = hrho;
                if (fact) {
                    const float Et = s_E[t];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        float tk[32];
                        tmem_ld32(tmem_addr(tb, hw * 32, P_H + 32 * h2), tk);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int i = 32 * h2 + c;
                            tk[c] = (i <= t) ? tk[c] * (Et * s_F[i]) : 0.f;
                        }
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) ppk[4 * h2 + c4] = pack8(tk + 8 * c4);
                    }
                } else {
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const Rows4 r = pa_rows_exact(tmem_addr(tb, hw * 32, P_H + 32 * h2), hrho, h2, s_gam, s_beta, scratch);
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) ppk[4 * h2 + c4] = r.v[c4];
                    }
                }
            } else {
                const int t = hrho - CH;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const bool lowleft = t >= 32 && h2 == 0;      // the 32-merge's block
#pragma unroll
                    for (int g4 = 0; g4 < 4; ++g4) {
                        const float4 a = lowleft ? *wrow4(wstage, t - 32, 8 * g4) : *srow4(scratch, t, 32 * h2 + 8 * g4);
                        const float4 b = lowleft ? *wrow4(wstage, t - 32, 8 * g4 + 4) : *srow4(scratch, t, 32 * h2 + 8 * g4 + 4);
                        const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                        ppk[4 * h2 + g4] = pack8(f);
                    }
                }
            }
            bar_help();
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) *reinterpret_cast<uint4 *>(sm + Q_Y + sw128_off(hrho, c8)) = ppk[c8];
            fence_async_smem();
            tc_fence_before();
            bar_help();
            // ---- [P;T] T -> H (rows 0-63: P T) ----
            if (issuer) {
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tb + P_H, dK_y + ((kk * 32) >> 4), dM_t + ((kk * 2048) >> 4), make_idesc_bf16(128, 64, 0, 1), kk > 0);
                mma_commit(&bar_pk2c);
                ++s_iss[12];
            }
            __syncwarp();
            wait_bar(&bar_pk2c, hc & 1, issuer ? 12 : -1, 83);
            __syncwarp();
            tc_fence_after();
            if (hrho < CH) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    float pt[32];
                    tmem_ld32(tmem_addr(tb, hw * 32, P_H + 32 * h2), pt);
                    tmem_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        *reinterpret_cast<uint4 *>(sm + Q_Y + sw128_off(hrho, 4 * h2 + c4)) = pack8(pt + 8 * c4);
                }
            }
            fence_async_smem();
            tc_fence_before();
            bar_help();
            if (issuer) mbar_arrive(&bar_hy);
            // ---- Khat = diag(2^{gamma_C - gamma_t}) K, once S3 of the previous chunk has read Khat ----
            if (hc > 0) wait_bar(&bar_s3, (hc - 1) & 1, -1, 84);
            {
                const float gC = s_gam[CH - 1];
                for (int it = ht; it < CH * 16; it += kHelpThreads) {
                    const int t = it >> 4, c16 = it & 15, hf = c16 >> 3, c8 = c16 & 7;
                    float f[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + Q_QK + hf * 16384 + sw128_off(64 + t, c8)), f);
                    const float scl = fact ? s_E[CH - 1] * s_F[t] : exp2f(fminf(gC - s_gam[t], 0.f));
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] *= scl;
                    *reinterpret_cast<uint4 *>(sm + Q_KH + hf * 8192 + sw128_off(t, c8)) = pack8(f);
                }
            }
            fence_async_smem();
            const bool stop2 = bar_help_abort(&s_abort);
            if (issuer) mbar_arrive(&bar_hk);
            ++hc;
            if (stop2) break;
        }
        if (issuer) {
            uint64_t *bars[2] = {&bar_pk1c, &bar_pk2c};
            for (int i = 0; i < 2; ++i)
                for (uint32_t p = s_ok[11 + i]; p < s_iss[11 + i]; ++p) mbar_wait(bars[i], p & 1, kDrainWaitIters);
        }
        cp_async_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 512);
}

}  // namespace
}  // namespace gdn

namespace gdn {

// Launch of the pipelined kernel (no ShortConv prologue, at most two views; the caller splits more).
// Returns cudaErrorNotSupported, launching nothing, if the kernel was not compiled with the
// per-thread register count its register split assumes.
cudaError_t launch_pipe(const Params &p, cudaStream_t stream) {
    Maps maps;
    const bool noisy = p.V > 0 && p.TR > 0;
    if (!encode_map(&maps.q, p.q, p.H, p.T) || !encode_map(&maps.k, p.k, p.H, p.T) ||
        !encode_map(&maps.v, p.v, p.H, p.T))
        return cudaErrorInvalidValue;
    if (noisy) {
        if (!encode_map(&maps.qn, p.qn, p.H, (int64_t)p.V * p.TR) ||
            !encode_map(&maps.kn, p.kn, p.H, (int64_t)p.V * p.TR) ||
            !encode_map(&maps.vn, p.vn, p.H, (int64_t)p.V * p.TR))
            return cudaErrorInvalidValue;
    } else {
        maps.qn = maps.q;
        maps.kn = maps.k;
        maps.vn = maps.v;
    }
    static int num_sms = 0;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
        cudaError_t e = cudaSuccess;
        for (auto fn : {gdn_pipe_kernel<1>, gdn_pipe_kernel<2>, gdn_pipe_kernel<4>, gdn_pipe_kernel<8>,
                        gdn_pipe_kernel<16>, gdn_pipe_kernel<32>, gdn_pipe_kernel<4, true>}) {
            cudaError_t r = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, Q_SMEM_BYTES);
            if (r != cudaSuccess) e = r;
            cudaFuncAttributes fa;
            r = cudaFuncGetAttributes(&fa, fn);
            if (r != cudaSuccess) e = r;
            else if (fa.numRegs != kLaunchRegs) e = cudaErrorNotSupported;   // the register split would not fit
        }
        attr_err = e;
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int sms = num_sms > 0 ? num_sms : 148;
    const int grid = std::min(p.num_units, sms);
    if (p.wait_test) {           // the test entry point: B = 4 only
        if (p.B != 4) return cudaErrorNotSupported;
        gdn_pipe_kernel<4, true><<<grid, kPipeThreads, Q_SMEM_BYTES, stream>>>(p, maps);
        return cudaGetLastError();
    }
    switch (p.B) {
        case 1: gdn_pipe_kernel<1><<<grid, kPipeThreads, Q_SMEM_BYTES, stream>>>(p, maps); break;
        case 2: gdn_pipe_kernel<2><<<grid, kPipeThreads, Q_SMEM_BYTES, stream>>>(p, maps); break;
        case 4: gdn_pipe_kernel<4><<<grid, kPipeThreads, Q_SMEM_BYTES, stream>>>(p, maps); break;
        case 8: gdn_pipe_kernel<8><<<grid, kPipeThreads, Q_SMEM_BYTES, stream>>>(p, maps); break;
        case 16: gdn_pipe_kernel<16><<<grid, kPipeThreads, Q_SMEM_BYTES, stream>>>(p, maps); break;
        case 32: gdn_pipe_kernel<32><<<grid, kPipeThreads, Q_SMEM_BYTES, stream>>>(p, maps); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace gdn
