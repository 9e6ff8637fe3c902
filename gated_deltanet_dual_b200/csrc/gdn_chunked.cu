// gdn_chunked.cu -- dual-stream Gated DeltaNet forward, chunked WY/UT form on tcgen05 tensor
// cores (sm_100a).  bf16 I/O, fp32 state and accumulation, d_k = d_v = 128, chunk C = 64.
//
// Method ("FLARE: Diffusion for Hybrid Language Model", papernotes.org notes, Method > Key
// design 2 and 3): clean causal gated delta rule
//     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t / sqrt(d),
// and a block-bidirectional noisy stream: block b of every view restarts from S_{e(b-1)}, runs
// its B noisy tokens and every position reads the block-end state.  No per-block state is ever
// formed: each noisy row is carried as one extra row against the chunk's start state.
//
// Chunked form (derived from the rule; gamma = inclusive cumsum of g inside the chunk):
//   A_ti = beta_t e^{gamma_t-gamma_i} k_t.k_i (i<t),  T = (I + A)^{-1},
//   P_ti = e^{gamma_t-gamma_i} q_t.k_i (i<=t),       R = beta V - beta Gamma K S0,
//   [P U ; U] = [P T ; T] R,  O = Gamma Q S0 + P U,  S_C = Gamma_C S0 + Khat^T U,
//   Khat_t = e^{gamma_C-gamma_t} k_t.
// Noisy row j of a block starting at chunk row bs (boundary e = bs-1): with y = Ptil_j Ttil
// (Ttil the block's own WY inverse, Ptil_jl = e^{gammatil_B-gammatil_l} q~_j.k~_l),
//   Z_j  = Gammatil_B q~_j - sum_l y_l beta~_l Gammatil_l k~_l,   WV_j = sum_l y_l beta~_l v~_l,
//   o~_j = Gamma_e Z_j S0 + (Z_j K^T o M_j) U + WV_j,   M_ji = e^{gamma_e-gamma_i} [i <= e].
//
// Persistent CTAs, one per SM, take (document, head) work items longest first by greedy list
// scheduling (a counter in the workspace); with fewer units than half the SMs each unit is split
// over two CTAs (the second rebuilds its split-point state with the clean-only chain).  256
// threads = 8 warps, all of them math warps; thread 0 also issues the TMA loads and the MMAs.
// Each chunk runs five tensor-core phases, each followed by a math phase:
//   PK1  [Q;K]K^T, [q~0;q~1][k~0;k~1]^T, [k~0;k~1][k~0;k~1]^T     (S-independent)
//   PK2  [P;T] T -> P T,  [Z0;Z1] K^T                              (S-independent)
//   S1   [Q;K] S0,  [Gamma_e Z] S0 (+= WV)                         (needs S0)
//   S2   [P T; T] R                                                (needs R)
//   S3   Khat^T U,  M'_Z U (+=)                                    (needs U)
// Inputs of the next chunk are prefetched by TMA while the current chunk's S-dependent phases
// run.  Outputs of chunks that lie inside their document leave by TMA stores from tiles that are
// free at that point (O in the [P;T] tile, the noisy rows in the K-hat and [P;T] tiles), not as
// row-per-lane global stores; chunks at a document edge store row by row, so that no store
// reaches into a neighbouring document.  All waits are bounded; on timeout the kernel records GDN_ERR_TIMEOUT, waits for the
// copies and MMAs it has issued, and exits.
#include <algorithm>
#include <cudaTypedefs.h>
#include <mutex>
#include <type_traits>

#include "gdn_internal.cuh"
#include "sm100.cuh"
#include "gdn_chunk_common.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kMathWarps = 8;
constexpr int kMathThreads = kMathWarps * 32;
constexpr int kThreads = kMathThreads;   // thread 0 also issues TMA and MMA

// Dynamic shared memory layout (offsets from a 1024-byte aligned base).
constexpr int OFF_S0 = 0;          // 32 KB  S0 bf16, MN-major B: 2 v-halves x [128 k-rows x 128 B]
constexpr int OFF_QK = 32768;      // 32 KB  [Q;K] K-major: 2 d-halves x [Q 64 rows | K 64 rows]
constexpr int OFF_V = 65536;       // 16 KB  V -> R -> U, MN-major: 2 v-halves x [64 rows x 128 B]
constexpr int OFF_KH = 81920;      // 16 KB  Khat, MN-major A: 2 k-halves x [64 rows x 128 B]
constexpr int OFF_Y = 98304;       // 16 KB  fp32 solve scratch, then [P;T] -> [P T;T] K-major
constexpr int OFF_NQ = 114688;     // 32 KB  [q~0;q~1] -> Z -> Gamma_e Z, K-major
constexpr int OFF_NK = 147456;     // 32 KB  [k~0;k~1] K-major; d-half 0 later holds M'_Z
constexpr int OFF_NV = 180224;     // 32 KB  [v~0;v~1] per v-half (row-major, swizzled)
constexpr int OFF_W = 212992;      //  4 KB  the triangular solve's 32-merge result (32x32 fp32)
constexpr int SMEM_USED = 217088;
constexpr int SMEM_BYTES = SMEM_USED + 1024;   // alignment slack

// TMEM columns (512 allocated)
constexpr uint32_t TM_R0 = 0;      // q~k~^T | [Q;K]S0 | dS
constexpr uint32_t TM_R1 = 128;    // k~k~^T | [P U; U]
constexpr uint32_t TM_N = 256;     // noisy accumulator (WV + Gamma_e Z S0 + M'_Z U)
constexpr uint32_t TM_TK = 384;    // [Q;K]K^T | P T
constexpr uint32_t TM_ZK = 448;    // Z K^T
// Route I export j (the block starting at row j B): free columns once S2's products are read
__device__ __forceinline__ uint32_t export_col(int j) { return j == 1 ? TM_N : (j == 2 ? TM_R1 : TM_TK); }

__device__ __forceinline__ void bar_all() { asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory"); }
__device__ __forceinline__ void bar_math() { bar_all(); }
// Warps 1..7 only: work overlapped with an MMA batch that thread 0 (warp 0) is issuing.
__device__ __forceinline__ void bar_side() { asm volatile("bar.sync 3, %0;" ::"n"(kThreads - 32) : "memory"); }
// Named barrier 4: warps 1..7 arrive (no wait), warp 0 waits for them.
__device__ __forceinline__ void bar_arrive_khat() { asm volatile("bar.arrive 4, %0;" ::"n"(kThreads) : "memory"); }
__device__ __forceinline__ void bar_sync_khat() { asm volatile("bar.sync 4, %0;" ::"n"(kThreads) : "memory"); }

// Noisy rows, step 1: block coefficients of this thread's row from [q~;k~]k~^T (TMEM), then the
// rows of W~ and -Y~ as tensor-memory A operands (columns [0,64) and [64,128) from TM_TK).
template <int B>
__device__ __forceinline__ float noisy_phase1(uint32_t tb, int q, int ch, int lane, int rho,
                                              const float *s_ngam, const float *s_nbeta, const float *s_nE,
                                              const float *s_nF, bool nfact, float *s_at) {
    float wq[32], wk[32];
    tmem_ld32(tmem_addr(tb, q * 32, TM_R0 + 32 * q), wq);
    tmem_ld32(tmem_addr(tb, q * 32, TM_R1 + 32 * q), wk);
    tmem_wait_ld();
    const int v = rho >> 6, j = rho & 63;
    float ycoef[B], wcoef[B], gend;
    noisy_coeffs<B>(wq, wk, lane, j, s_ngam + 64 * v, s_nbeta + 64 * v, s_nE + 64 * v, s_nF + 64 * v, nfact,
                    s_at, ycoef, wcoef, gend);
    bar_math();   // every warp has finished reading TM_TK before it is overwritten
    const int bs = (j / B) * B;
    store_block_row<B>(tmem_addr(tb, q * 32, TM_TK + 32 * ch), ch, v, bs, wcoef, 1.f);
    store_block_row<B>(tmem_addr(tb, q * 32, TM_TK + 64 + 32 * ch), ch, v, bs, ycoef, -1.f);
    return gend;
}

// Noisy rows, step 2: Z_j = Gammatil_B q~_j + (-Y~ K~)_j over the q~ row (d columns [64ch, 64ch+64)).
// zs: a row scale applied on the way out (Gamma_e of the row's block boundary when the chunk's
// decays factorise, so the later Gamma_e Z pass is not needed; else 1).
__device__ __forceinline__ void z_epilogue(uint8_t *sm, uint32_t tb, int q, int ch, int rho, float gend, float zs) {
    const float Gend = exp2f(gend) * zs;
    uint8_t *nq = sm + OFF_NQ + ch * 16384;
    float ykb[2][32];
    tmem_ld32(tmem_addr(tb, q * 32, TM_R1 + 64 * ch), ykb[0]);
    tmem_ld32(tmem_addr(tb, q * 32, TM_R1 + 64 * ch + 32), ykb[1]);
    tmem_wait_ld();
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        float (&yk)[32] = ykb[hf];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t o = sw128_off(rho, 4 * hf + c4);
            float z[8];
            unpack8(*reinterpret_cast<const uint4 *>(nq + o), z);
#pragma unroll
            for (int e = 0; e < 8; ++e) z[e] = fmaf(Gend, z[e], zs * yk[8 * c4 + e]);
            *reinterpret_cast<uint4 *>(nq + o) = pack8(z);
        }
    }
}

// T = (I + A)^{-1} for the strictly lower 64x64 A in the fp32 scratch, while warp 0 issues an MMA
// batch: warps 1-2 invert the eight 8x8 diagonal blocks (one thread per column, right-looking
// forward substitution), warps 1-4 run the four 8-merges (one warp each, in place) and the two
// 16-merges (two warps each, in place after a barrier); then all warps run the 32-merge, whose
// lower-left block goes to the 32 x 32 staging block `wb` (rows 32..63, columns 0..31 of T) so that
// no warp overwrites A while another still reads it.
__device__ void solve_T(float *sa, float *wb, int tid, int warp) {
    const int lane = tid & 31;
    if (warp > 0) {
        const int t = tid - 32;
        if (t < 64) {
            const int o = (t >> 3) * 8, c = t & 7;
            // column c of the block's inverse, right-looking: x_l is final once every earlier
            // x has been taken out of it
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
        bar_side();
        auto in_place = [sa](int o, int S) {
            return [sa, o, S](int r, int c, float v) { sa[sidx(o + S + r, o + c)] = v; };
        };
        if (warp <= 4) {           // four 8-merges, one warp each (a warp owns its whole merge)
            const int o = 16 * (warp - 1);
            warp_merge<8, 8>(sa, o, 0, lane, in_place(o, 8), [] {});
        }
        bar_side();
        if (warp <= 4) {           // two 16-merges, two warps each (8 columns per warp)
            const int o = 32 * ((warp - 1) >> 1), cb = 8 * ((warp - 1) & 1);
            warp_merge<16, 8>(sa, o, cb, lane, in_place(o, 16), [] { bar_side(); });
        } else {
            bar_side();            // the 16-merges' reads precede their writes
        }
    }
    bar_math();
    // warp 0 arrives last (it issued the MMA batch): it takes the columns with the least work
    warp_merge<32, 4>(sa, 0, 4 * (7 - warp), lane, [&](int r, int c, float v) { wb[widx(r, c)] = v; }, [] {});
    bar_math();
}

// ----------------------------------------------------------------------------- ShortConv
// Width-4 depthwise causal conv on q, k, v (Key design 3 of the FLARE notes), applied in place to
// the chunk's tiles before anything reads them.  Tap 3 is the current token.  Clean taps before
// the document start read 0; a noisy tap that reaches before its block start reads the clean raw
// input (rows of this chunk, or the three raw rows carried over from the previous chunk).
//
// Work item: a few rows (a segment) of one 8-channel column of one tensor.  Lane bits 0-3 pick
// the column, so the 8 lanes of a shared-memory phase touch 8 distinct 16-byte chunks of one row.
// Every item reads all its rows into registers before any item of the same round writes, so the
// in-place update needs one barrier per round at most.  Arithmetic is fp32, two channels per
// instruction (packed FFMA2), rounded once to bf16.
constexpr int OFF_CW = OFF_KH;   // conv weights (6 KB) until K-hat is built

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ float2 bf2_lo_hi(uint32_t w) {   // bf16 pair -> (even channel, odd channel)
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2(float2 f) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t &word_of(uint4 &u, int i) {
    return i == 0 ? u.x : (i == 1 ? u.y : (i == 2 ? u.z : u.w));
}
// Shared address of row r of 8-channel column c8 in a 64-row, 128-byte-swizzled half tile.
__device__ __forceinline__ uint32_t conv_row(uint32_t half, int r, int c8) {
    return half + r * 128 + ((c8 ^ (r & 7)) << 4);
}
// Byte offset of the half tile (64 channels) holding column half hf of clean tensor X / noisy
// tensor X of view v.
__device__ __forceinline__ int clean_half(int X, int hf) {
    return X == 2 ? OFF_V + hf * 8192 : OFF_QK + hf * 16384 + X * 8192;
}
__device__ __forceinline__ int noisy_half(int X, int v, int hf) {
    return (X == 0 ? OFF_NQ : (X == 1 ? OFF_NK : OFF_NV)) + hf * 16384 + v * 8192;
}
// Noisy segment of LEN rows that starts on a block boundary (B <= LEN): is clean row d (relative
// to the segment start, -3 <= d < LEN - 1) a tap of one of its rows?
__host__ __device__ constexpr bool conv_clean_tap(int B, int LEN, int d) {
    for (int t = 0; t < LEN; ++t)
        for (int l = 1; l <= 3; ++l)
            if (t - l == d && d < t - t % B) return true;
    return false;
}

// One work item: the LEN rows r0.. of one 8-channel column of one tensor, convolved in place;
// a noisy item covers both views.  own[v][t] = raw row r0 + t of view v; ini = the raw rows
// before them: for a noisy segment that starts on a block boundary (B <= LEN) every clean row
// d (relative to r0, -3 <= d < LEN - 1) that a block start taps, shared by the views; otherwise
// rows r0-3..r0-1 per view (clean, or the noisy rows of the view when r0 is inside a block).
// All reads happen in load(); the caller puts a barrier between the loads and the stores.
template <int B, bool NOISY, int LEN>
struct ConvSeg {
    static constexpr int NV = NOISY ? 2 : 1;
    static constexpr bool TAPS = NOISY && B <= LEN;
    static constexpr int NI = TAPS ? LEN + 2 : 3;
    static constexpr int NIV = (NOISY && !TAPS) ? NV : 1;
    uint4 own[NV][LEN];
    uint4 ini[NIV][NI];

    // own0: half tile of the tensor (view 0; view 1 follows 8 KB later); cln: half tile of the
    // clean tensor; halo: carried raw clean rows [row][column] (rows cstart-3..cstart-1); zr:
    // chunk rows r < zr lie before the document start and read 0 when clean; bstart: r0 starts
    // a block (noisy items).
    __device__ __forceinline__ uint4 clean_row(uint32_t cln, const uint4 (*halo)[16], int cc, int r, int c8,
                                               int zr) {
        if (r < zr) return make_uint4(0u, 0u, 0u, 0u);
        if (r < 0) return halo[3 + r][cc];
        return lds128(conv_row(cln, r, c8));
    }
    __device__ __forceinline__ void load(uint32_t own0, uint32_t cln, const uint4 (*halo)[16], int cc, int r0,
                                         int c8, int zr, bool bstart) {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
#pragma unroll
            for (int t = 0; t < LEN; ++t) own[v][t] = lds128(conv_row(own0 + v * 8192, r0 + t, c8));
        }
        if (!NOISY && zr > r0) {
#pragma unroll
            for (int t = 0; t < LEN; ++t)
                if (r0 + t < zr) own[0][t] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (TAPS) {
#pragma unroll
            for (int k = 0; k < NI; ++k)
                ini[0][k] = conv_clean_tap(B, LEN, k - 3) ? clean_row(cln, halo, cc, r0 + k - 3, c8, zr)
                                                          : make_uint4(0u, 0u, 0u, 0u);
        } else if (!NOISY) {
#pragma unroll
            for (int k = 0; k < 3; ++k) ini[0][k] = clean_row(cln, halo, cc, r0 + k - 3, c8, zr);
        } else if (bstart) {
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                ini[0][k] = clean_row(cln, halo, cc, r0 + k - 3, c8, zr);
                ini[NIV - 1][k] = ini[0][k];
            }
        } else {
#pragma unroll
            for (int v = 0; v < NIV; ++v) {
#pragma unroll
                for (int k = 0; k < 3; ++k) ini[v][k] = lds128(conv_row(own0 + v * 8192, r0 + k - 3, c8));
            }
        }
    }

    // Convolve and write over the rows.  w: weights of this (tensor, column).
    __device__ __forceinline__ void store(uint32_t own0, uint32_t w, int r0, int c8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {                 // channel pair (2i, 2i+1)
            const float4 wa = lds128f(w + i * 512), wb = lds128f(w + i * 512 + 256);
            const float2 w0 = make_float2(wa.x, wa.y), w1 = make_float2(wa.z, wa.w);
            const float2 w2 = make_float2(wb.x, wb.y), w3 = make_float2(wb.z, wb.w);
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                uint4 (&in)[NI] = ini[TAPS ? 0 : (NIV > 1 ? v : 0)];
                float2 x1 = bf2_lo_hi(word_of(in[2], i)), x2 = bf2_lo_hi(word_of(in[1], i)),
                       x3 = bf2_lo_hi(word_of(in[0], i));
#pragma unroll
                for (int t = 0; t < LEN; ++t) {
                    if (TAPS && t > 0 && t % B == 0) {   // block start: clean taps
                        x1 = bf2_lo_hi(word_of(in[t + 2], i));
                        x2 = bf2_lo_hi(word_of(in[t + 1], i));
                        x3 = bf2_lo_hi(word_of(in[t], i));
                    }
                    const float2 x0 = bf2_lo_hi(word_of(own[v][t], i));
                    float2 acc = __fmul2_rn(w3, x0);
                    acc = __ffma2_rn(w2, x1, acc);
                    acc = __ffma2_rn(w1, x2, acc);
                    acc = __ffma2_rn(w0, x3, acc);
                    word_of(own[v][t], i) = f2_to_bf2(acc);   // the raw word is dead once unpacked
                    x3 = x2; x2 = x1; x1 = x0;
                }
            }
        }
#pragma unroll
        for (int v = 0; v < NV; ++v) {
#pragma unroll
            for (int t = 0; t < LEN; ++t) sts128(conv_row(own0 + v * 8192, r0 + t, c8), own[v][t]);
        }
    }
};

// Weights of (tensor X, column cc): fp32 [channel pair i][taps 0-1 | taps 2-3][cc][tap][pair], so
// the eight lanes of a shared-memory phase read eight consecutive 16-byte words and every word
// is an operand pair of a packed FFMA2.
__device__ __forceinline__ uint32_t conv_weights(uint32_t s, int X, int cc) {
    return s + OFF_CW + (X * 128 + cc) * 16;
}
// Noisy item (both views): tensor X, rows r0..r0+LEN-1.  bar: barrier between loads and stores
// (uniform over the CTA).  Out of line: both noisy rounds share one copy of the code.
template <int B, int LEN>
__device__ __noinline__ void conv_noisy_item(uint32_t s, uint4 (*halo)[3][16], int X, int cc, int r0, int zr,
                                             bool bar) {
    const int hf = cc >> 3, c8 = cc & 7;
    const uint32_t own = s + noisy_half(X, 0, hf);
    ConvSeg<B, true, LEN> sg;
    sg.load(own, s + clean_half(X, hf), halo[X], cc, r0, c8, zr, (r0 % B) == 0);
    if (bar) bar_math();
    sg.store(own, conv_weights(s, X, cc), r0, c8);
}
// Clean item: tensor X, rows r0..r0+LEN-1; the item ending at row 63 carries rows 61..63 (raw)
// to the next chunk.
template <int B, int LEN>
__device__ __forceinline__ void conv_clean_item(uint32_t s, uint4 (*halo)[3][16], int X, int cc, int r0, int zr) {
    const int hf = cc >> 3, c8 = cc & 7;
    const uint32_t own = s + clean_half(X, hf);
    ConvSeg<B, false, LEN> sg;
    sg.load(own, own, halo[X], cc, r0, c8, zr, true);
    bar_math();
    if (r0 + LEN == CH) {
#pragma unroll
        for (int l = 0; l < 3; ++l) halo[X][l][cc] = sg.own[0][LEN - 3 + l];
    }
    sg.store(own, conv_weights(s, X, cc), r0, c8);
}

// The whole prologue for one chunk (all threads; a barrier between the reads and the writes of
// each round that rewrites rows another item reads).  A noisy tile is convolved before the clean
// tile of the same tensor is overwritten (its block-start taps read the raw clean rows); a halo
// is read before the round that rewrites it.  Rounds of 256 items, 36 output rows per thread:
//   1  noisy q, k (8-row items, both views)
//   2  noisy v (8-row items, both views) | clean q, k (16-row items)
//   3  clean v (4-row items)
// A chunk without noisy rows runs clean q, k as 8-row items, then round 3.
// zr = document start - chunk start.
template <int B>
__device__ __noinline__ void conv_chunk(uint8_t *sm, uint4 (*halo)[3][16], bool noisy, int zr, int tid) {
    const uint32_t s = smem_u32(sm);
    const int cc = tid & 15;
    if (noisy) {
        conv_noisy_item<B, 8>(s, halo, tid >> 7, cc, 8 * ((tid >> 4) & 7), zr, B > 8);
        if (tid < 128) conv_noisy_item<B, 8>(s, halo, 2, cc, 8 * ((tid >> 4) & 7), zr, true);
        else conv_clean_item<B, 16>(s, halo, (tid >> 6) & 1, cc, 16 * ((tid >> 4) & 3), zr);
    } else {
        conv_clean_item<B, 8>(s, halo, tid >> 7, cc, 8 * ((tid >> 4) & 7), zr);
    }
    conv_clean_item<B, 4>(s, halo, 2, cc, 4 * (tid >> 4), zr);
    fence_async_smem();                      // the tiles are next read by the tensor cores
}

// Next work item of the CTA: thread 0 takes one from the workspace counter and broadcasts it (the
// first gridDim.x items are taken by blockIdx.x at start).  Kept out of line so that the main
// loop's register allocation does not depend on it.
__device__ __noinline__ int next_work_item(WorkspaceHeader *ws, int *s_next) {
    if (threadIdx.x == 0) *s_next = (int)gridDim.x + atomicAdd(&ws->next_unit, 1);
    __syncthreads();
    const int nx = *s_next;
    __syncthreads();                          // read by all before thread 0 writes it again
    return nx;
}

// TW: the test instantiation, whose waits poll with the caller's bound (gdn_dual_forward_test_wait_limit).
// CONV: the instantiation with the fused ShortConv prologue (the other one has no conv code at
// all, which keeps its loop body smaller for the instruction cache).
// EXPORT: Route I's first stage (no noisy views; B = 16 or 32): besides the clean outputs, the
// state before every response block, S_e = Gamma_e S0 + Khat_e^T U with Khat_e,i =
// e^{gamma_e - gamma_i} k_i (i <= e), is written to P.states as a 32 KB blob in the bf16 S0 tile
// layout (the kernels' MMA B operand): the chunk's own S0 for the block at its row 0, and one
// more MMA per later block start, into tensor-memory columns and shared tiles that carry the
// noisy rows when there are views.
template <int B, bool TW = false, bool CONV = false, bool EXPORT = false>
__global__ void __launch_bounds__(kThreads, 1)
gdn_chunked_kernel(const __grid_constant__ Params P, const __grid_constant__ Maps M) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_a, bar_b, bar_mma, bar_mma2;   // bar_mma2: the noisy half of PK1 only
    __shared__ uint64_t bar_drain;                         // error path: all MMAs of thread 0 done
    __shared__ uint64_t bar_ost;                           // thread 0: the O tile's store has read [P;T]
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    // Per-chunk scalars, double-buffered so the next chunk's are prepared while this chunk's
    // state phases run: [buffer][gamma | beta | E = 2^gamma | F = 2^-gamma | noisy gamma | noisy beta]
    constexpr int SC_GAM = 0, SC_BETA = CH, SC_E = 2 * CH, SC_F = 3 * CH, SC_NGAM = 4 * CH, SC_NBETA = 6 * CH;
    constexpr int SC_NE = 8 * CH, SC_NF = 10 * CH;   // noisy rows: 2^gamma~ and 2^-gamma~ (B >= 16)
    __shared__ float s_sc[2][(B >= 16 ? 12 : 8) * CH];
    __shared__ int s_okw[2][2];
    __shared__ int s_okn[2][4];               // every |gamma~| of a 32-row noisy group below 100
    __shared__ float s_g[CH];                 // scan scratch
    __shared__ float s_raw[2][3 * CH];        // [gate, beta][row]: cp.async staging (read before restaged)
    __shared__ uint4 s_halo[3][3][16];        // ShortConv: raw clean rows cstart-3..cstart-1 [q,k,v][row][chunk]

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, ch = (warp >> 2) & 1, rho = q * 32 + lane;   // TMEM row (lane) and column half
    const int H = P.H, V = P.V;
    const int64_t TR = P.TR;
    const float scale = P.scale;
    constexpr bool conv = CONV;   // the host launches CONV exactly when P.conv_width > 0

    if (tid == 0) {
        mbar_init(&bar_a, 1);
        mbar_init(&bar_b, 1);
        mbar_init(&bar_mma, 1);
        mbar_init(&bar_mma2, 1);
        mbar_init(&bar_drain, 1);
        mbar_init(&bar_ost, 1);
        fence_mbar_init();
        s_abort = 0;
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
    // Every mbarrier has at most one outstanding phase when it is waited on, so parities never alias.
    uint32_t ph_a = 0, ph_b = 0, ph_mma = 0, ph_mma2 = 0, ph_ost = 0;

    auto fail = [&](int where) {
        if (atomicExch(&s_abort, 1) == 0) {
            atomicExch(&P.ws->status, (int)GDN_ERR_TIMEOUT);
            atomicExch(&P.ws->timeout_where, where);
        }
    };
    // Error path.  A wait that gives up records GDN_ERR_TIMEOUT, and the CTA leaves its loop at the
    // next abort check (all threads at the same barrier).  Thread 0, the only thread that issues TMA
    // loads and MMAs, issues no further TMA load once one of its own waits has given up (`dead`), so
    // on each TMA barrier at most the last load it issued can still be in flight when the CTA leaves
    // (every earlier one was waited for: a prefetch is only issued after the previous load's wait).
    // Before the CTA frees its tensor memory, thread 0 waits for that last load (s_iss counts the
    // loads) and, with one more commit, for every MMA it issued, so no bulk copy or MMA is left
    // writing into shared or tensor memory that is no longer the CTA's.
    bool dead = false;
    __shared__ uint32_t s_iss[2];
    if (tid == 0) s_iss[0] = s_iss[1] = 0;
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph, int where) {
        if (!kwait<TW>(bar, ph & 1, kWaitIters, P.wait_iters)) {
            fail(where);
            dead = true;
        }
        ++ph;
    };
    // bar_all that also tells every thread, uniformly, whether the CTA is aborting
    auto abort_check = [&] { return bar_sync_or(1, kThreads, *reinterpret_cast<volatile int *>(&s_abort) != 0); };
    auto wait_mma = [&](int where) {
        wait_bar(&bar_mma, ph_mma, where);
        __syncwarp();            // reconverge before warp-collective tcgen05.ld/st
        tc_fence_after();
    };
    auto wait_mma2 = [&](int where) {
        wait_bar(&bar_mma2, ph_mma2, where);
        __syncwarp();
        tc_fence_after();
    };
    auto commit_mma = [&] { mma_commit(&bar_mma); };   // thread 0

    // Issue the TMA loads of chunk m of unit U (control lane 0).  group A: [Q;K] and, for a
    // response chunk, [q~;.] and v~;  group B: V and, for a response chunk, [k~;.].
    auto issue_a = [&](const Unit &U, int m, bool nz) {
        const int cstart = U.s + U.prompt + CH * m;
        ++s_iss[0];
        mbar_arrive_expect_tx(&bar_a, 32768u + (nz ? 65536u : 0u));
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(sm + OFF_QK + hf * 16384, &M.q, &bar_a, hf * 64, U.h, cstart);
            tma_load_3d(sm + OFF_QK + hf * 16384 + 8192, &M.k, &bar_a, hf * 64, U.h, cstart);
        }
        if (nz) {
            for (int vw = 0; vw < 2; ++vw) {
                const int row = vw * (int)TR + U.roff + CH * m;
                for (int hf = 0; hf < 2; ++hf) {
                    tma_load_3d(sm + OFF_NQ + hf * 16384 + vw * 8192, &M.qn, &bar_a, hf * 64, U.h, row);
                    tma_load_3d(sm + OFF_NV + hf * 16384 + vw * 8192, &M.vn, &bar_a, hf * 64, U.h, row);
                }
            }
        }
    };
    auto issue_b = [&](const Unit &U, int m, bool nz) {
        const int cstart = U.s + U.prompt + CH * m;
        ++s_iss[1];
        mbar_arrive_expect_tx(&bar_b, 16384u + (nz ? 32768u : 0u));
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(sm + OFF_V + hf * 8192, &M.v, &bar_b, hf * 64, U.h, cstart);
        if (nz) {
            for (int vw = 0; vw < 2; ++vw) {
                const int row = vw * (int)TR + U.roff + CH * m;
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_3d(sm + OFF_NK + hf * 16384 + vw * 8192, &M.kn, &bar_b, hf * 64, U.h, row);
            }
        }
    };

    const uint32_t a_s0 = smem_u32(sm + OFF_S0), a_qk = smem_u32(sm + OFF_QK), a_v = smem_u32(sm + OFF_V);
    const uint32_t a_kh = smem_u32(sm + OFF_KH), a_y = smem_u32(sm + OFF_Y), a_nq = smem_u32(sm + OFF_NQ);
    const uint32_t a_nk = smem_u32(sm + OFF_NK);
    // Base shared-memory descriptors; an operand offset of `off` bytes adds off >> 4.
    const uint64_t dK_qk = make_sdesc(a_qk, 16, 1024);           // [Q;K] K-major (A), K rows (B)
    const uint64_t dK_nq = make_sdesc(a_nq, 16, 1024);           // [q~;.] / Z, K-major
    const uint64_t dK_nk = make_sdesc(a_nk, 16, 1024);           // [k~;.] / M'_Z, K-major
    const uint64_t dK_y = make_sdesc(a_y, 16, 1024);             // [P;T] / [PT;T], K-major A
    const uint64_t dM_t = make_sdesc(a_y + 8192, 8192, 1024);    // T rows as MN-major B
    const uint64_t dM_s0 = make_sdesc(a_s0, 16384, 1024);        // S0, MN-major B
    const uint64_t dM_v = make_sdesc(a_v, 8192, 1024);           // R / U, MN-major B
    const uint64_t dM_kh = make_sdesc(a_kh, 8192, 1024);         // Khat, MN-major A
    const uint64_t dM_nv = make_sdesc(smem_u32(sm + OFF_NV), 16384, 1024);  // [v~0;v~1], MN-major B
    const uint64_t dM_nk = make_sdesc(a_nk, 16384, 1024);        // [k~0;k~1], MN-major B
    float *scratch = reinterpret_cast<float *>(sm + OFF_Y);
    float *wstage = reinterpret_cast<float *>(sm + OFF_W);

    constexpr float kLog2e = 1.4426950408889634f;
    // Stage (cp.async) the gate and beta of this thread's row in chunk mq of unit Uq into buffer
    // `buf`: threads 0-63 the clean rows, threads 64-191 the noisy rows of both views; rows
    // outside the document read as 0.
    // Rows are handled by warps 1..6 (sr = tid - 32): sr 0-63 the clean rows, sr 64-191 the noisy
    // rows of both views.
    const int sr = tid - 32;
    auto stage_scalars = [&](const Unit &Uq, int mq, int buf) {
        if (sr < 0 || sr >= 3 * CH) return;
        const float *gp = P.g, *bp = P.beta;
        uint32_t nb = 0;
        if (sr < CH) {
            const int tok = Uq.s + Uq.prompt + CH * mq + sr;
            if (tok >= Uq.s && tok < Uq.s + Uq.len) {
                gp = P.g + (int64_t)tok * H + Uq.h;
                bp = P.beta + (int64_t)tok * H + Uq.h;
                nb = 4;
            }
        } else if (mq >= 0 && V > 0) {
            const int idx = sr - CH, vw = idx >> 6, jj = idx & 63;
            const int rr = CH * mq + jj;
            if (vw < V && rr < Uq.R) {
                const int64_t row = (int64_t)vw * TR + Uq.roff + rr;
                gp = P.gn + row * H + Uq.h;
                bp = P.betan + row * H + Uq.h;
                nb = 4;
            }
        }
        (void)buf;
        if (nb && !GDN_IN_RANGE(P.ws, sr < CH ? (gp - P.g) < P.T * H : (gp - P.gn) < (int64_t)V * TR * H, 201)) nb = 0;
        cp_async4(&s_raw[0][sr], gp, nb);
        cp_async4(&s_raw[1][sr], bp, nb);
        cp_async_commit();
    };
    int rb = 0;      // s_raw buffer holding the next chunk to prepare
    int cb = 0;      // s_sc buffer of the current chunk
    // Scan the staged gates of chunk mq into scalar buffer `buf` (cumulative log2-decays, betas,
    // per-row factors) and stage the gates of chunk mq+1.  Called by all threads.
    auto prep_scalars = [&](const Unit &Uq, int mq, int buf) {   // warps 1..7 only
        cp_async_wait_all();
        float gv = 0.f, bv = 0.f;
        if (sr < 3 * CH) {
            gv = s_raw[0][sr] * kLog2e;
            bv = s_raw[1][sr];
        }
        rb ^= 1;
        if (mq + 1 < Uq.m_first + Uq.nchunks) stage_scalars(Uq, mq + 1, rb);
        float *sc = s_sc[buf];
        if (sr < CH) {                        // clean: inclusive scan over the chunk (warps 1, 2)
            sc[SC_BETA + sr] = bv;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const float o2 = __shfl_up_sync(0xffffffffu, gv, d);
                if (lane >= d) gv += o2;
            }
            s_g[sr] = gv;                      // per-warp inclusive scan
        } else if (mq >= 0 && V > 0 && sr < 3 * CH) {   // noisy: inclusive scan inside each block
            const int idx = sr - CH;
            sc[SC_NBETA + idx] = bv;
            const int jl = (idx & 63) % B;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const float o2 = __shfl_up_sync(0xffffffffu, gv, d);
                if (d < B && jl >= d) gv += o2;
            }
            sc[SC_NGAM + idx] = gv;
            if constexpr (B >= 16) {      // long blocks: the coefficients use precomputed factors
                sc[SC_NE + idx] = exp2f(gv);
                sc[SC_NF + idx] = exp2f(-gv);
                const bool okn = __all_sync(0xffffffffu, fabsf(gv) < 100.f);
                if (lane == 0) s_okn[buf][idx >> 5] = okn;
            }
        }
        bar_side();
        if (sr < CH) {
            const float gm = s_g[sr] + (sr >= 32 ? s_g[31] : 0.f);
            sc[SC_GAM + sr] = gm;
            sc[SC_E + sr] = exp2f(gm);
            sc[SC_F + sr] = exp2f(-gm);
            // e^{gamma_t - gamma_i} = E_t F_i is used only while every |gamma| of the chunk is
            // far from the fp32 exponent range; otherwise the difference is exponentiated.
            const bool okf = __all_sync(0xffffffffu, fabsf(gm) < 100.f);
            if (lane == 0) s_okw[buf][sr >> 5] = okf;
        }
    };

    // With few units each one is split over two CTAs: part 0 runs chunks [0, split) in full; part 1
    // runs [0, split) clean-only (no noisy rows, no outputs: only the state chain, which does not
    // depend on the noisy stream) and then [split, n) in full.  The split balances the two parts
    // for a clean-only chunk costing kCleanCost of a full one (lower for long blocks, whose noisy
    // work weighs more).
    constexpr float kCleanCost = B >= 32 ? 0.42f : (B >= 16 ? 0.55f : 0.65f);   // measured balance
    static_assert(4 * kAtQuadBytes<B> <= 16384, "block coefficients must fit the Khat buffer");
    // Work items are (unit, part), longest documents first; each CTA starts with item blockIdx.x and
    // then takes the next untaken item from a counter in the workspace (greedy list scheduling:
    // uneven documents no longer pile up on the CTAs that a fixed stride would give them).
    const int parts = P.parts;
    __shared__ int s_next;
    bool stop = false;        // uniform over the CTA: leave the work loop (a wait gave up)
    for (int w = blockIdx.x; w < P.num_units * parts; w = next_work_item(P.ws, &s_next)) {
        const int u = w / parts, part = w % parts;
        const Unit U = make_unit(P, u);
        int ci_full = 0, ci_end = U.nchunks;   // chunks ci < ci_full are clean-only
        bool final_part = true;
        if (parts == 2) {
            if (U.nchunks < 2) {
                if (part == 0) continue;
            } else {
                const int npre = -U.m_first;
                int split = (int)((U.nchunks + npre * (1.f - kCleanCost)) / (2.f - kCleanCost) + 0.5f);
                split = max(1, min(U.nchunks - 1, split));
                if (part == 0) {
                    ci_end = split;
                    final_part = false;
                } else {
                    ci_full = split;
                }
            }
        }
        auto chunk_noisy = [&](int ci) { return (U.m_first + ci >= 0) && V > 0 && ci >= ci_full; };
        float S[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) S[c] = 0.f;
        {
            // zero S0 (bf16): thread (rho, ch) owns row rho of v-half ch
            uint8_t *s0 = sm + OFF_S0 + ch * 16384;
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) *reinterpret_cast<uint4 *>(s0 + sw128_off(rho, c8)) = z;
            fence_async_smem();
            if (U.nchunks == 0 && final_part && GDN_IN_RANGE(P.ws, U.n < P.N && U.h < H, 203)) {
                float *fs = P.final_state + ((int64_t)U.n * H + U.h) * D * D + (int64_t)rho * D + 64 * ch;
#pragma unroll
                for (int c = 0; c < 64; c += 4) *reinterpret_cast<float4 *>(fs + c) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        if (tid == 0 && ci_end > 0) {
            issue_a(U, U.m_first, chunk_noisy(0));
            issue_b(U, U.m_first, chunk_noisy(0));
        }
        for (int ci = 0; ci < ci_end; ++ci) {
            const int m = U.m_first + ci;
            const bool noisy = chunk_noisy(ci);
            const bool last = ci == ci_end - 1;
            const int cstart = U.s + U.prompt + CH * m;   // global token of chunk row 0
            // whole chunks inside the document leave by TMA stores staged in free tiles: O in
            // the [P;T] tile after S2, the noisy rows in the K-hat and [P;T] tiles after S3 (not
            // with the in-kernel conv, whose weights live in the K-hat tile at the chunk top)
            const bool o_tma = cstart >= U.s && cstart + CH <= U.s + U.len && ci >= ci_full;
            // a clean-only chunk of a split unit only carries the state: no P, PT or O
            const bool need_o = ci >= ci_full;
            const bool n_tma = noisy && !conv && CH * m + CH <= U.R;
            float *s_gam = s_sc[cb] + SC_GAM, *s_beta = s_sc[cb] + SC_BETA;
            float *s_E = s_sc[cb] + SC_E, *s_F = s_sc[cb] + SC_F;
            float *s_ngam = s_sc[cb] + SC_NGAM, *s_nbeta = s_sc[cb] + SC_NBETA;
            const float *s_nE = s_sc[cb] + (B >= 16 ? SC_NE : 0), *s_nF = s_sc[cb] + (B >= 16 ? SC_NF : 0);
            if (ci == 0 && warp > 0) {
                stage_scalars(U, m, rb);
                prep_scalars(U, m, cb);
            }
            // ---- conv weights of this head (cp.async into the K-hat buffer, free until PE1) ----
            if (conv) {
                for (int it = tid; it < 3 * 128 * 4; it += kThreads) {   // (tensor X, channel c, tap j)
                    const int X = it >> 9, c = (it >> 2) & 127, j = it & 3;
                    const int dst = (X * 128 + ((c & 7) >> 1) * 32 + (j >> 1) * 16 + (c >> 3)) * 4 + (j & 1) * 2 + (c & 1);
                    const int64_t wi = (((int64_t)X * H + U.h) * 128 + c) * 4 + j;
                    cp_async4(sm + OFF_CW + dst * 4, P.conv_w + wi, GDN_IN_RANGE(P.ws, wi < 3LL * H * 128 * 4, 202) ? 4 : 0);
                }
                cp_async_commit();
            }
            // ---- wait for this chunk's tiles ----
            wait_bar(&bar_a, ph_a, 1);
            if (conv) {
                wait_bar(&bar_b, ph_b, 2);
                cp_async_wait_all();
                // The state rows wait in tensor memory (columns free until the batch MMAs) while
                // the conv needs the registers.
                {
                    float t0[32], t1[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) { t0[c] = S[c]; t1[c] = S[32 + c]; }
                    tmem_st32(tmem_addr(tb, q * 32, TM_N + 64 * ch), t0);
                    tmem_st32(tmem_addr(tb, q * 32, TM_N + 64 * ch + 32), t1);
                    tmem_wait_st();
                }
                __syncwarp();
                bar_all();
                conv_chunk<B>(sm, s_halo, noisy, U.s - cstart, tid);
                {
                    float t0[32], t1[32];
                    tmem_ld32(tmem_addr(tb, q * 32, TM_N + 64 * ch), t0);
                    tmem_ld32(tmem_addr(tb, q * 32, TM_N + 64 * ch + 32), t1);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) { S[c] = t0[c]; S[32 + c] = t1[c]; }
                }
            }
            __syncwarp();
            if ((stop = abort_check())) break;
            const bool fact = s_okw[cb][0] && s_okw[cb][1];
            // Route I export: blocks that start in this chunk (its rows are response positions)
            constexpr int kNbE = EXPORT ? CH / B : 0;
            const int eb0 = (CH * m) / B, enb = U.R / B;     // first block of the chunk, blocks in all
            const bool exporting = EXPORT && need_o && m >= 0;
            auto blob = [&](int b) {
                return static_cast<uint8_t *>(P.states) + ((int64_t)(U.roff / B + b) * H + U.h) * 32768;
            };

            // ================= PK1: [Q;K]K^T now, the noisy products once group B is in ========
            if (tid == 0) {
                tc_fence_after();
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tb + TM_TK, dK_qk + (off >> 4), dK_qk + ((8192 + off) >> 4),
                             make_idesc_bf16(128, 64, 0, 0), kk > 0);
                }
                // the last chunk's output stores have read the K-hat and [P;T] tiles before this
                // barrier completes: those tiles are next written after it
                bulk_wait_read_all();
                commit_mma();
                if constexpr (EXPORT) {
                    // the first block starts from S0 (stored after the wait above, so that the
                    // products need not wait for it; S0 is rewritten only after S3)
                    if (exporting && eb0 < enb && !dead) {
                        bulk_store(blob(eb0), sm + OFF_S0, 32768);
                        bulk_commit();
                    }
                }
            }
            __syncwarp();
            // Khat = diag(e^{gamma_C - gamma_t}) K  (MN-major A tile, same swizzled layout), built by
            // warps 1..7 in the S2 phase, before the next chunk's tiles replace K: until PK1
            // completes its buffer still feeds the last chunk's noisy output stores, and with
            // B >= 16 it then stages the noisy block coefficients.
            auto build_khat = [&] {
                const float gC = s_gam[CH - 1];
                for (int it = tid - 32; it >= 0 && it < 64 * 16; it += kMathThreads - 32) {
                    const int t = it >> 4, c16 = it & 15, hf = c16 >> 3, c8 = c16 & 7;
                    float f[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_QK + hf * 16384 + sw128_off(64 + t, c8)), f);
                    const float sc = fact ? s_E[CH - 1] * s_F[t] : exp2f(fminf(gC - s_gam[t], 0.f));
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] *= sc;
                    *reinterpret_cast<uint4 *>(sm + OFF_KH + hf * 8192 + sw128_off(t, c8)) = pack8(f);
                }
            };
            if (!conv) wait_bar(&bar_b, ph_b, 2);   // V and [k~0;k~1]
            __syncwarp();
            if (noisy && tid == 0) {
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tb + TM_R0, dK_nq + (off >> 4), dK_nk + (off >> 4),
                             make_idesc_bf16(128, 128, 0, 0), kk > 0);
                    mma_bf16(tb + TM_R1, dK_nk + (off >> 4), dK_nk + (off >> 4),
                             make_idesc_bf16(128, 128, 0, 0), kk > 0);
                }
                mma_commit(&bar_mma2);
            }
            __syncwarp();
            wait_mma(10);
            // clean: P rows (lanes 0-63, bf16 packed in registers until the solve is done) and
            // A rows (lanes 64-127) into the fp32 scratch
            uint4 ppk[4];
            if (fact) {
                float tk[32];
                tmem_ld32(tmem_addr(tb, q * 32, TM_TK + 32 * ch), tk);
                tmem_wait_ld();
                if (rho < 64) {
                    const int t = rho;
                    const float Et = s_E[t];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int i = 32 * ch + c;
                        tk[c] = (i <= t && need_o) ? tk[c] * (Et * s_F[i]) : 0.f;
                    }
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) ppk[c4] = pack8(tk + 8 * c4);
                } else {
                    const int t = rho - 64;
                    const float bEt = s_beta[t] * s_E[t];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int i = 32 * ch + c;
                        tk[c] = (i < t) ? (bEt * s_F[i]) * tk[c] : 0.f;
                    }
#pragma unroll
                    for (int g4 = 0; g4 < 8; ++g4)
                        *srow4(scratch, t, 32 * ch + 4 * g4) = make_float4(tk[4 * g4], tk[4 * g4 + 1], tk[4 * g4 + 2], tk[4 * g4 + 3]);
                }
            } else {
                const Rows4 r = pa_rows_exact(tmem_addr(tb, q * 32, TM_TK + 32 * ch), rho, ch, s_gam, s_beta, scratch);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) ppk[c4] = r.v[c4];
            }
            if (noisy) wait_mma2(11);                   // noisy block products of PK1
            // noisy: block coefficients, then W~ and -Y~ rows into TMEM as A operands
            float gend = 0.f;
            if (noisy) {
                const bool nfact = B >= 16 && s_okn[cb][0] && s_okn[cb][1] && s_okn[cb][2] && s_okn[cb][3];
                gend = noisy_phase1<B>(tb, q, ch, lane, rho, s_ngam, s_nbeta, s_nE, s_nF, nfact,
                                      reinterpret_cast<float *>(sm + OFF_KH + q * kAtQuadBytes<B>));
            }
            tmem_wait_st();
            tc_fence_before();
            bar_math();
            // On the tensor cores while the solve runs: [Q;K] S0 -> TM_R0 and, for the noisy rows,
            // W~V~ -> TM_N and (-Y~)K~ -> TM_R1 (A operands in TMEM).
            if (tid == 0) {
                tc_fence_after();
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tb + TM_R0, dK_qk + (off >> 4), dM_s0 + ((kk * 2048) >> 4),
                             make_idesc_bf16(128, 128, 0, 1), kk > 0);
                }
                if (noisy) {
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tb + TM_N, tb + TM_TK + kk * 8, dM_nv + ((kk * 2048) >> 4),
                                    make_idesc_bf16(128, 128, 0, 1), kk > 0);
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tb + TM_R1, tb + TM_TK + 64 + kk * 8, dM_nk + ((kk * 2048) >> 4),
                                    make_idesc_bf16(128, 128, 0, 1), kk > 0);
                }
                commit_mma();
            }
            __syncwarp();
            solve_T(scratch, wstage, tid, warp);
            // [P ; T] as bf16 K-major A (128 rows x 64): this thread writes row rho, cols [32ch, 32ch+32)
            if (rho >= 64) {
                const int t = rho - 64;
                const bool lowleft = t >= 32 && ch == 0;          // the 32-merge's block
#pragma unroll
                for (int g4 = 0; g4 < 4; ++g4) {
                    const float4 a = lowleft ? *wrow4(wstage, t - 32, 8 * g4) : *srow4(scratch, t, 32 * ch + 8 * g4);
                    const float4 b = lowleft ? *wrow4(wstage, t - 32, 8 * g4 + 4) : *srow4(scratch, t, 32 * ch + 8 * g4 + 4);
                    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                    ppk[g4] = pack8(f);
                }
            }
            bar_math();
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) *reinterpret_cast<uint4 *>(sm + OFF_Y + sw128_off(rho, 4 * ch + c4)) = ppk[c4];
            wait_mma(15);
            // R = beta V - beta Gamma (K S0), over V (K S0 are rows 64..127 of TM_R0)
            if (rho >= 64) {
                const int t = rho - 64;
                const float bt = s_beta[t], bg = bt * s_E[t];
                uint8_t *vrow = sm + OFF_V + ch * 8192;
                float ksb[2][32];
                tmem_ld32(tmem_addr(tb, q * 32, TM_R0 + 64 * ch), ksb[0]);
                tmem_ld32(tmem_addr(tb, q * 32, TM_R0 + 64 * ch + 32), ksb[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float (&ks)[32] = ksb[hf];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        float f[8];
                        const uint32_t o = sw128_off(t, 4 * hf + c4);
                        unpack8(*reinterpret_cast<const uint4 *>(vrow + o), f);
#pragma unroll
                        for (int x = 0; x < 8; ++x) f[x] = bt * f[x] - bg * ks[8 * c4 + x];
                        *reinterpret_cast<uint4 *>(vrow + o) = pack8(f);
                    }
                }
            }
            if (noisy) {
                const int eb = ((rho & 63) / B) * B - 1;     // the row's block boundary (-1: S0)
                z_epilogue(sm, tb, q, ch, rho, gend, (fact && eb >= 0) ? s_E[eb] : 1.f);
            }
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            if ((stop = abort_check())) break;

            // ================= PK2 (not in a clean-only chunk: PT feeds only O) =================
            if (need_o) {
                if (tid == 0) {
                    tc_fence_after();
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tb + TM_TK, dK_y + ((kk * 32) >> 4),
                                 dM_t + ((kk * 2048) >> 4), make_idesc_bf16(128, 64, 0, 1), kk > 0);
                    if (noisy) {
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            mma_bf16(tb + TM_ZK, dK_nq + (off >> 4), dK_qk + ((8192 + off) >> 4),
                                     make_idesc_bf16(128, 64, 0, 0), kk > 0);
                        }
                    }
                    commit_mma();
                }
                __syncwarp();
                wait_mma(20);
                if (rho < 64) {
                    float pt[32];
                    tmem_ld32(tmem_addr(tb, q * 32, TM_TK + 32 * ch), pt);
                    tmem_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        *reinterpret_cast<uint4 *>(sm + OFF_Y + sw128_off(rho, 4 * ch + c4)) = pack8(pt + 8 * c4);
                }
                if (noisy) {
                    const int e = ((rho & 63) / B) * B - 1;   // chunk-local boundary row (-1: S0)
                    if (fact) {
                        float zk[32];
                        tmem_ld32(tmem_addr(tb, q * 32, TM_ZK + 32 * ch), zk);
                        tmem_wait_ld();
                        // the rows already hold Gamma_e Z: M'_Z = (Gamma_e Z K^T) e^{-gamma_i} [i <= e]
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int i = 32 * ch + c;
                            zk[c] = (i <= e) ? zk[c] * s_F[i] : 0.f;
                        }
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)    // M'_Z: K-major 128 x 64 in d-half 0 of the k~ tile
                            *reinterpret_cast<uint4 *>(sm + OFF_NK + sw128_off(rho, 4 * ch + c4)) = pack8(zk + 8 * c4);
                    } else {
                        mz_rows_exact(sm + OFF_NK, sm + OFF_NQ, tmem_addr(tb, q * 32, TM_ZK + 32 * ch), rho, ch, e, s_gam, s_E);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                if ((stop = abort_check())) break;
            }

            // ================= S2: [PT;T] R and the noisy rows' state product =================
            if (tid == 0) {
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tb + TM_R1, dK_y + ((kk * 32) >> 4), dM_v + ((kk * 2048) >> 4),
                             make_idesc_bf16(128, 128, 0, 1), kk > 0);
                if (noisy) {
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_bf16(tb + TM_N, dK_nq + (off >> 4), dM_s0 + ((kk * 2048) >> 4),
                                 make_idesc_bf16(128, 128, 0, 1), 1u);
                    }
                }
                commit_mma();
            }
            __syncwarp();
            // Khat reads K from the [Q;K] tile: warps 1..7 build it, then signal warp 0, whose
            // lane 0 lets the next chunk's group A overwrite the tile once [Q;K] and Z are consumed.
            if (warp > 0) {
                build_khat();
                if constexpr (EXPORT) {
                    // Khat_e for the block starting at row j B (e = j B - 1), j >= 1: K rows i <= e
                    // scaled by e^{gamma_e - gamma_i}, the rest zero; MN-major A tiles at NQ
                    if (exporting) {
                        for (int it = tid - 32; it < 64 * 16; it += kMathThreads - 32) {
                            const int t = it >> 4, c16 = it & 15, hf = c16 >> 3, c8 = c16 & 7;
                            float f[8], g8[8];
                            unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_QK + hf * 16384 + sw128_off(64 + t, c8)), f);
#pragma unroll
                            for (int j = 1; j < kNbE; ++j) {
                                const int e = j * B - 1;
                                const float sc = t <= e ? exp2f(s_gam[e] - s_gam[t]) : 0.f;
#pragma unroll
                                for (int x = 0; x < 8; ++x) g8[x] = f[x] * sc;
                                *reinterpret_cast<uint4 *>(sm + OFF_NQ + (j - 1) * 16384 + hf * 8192 + sw128_off(t, c8)) =
                                    pack8(g8);
                            }
                        }
                        fence_async_smem();
                    }
                }
                bar_arrive_khat();
            } else {
                bar_sync_khat();
                if (tid == 0 && !last && !dead) {
                    if (!kwait<TW>(&bar_mma, ph_mma & 1, kWaitIters, P.wait_iters)) {
                        dead = true;
                        fail(40);
                    } else {
                        issue_a(U, m + 1, chunk_noisy(ci + 1));
                    }
                }
                __syncwarp();
            }
            if (!last && warp > 0) prep_scalars(U, m + 1, cb ^ 1);   // next chunk's scalars meanwhile
            wait_mma(40);
            if (rho < 64) {
                if (need_o) {
                    const int t = rho;
                    const int tok = cstart + t;
                    const bool ok = tok >= U.s && tok < U.s + U.len && ci >= ci_full;
                    const float Gt = s_E[t];
                    __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(P.out) + ((int64_t)tok * H + U.h) * D + 64 * ch;
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        float qs[32], pu[32];
                        tmem_ld32(tmem_addr(tb, q * 32, TM_R0 + 64 * ch + 32 * hf), qs);
                        tmem_ld32(tmem_addr(tb, q * 32, TM_R1 + 64 * ch + 32 * hf), pu);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 32; ++x) qs[x] = (Gt * qs[x] + pu[x]) * scale;
                        if (o_tma) {
#pragma unroll
                            for (int c4 = 0; c4 < 4; ++c4)
                                *reinterpret_cast<uint4 *>(sm + OFF_Y + ch * 8192 + sw128_off(t, 4 * hf + c4)) = pack8(qs + 8 * c4);
                        } else if (ok && GDN_IN_RANGE(P.ws, tok >= 0 && tok < P.T, 205)) {
#pragma unroll
                            for (int c4 = 0; c4 < 4; ++c4)
                                *reinterpret_cast<uint4 *>(orow + 32 * hf + 8 * c4) = pack8(qs + 8 * c4);
                        }
                    }
                }
            } else {
                const int t = rho - 64;
                uint8_t *vrow = sm + OFF_V + ch * 8192;
                float uub[2][32];
                tmem_ld32(tmem_addr(tb, q * 32, TM_R1 + 64 * ch), uub[0]);
                tmem_ld32(tmem_addr(tb, q * 32, TM_R1 + 64 * ch + 32), uub[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float (&uu)[32] = uub[hf];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        *reinterpret_cast<uint4 *>(vrow + sw128_off(t, 4 * hf + c4)) = pack8(uu + 8 * c4);
                }
            }
            fence_async_smem();
            tc_fence_before();
            if ((stop = abort_check())) break;

            // ================= S3 =================
            if (tid == 0) {
                tc_fence_after();
                bool o_stored = false;
                if (o_tma && !dead && GDN_IN_RANGE(P.ws, cstart >= 0 && cstart + CH <= P.T, 206)) {
                    tma_store_3d(&M.o, sm + OFF_Y, 0, U.h, cstart);
                    tma_store_3d(&M.o, sm + OFF_Y + 8192, 64, U.h, cstart);
                    bulk_commit();
                    o_stored = true;
                }
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tb + TM_R0, dM_kh + ((kk * 2048) >> 4), dM_v + ((kk * 2048) >> 4),
                             make_idesc_bf16(128, 128, 1, 1), kk > 0);
                if (noisy) {
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tb + TM_N, dK_nk + ((kk * 32) >> 4), dM_v + ((kk * 2048) >> 4),
                                 make_idesc_bf16(128, 128, 0, 1), 1u);
                }
                if constexpr (EXPORT) {
                    if (exporting) {
                        for (int j = 1; j < kNbE; ++j) {
                            if (eb0 + j >= enb) break;
                            const uint64_t dM_khe = make_sdesc(smem_u32(sm + OFF_NQ + (j - 1) * 16384), 8192, 1024);
                            for (int kk = 0; kk < 4; ++kk)
                                mma_bf16(tb + export_col(j), dM_khe + ((kk * 2048) >> 4), dM_v + ((kk * 2048) >> 4),
                                         make_idesc_bf16(128, 128, 1, 1), kk > 0);
                        }
                    }
                    // the S0 blob has been read before the update rewrites S0; the output tile's store,
                    // the newest bulk group when issued just above, may still be reading
                    if (o_stored) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                    else bulk_wait_read_all();
                }
                commit_mma();
                if (!last && !dead) {
                    if (!kwait<TW>(&bar_mma, ph_mma & 1, kWaitIters, P.wait_iters)) {
                        dead = true;
                        fail(50);
                    } else {
                        issue_b(U, m + 1, chunk_noisy(ci + 1));
                    }
                }
                if (o_tma && n_tma) {          // the noisy rows are staged over the O tile
                    bulk_wait_read_all();
                    mbar_arrive(&bar_ost);
                }
            }
            __syncwarp();
            wait_mma(50);
            const float GC = s_E[CH - 1];
            uint8_t *srow = sm + OFF_S0 + ch * 16384;
            if constexpr (EXPORT) {
                if (exporting) {
                    for (int j = 1; j < kNbE; ++j) {
                        if (eb0 + j >= enb) break;
                        const float Ge = s_E[j * B - 1];
                        uint8_t *st = sm + OFF_NQ + (j - 1) * 32768 + ch * 16384;
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            float ex[32];
                            tmem_ld32(tmem_addr(tb, q * 32, export_col(j) + 64 * ch + 32 * hf), ex);
                            tmem_wait_ld();
#pragma unroll
                            for (int x = 0; x < 32; ++x) ex[x] = fmaf(Ge, S[32 * hf + x], ex[x]);
#pragma unroll
                            for (int c4 = 0; c4 < 4; ++c4)
                                *reinterpret_cast<uint4 *>(st + sw128_off(rho, 4 * hf + c4)) = pack8(ex + 8 * c4);
                        }
                    }
                }
            }
            {
                float ds0[32], ds1[32];
                tmem_ld32(tmem_addr(tb, q * 32, TM_R0 + 64 * ch), ds0);
                tmem_ld32(tmem_addr(tb, q * 32, TM_R0 + 64 * ch + 32), ds1);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    S[x] = fmaf(GC, S[x], ds0[x]);
                    S[32 + x] = fmaf(GC, S[32 + x], ds1[x]);
                }
            }
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8)
                *reinterpret_cast<uint4 *>(srow + sw128_off(rho, c8)) = pack8(S + 8 * c8);
            if (last && final_part && GDN_IN_RANGE(P.ws, U.n < P.N && U.h < H, 204)) {
                float *fs = P.final_state + ((int64_t)U.n * H + U.h) * D * D + (int64_t)rho * D + 64 * ch;
#pragma unroll
                for (int c = 0; c < 64; c += 4)
                    *reinterpret_cast<float4 *>(fs + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
            }
            if (o_tma && n_tma) {
                wait_bar(&bar_ost, ph_ost, 60);
                __syncwarp();            // reconverge before the warp-collective tcgen05.ld
            }
            if (noisy) {
                const int vw = rho >> 6, jj = rho & 63;
                const int rr = CH * m + jj;
                const bool ok = vw < V && rr < U.R;
                __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(P.out_noisy) +
                                      (((int64_t)vw * TR + U.roff + rr) * H + U.h) * D + 64 * ch;
                float onb[2][32];
                tmem_ld32(tmem_addr(tb, q * 32, TM_N + 64 * ch), onb[0]);
                tmem_ld32(tmem_addr(tb, q * 32, TM_N + 64 * ch + 32), onb[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float (&on)[32] = onb[hf];
#pragma unroll
                    for (int x = 0; x < 32; ++x) on[x] *= scale;
                    if (n_tma) {            // view vw's tile: 16 KB at K-hat (view 0) / [P;T] (view 1)
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            *reinterpret_cast<uint4 *>(sm + OFF_KH + vw * 16384 + ch * 8192 + sw128_off(jj, 4 * hf + c4)) =
                                pack8(on + 8 * c4);
                    } else if (ok && GDN_IN_RANGE(P.ws, (int64_t)vw * TR + U.roff + rr < (int64_t)V * TR, 207)) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            *reinterpret_cast<uint4 *>(orow + 32 * hf + 8 * c4) = pack8(on + 8 * c4);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            cb ^= 1;
            if ((stop = abort_check())) break;
            if constexpr (EXPORT) {
                if (tid == 0 && exporting && !dead) {
                    for (int j = 1; j < kNbE; ++j) {
                        if (eb0 + j >= enb) break;
                        bulk_store(blob(eb0 + j), sm + OFF_NQ + (j - 1) * 32768, 32768);
                    }
                    bulk_commit();
                }
            }
            if (tid == 0 && n_tma && !dead) {
                for (int vw = 0; vw < V && vw < 2; ++vw) {
                    const int64_t row0 = (int64_t)vw * TR + U.roff + CH * m;
                    if (!GDN_IN_RANGE(P.ws, row0 >= 0 && row0 + CH <= (int64_t)V * TR, 208)) continue;
                    for (int hf = 0; hf < 2; ++hf)
                        tma_store_3d(&M.on, sm + OFF_KH + vw * 16384 + hf * 8192, hf * 64, U.h, (int)row0);
                }
                bulk_commit();
            }
        }
        if (stop) break;
    }
    // Drain (thread 0): the output stores complete; then (immediate unless a wait gave up) the last
    // TMA load on each barrier and, with one more commit, every MMA.  Then the cp.async groups.
    if (tid == 0) {
        bulk_wait_all();
        if (s_iss[0] > 0) mbar_wait(&bar_a, (s_iss[0] - 1) & 1, kDrainWaitIters);
        if (s_iss[1] > 0) mbar_wait(&bar_b, (s_iss[1] - 1) & 1, kDrainWaitIters);
        if (stop) {
            mma_commit(&bar_drain);
            mbar_wait(&bar_drain, 0, kDrainWaitIters);
        }
    }
    cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 512);
}

}  // namespace

bool chunked_supported(int dtype, int d, int B, int conv_width) {
    return dtype == GDN_BF16 && d == D && (conv_width == 0 || conv_width == 4) && B >= 1 && B <= 32 && (32 % B) == 0;
}

namespace {

// One launch over at most two noisy views: the pipelined kernel, or this file's in-order kernel.
cudaError_t launch_chunked_views(const Params &p, bool pipelined, cudaStream_t stream) {
    if (pipelined) return launch_pipe(p, stream);
    Maps maps;
    const bool noisy = p.V > 0 && p.TR > 0;
    if (!encode_map(&maps.q, p.q, p.H, p.T) || !encode_map(&maps.k, p.k, p.H, p.T) ||
        !encode_map(&maps.v, p.v, p.H, p.T) || !encode_map(&maps.o, p.out, p.H, p.T))
        return cudaErrorInvalidValue;
    if (noisy) {
        if (!encode_map(&maps.qn, p.qn, p.H, (int64_t)p.V * p.TR) || !encode_map(&maps.kn, p.kn, p.H, (int64_t)p.V * p.TR) ||
            !encode_map(&maps.vn, p.vn, p.H, (int64_t)p.V * p.TR) ||
            !encode_map(&maps.on, p.out_noisy, p.H, (int64_t)p.V * p.TR))
            return cudaErrorInvalidValue;
    } else {
        maps.qn = maps.q;
        maps.kn = maps.k;
        maps.vn = maps.v;
        maps.on = maps.o;
    }
    static int num_sms = 0;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
        cudaError_t e = cudaSuccess;
        for (auto fn : {gdn_chunked_kernel<1>, gdn_chunked_kernel<2>, gdn_chunked_kernel<4>,
                        gdn_chunked_kernel<8>, gdn_chunked_kernel<16>, gdn_chunked_kernel<32>,
                        gdn_chunked_kernel<1, false, true>, gdn_chunked_kernel<2, false, true>,
                        gdn_chunked_kernel<4, false, true>, gdn_chunked_kernel<8, false, true>,
                        gdn_chunked_kernel<16, false, true>, gdn_chunked_kernel<32, false, true>,
                        gdn_chunked_kernel<4, true>, gdn_chunked_kernel<4, true, true>,
                        gdn_chunked_kernel<16, false, false, true>, gdn_chunked_kernel<32, false, false, true>}) {
            cudaError_t r = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
            if (r != cudaSuccess) e = r;
        }
        attr_err = e;
    });
    if (attr_err != cudaSuccess) return attr_err;
    // Few units: two CTAs per unit (see the kernel's unit loop).
    const int sms = num_sms > 0 ? num_sms : 148;
    Params q = p;
    q.parts = ((noisy || p.states) && 2 * p.num_units <= sms) ? 2 : 1;
    const int grid = std::min(p.num_units * q.parts, sms);
    const bool conv = p.conv_width > 0;
    if (p.states) {              // Route I's first stage: no views, no ShortConv, B = 16 or 32
        if (noisy || conv || p.wait_test) return cudaErrorNotSupported;
        if (p.B == 16) gdn_chunked_kernel<16, false, false, true><<<grid, kThreads, SMEM_BYTES, stream>>>(q, maps);
        else if (p.B == 32) gdn_chunked_kernel<32, false, false, true><<<grid, kThreads, SMEM_BYTES, stream>>>(q, maps);
        else return cudaErrorNotSupported;
        return cudaGetLastError();
    }
    if (p.wait_test) {           // the test entry point: B = 4 only
        if (p.B != 4) return cudaErrorNotSupported;
        if (conv) gdn_chunked_kernel<4, true, true><<<grid, kThreads, SMEM_BYTES, stream>>>(q, maps);
        else gdn_chunked_kernel<4, true><<<grid, kThreads, SMEM_BYTES, stream>>>(q, maps);
        return cudaGetLastError();
    }
#define GDN_CHUNKED_CASE(b)                                                                        \
    case b:                                                                                        \
        if (conv) gdn_chunked_kernel<b, false, true><<<grid, kThreads, SMEM_BYTES, stream>>>(q, maps); \
        else gdn_chunked_kernel<b><<<grid, kThreads, SMEM_BYTES, stream>>>(q, maps);              \
        break;
    switch (p.B) {
        GDN_CHUNKED_CASE(1)
        GDN_CHUNKED_CASE(2)
        GDN_CHUNKED_CASE(4)
        GDN_CHUNKED_CASE(8)
        GDN_CHUNKED_CASE(16)
        GDN_CHUNKED_CASE(32)
        default: return cudaErrorInvalidValue;
    }
#undef GDN_CHUNKED_CASE
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunked(const Params &p, bool pipelined, cudaStream_t stream) {
    if (p.num_units == 0) return cudaSuccess;
    // Every document empty: nothing to read, and each final state is the zero initial state.
    if (p.T == 0) return cudaMemsetAsync(p.final_state, 0, (size_t)p.num_units * D * D * sizeof(float), stream);
    if (p.V <= 2) return launch_chunked_views(p, pipelined, stream);
    // More than two views: one launch per pair of views.  Each launch recomputes the clean
    // stream (the views only share the clean boundary states) and rewrites the same clean
    // outputs; the work counter in the workspace restarts at zero for every launch.
    const int64_t row = p.TR * p.H;          // elements of one view's [T_R, H] plane
    for (int v0 = 0; v0 < p.V; v0 += 2) {
        Params q = p;
        q.V = std::min(2, p.V - v0);
        q.qn = static_cast<const __nv_bfloat16 *>(p.qn) + v0 * row * D;
        q.kn = static_cast<const __nv_bfloat16 *>(p.kn) + v0 * row * D;
        q.vn = static_cast<const __nv_bfloat16 *>(p.vn) + v0 * row * D;
        q.gn = p.gn + v0 * row;
        q.betan = p.betan + v0 * row;
        q.out_noisy = static_cast<__nv_bfloat16 *>(p.out_noisy) + v0 * row * D;
        if (v0 > 0) {
            cudaError_t e = cudaMemsetAsync(&p.ws->next_unit, 0, sizeof(int32_t), stream);
            if (e != cudaSuccess) return e;
        }
        cudaError_t e = launch_chunked_views(q, pipelined, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdn
