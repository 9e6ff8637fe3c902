// gdn_chunk_common.cuh -- device helpers shared by the two chunked tensor-core kernels of the
// dual-stream Gated DeltaNet forward (gdn_chunked.cu: in-order, with the ShortConv prologue;
// gdn_pipe.cu: warp-specialised pipeline), and the host-side tensor-map encoder.  Not part of the
// public ABI.  Everything has internal linkage: each translation unit gets its own copy.
#pragma once

#include <cudaTypedefs.h>
#include <mutex>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int D = 128;                 // d_k = d_v
constexpr int CH = 64;                 // chunk length

struct Maps {
    CUtensorMap q, k, v, qn, kn, vn;
    CUtensorMap o, on;            // outputs (TMA stores of whole chunks)
};

__device__ __forceinline__ uint4 pack8(const float *f) {
    uint4 r;
    __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
    __nv_bfloat162 c = __floats2bfloat162_rn(f[4], f[5]);
    __nv_bfloat162 d = __floats2bfloat162_rn(f[6], f[7]);
    r.x = *reinterpret_cast<uint32_t *>(&a);
    r.y = *reinterpret_cast<uint32_t *>(&b);
    r.z = *reinterpret_cast<uint32_t *>(&c);
    r.w = *reinterpret_cast<uint32_t *>(&d);
    return r;
}

__device__ __forceinline__ void unpack8(uint4 u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
        float2 p = __bfloat1622float2(h);
        f[2 * i] = p.x;
        f[2 * i + 1] = p.y;
    }
}

// fp32 64x64 solve scratch: 16-byte chunk c>>2 of row r sits at chunk (c>>2) ^ (r & 7), so both
// row-segment accesses by one thread (float4) and column accesses across a warp avoid conflicts.
__device__ __forceinline__ int sidx(int r, int c) { return r * 64 + ((((c >> 2) ^ (r & 7))) << 2) + (c & 3); }
__device__ __forceinline__ float4 *srow4(float *sa, int r, int c4) {
    return reinterpret_cast<float4 *>(sa + r * 64 + ((((c4 >> 2) ^ (r & 7))) << 2));
}

struct Unit {
    int n, h;
    int s, len, prompt, R, roff;
    int nchunks, m_first;
};

__device__ __forceinline__ Unit make_unit(const Params &P, int u) {
    Unit U;
    U.n = P.unit_doc[u / P.H];
    U.h = u % P.H;
    U.s = P.doc_start[U.n];
    U.len = P.doc_start[U.n + 1] - U.s;
    U.prompt = P.doc_prompt[U.n];
    U.R = U.len - U.prompt;
    U.roff = P.resp_off[U.n];
    const int npre = (U.prompt + CH - 1) / CH;
    const int nres = (U.R + CH - 1) / CH;
    U.m_first = -npre;
    U.nchunks = npre + nres;
    return U;
}

// Block coefficients of one noisy row: y = Ptil_j Ttil (back substitution against the block's
// own I + Atil), then ycoef = y beta~ Gammatil (for Z) and wcoef = y beta~ (for WV).
// Shared-memory staging of the noisy block coefficients (B >= 16): per TMEM lane quadrant, 32
// rows of B fp32 values (one 16-byte pad between the two blocks of a quadrant when B = 16, so
// the two blocks' broadcast reads fall in different bank groups).
template <int B>
constexpr int kAtQuadBytes = 32 * B * 4 + (B < 32 ? 16 : 0);
template <int B>
__device__ __forceinline__ constexpr int at_swz(int r) { return B >= 32 ? (r & 7) : ((r >> 1) & 3); }

// STAGE: stage the block rows in shared memory (s_at) for the back substitution instead of moving
// them by warp shuffles (pays for B >= 16; needs 4 * kAtQuadBytes<B> bytes of shared memory).
template <int B, bool STAGE = (B >= 16)>
__device__ __forceinline__ void noisy_coeffs(const float (&wq)[32], const float (&wk)[32], int lane, int j,
                                             const float *ngam, const float *nbeta, const float *nE,
                                             const float *nF, bool nfact, float *s_at,
                                             float (&ycoef)[B], float (&wcoef)[B], float &gend) {
    const int bs = (j / B) * B;
    const int jl = j - bs;
    const int wofs = bs & 31;
    float aq[B], ak[B], gl[B], bl[B];
#pragma unroll
    for (int l = 0; l < B; ++l) {
        aq[l] = 0.f;
        ak[l] = 0.f;
        gl[l] = ngam[bs + l];
        bl[l] = nbeta[bs + l];
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        if ((c / B) * B == wofs) {
            aq[c % B] = wq[c];
            ak[c % B] = wk[c];
        }
    }
    const float gj = ngam[j], bj = nbeta[j];
    gend = gl[B - 1];
    float arow[B], pt[B], y[B];
    if (B >= 16 && nfact) {       // e^{gamma~_a - gamma~_b} = E_a F_b, prepared once per row
        const float Ej = nE[j], Eend = nE[bs + B - 1];
#pragma unroll
        for (int l = 0; l < B; ++l) {
            const float Fl = nF[bs + l];
            arow[l] = (l < jl) ? bj * (Ej * Fl) * ak[l] : 0.f;
            pt[l] = aq[l] * (Eend * Fl);
        }
    } else {
#pragma unroll
        for (int l = 0; l < B; ++l) {
            arow[l] = (l < jl) ? bj * exp2f(fminf(gj - gl[l], 0.f)) * ak[l] : 0.f;
            pt[l] = aq[l] * exp2f(gend - gl[l]);
        }
    }
    // Right-looking back substitution: once y_mm is final it is taken out of every earlier
    // position at once, so the dependent chain is B steps of one FMA each.
    if constexpr (STAGE) {
        // Row mm of the block's Atil is needed by every lane of the block: the rows go through
        // shared memory once and are read back as broadcast 16-byte loads (about B^2/8 loads
        // instead of B^2/2 shuffles).  16-byte column c4 of row r sits at c4 ^ at_swz(r), so the
        // row stores of 8 consecutive lanes hit 8 distinct bank groups; r & 7 of a block row is
        // mm & 7, known at compile time.
        float *myrow = s_at + lane * B + (B < 32 ? (lane / B) * 4 : 0);
#pragma unroll
        for (int c4 = 0; c4 < B / 4; ++c4)
            *reinterpret_cast<float4 *>(myrow + 4 * (c4 ^ at_swz<B>(jl))) =
                make_float4(arow[4 * c4], arow[4 * c4 + 1], arow[4 * c4 + 2], arow[4 * c4 + 3]);
        __syncwarp();
        const float *blk = myrow - jl * B;
#pragma unroll
        for (int mm = B - 1; mm >= 0; --mm) {
            y[mm] = pt[mm];
#pragma unroll
            for (int c4 = 0; c4 < (mm + 3) / 4; ++c4) {
                const float4 a = *reinterpret_cast<const float4 *>(blk + mm * B + 4 * (c4 ^ at_swz<B>(mm)));
                const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * c4 + e < mm) pt[4 * c4 + e] = fmaf(-y[mm], av[e], pt[4 * c4 + e]);
            }
        }
    } else {
        const int base = lane - jl;
#pragma unroll
        for (int mm = B - 1; mm >= 0; --mm) {
            y[mm] = pt[mm];
#pragma unroll
            for (int l = 0; l < mm; ++l) pt[l] = fmaf(-y[mm], __shfl_sync(0xffffffffu, arow[l], base + mm), pt[l]);
        }
    }
#pragma unroll
    for (int l = 0; l < B; ++l) {
        wcoef[l] = y[l] * bl[l];
        ycoef[l] = wcoef[l] * ((B >= 16 && nfact) ? nE[bs + l] : exp2f(gl[l]));
    }
}

// This thread's half (K columns [64ch, 64ch+64), i.e. the noisy rows of view ch) of the
// block-diagonal row `sign * coef` of noisy row (view v, block start bs), stored into tensor
// memory as bf16 pairs (low half = even k): an A operand for a tensor-memory MMA.
template <int B>
__device__ __forceinline__ void store_block_row(uint32_t taddr, int ch, int v, int bs, const float (&coef)[B],
                                                float sign) {
    float w[32];
    if constexpr (B == 1) {
        __nv_bfloat162 pr = (bs & 1) ? __floats2bfloat162_rn(0.f, sign * coef[0]) : __floats2bfloat162_rn(sign * coef[0], 0.f);
        const float pf = __uint_as_float(*reinterpret_cast<uint32_t *>(&pr));
#pragma unroll
        for (int x = 0; x < 32; ++x) w[x] = (ch == v && x == (bs >> 1)) ? pf : 0.f;
    } else {
        constexpr int HB = B / 2;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
            const int l0 = 2 * (x % HB);
            __nv_bfloat162 pr = __floats2bfloat162_rn(sign * coef[l0], sign * coef[l0 + 1]);
            const float pf = __uint_as_float(*reinterpret_cast<uint32_t *>(&pr));
            w[x] = (ch == v && (x / HB) == (bs / B)) ? pf : 0.f;
        }
    }
    tmem_st32(taddr, w);
}

// 32 x 32 fp32 staging block (the 32-merge's result): 128-byte rows, 16-byte chunks swizzled by
// the row like the solve scratch.
__device__ __forceinline__ int widx(int r, int c) { return r * 32 + ((((c >> 2) ^ (r & 7))) << 2) + (c & 3); }
__device__ __forceinline__ float4 *wrow4(float *w, int r, int c4) {
    return reinterpret_cast<float4 *>(w + r * 32 + ((((c4 >> 2) ^ (r & 7))) << 2));
}

// One merge of the triangular inverse by one warp that owns NC consecutive output columns
// [cb, cb + NC) of the S x S block below the diagonal at offset o.  With T11 = T[o.., o..] and
// T22 = T[o+S.., o+S..] already inverted (unit lower, zeros above the diagonal):
//   X = A[o+S.., o..] T11,   T[o+S.., o..] = -T22 X.
// Lane (g = lane / NC, cl = lane % NC) holds column cb + cl for the rows g + RG*i.  X moves between
// the lanes by shuffles, so the warp needs no barrier; T11[k][c] = 0 for k < c lets the first
// product start at k = cb, and the second product of row r stops at k = r (warp-uniform bounds).
// The result goes out through `store` (block-local row and column) after `before_store()`, which
// separates this warp's reads from other warps' writes when several warps share one merge.
template <int S, int NC, typename Store, typename Sync>
__device__ __forceinline__ void warp_merge(const float *sa, int o, int cb, int lane, Store store, Sync before_store) {
    constexpr int RG = 32 / NC, NR = S / RG;
    const int cl = lane % NC, g = lane / NC, c = cb + cl;
    float x[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) x[i] = 0.f;
#pragma unroll
    for (int k4 = 0; k4 < S; k4 += 4) {
        if (k4 < (cb & ~3)) continue;
        float tv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) tv[e] = sa[sidx(o + k4 + e, o + c)];
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            const float4 a = *srow4(const_cast<float *>(sa), o + S + g + RG * i, o + k4);
            x[i] = fmaf(a.w, tv[3], fmaf(a.z, tv[2], fmaf(a.y, tv[1], fmaf(a.x, tv[0], x[i]))));
        }
    }
    float y[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) y[i] = 0.f;
#pragma unroll
    for (int k4 = 0; k4 < S; k4 += 4) {
        float xk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) xk[e] = __shfl_sync(0xffffffffu, x[(k4 + e) / RG], ((k4 + e) % RG) * NC + cl);
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            if (k4 <= RG * i + RG - 1) {
                const float4 a = *srow4(const_cast<float *>(sa), o + S + g + RG * i, o + S + k4);
                y[i] = fmaf(a.w, xk[3], fmaf(a.z, xk[2], fmaf(a.y, xk[1], fmaf(a.x, xk[0], y[i]))));
            }
        }
    }
    before_store();
#pragma unroll
    for (int i = 0; i < NR; ++i) store(g + RG * i, c, -y[i]);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
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

// 3-D map over a [rows, H, 128] bf16 tensor; box = 64 rows x 1 head x 64 columns, 128B swizzle.
bool encode_map(CUtensorMap *m, const void *ptr, int H, int64_t rows) {
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Exact-decay variants of two epilogues, for a chunk whose cumulative decays leave the range in
// which e^{gamma_t - gamma_i} factorises as E_t F_i.  Such chunks are rare; out of line, they keep
// the common path's instruction footprint small.
struct Rows4 {
    uint4 v[4];
};

// P rows (rho < 64: returned as bf16) or A rows (rho >= 64: written to the fp32 solve scratch)
// of [Q;K]K^T (TMEM columns at taddr), with the decays exponentiated one by one.
__device__ __noinline__ Rows4 pa_rows_exact(uint32_t taddr, int rho, int ch, const float *s_gam,
                                           const float *s_beta, float *scratch) {
    float tk[32];
    tmem_ld32(taddr, tk);
    tmem_wait_ld();
    Rows4 r;
    if (rho < 64) {
        const int t = rho;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const int i = 32 * ch + c;
            tk[c] = (i <= t) ? tk[c] * exp2f(fminf(s_gam[t] - s_gam[i], 0.f)) : 0.f;
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) r.v[c4] = pack8(tk + 8 * c4);
    } else {
        const int t = rho - 64;
        const float bt = s_beta[t];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const int i = 32 * ch + c;
            tk[c] = (i < t) ? bt * exp2f(fminf(s_gam[t] - s_gam[i], 0.f)) * tk[c] : 0.f;
        }
#pragma unroll
        for (int g4 = 0; g4 < 8; ++g4)
            *srow4(scratch, t, 32 * ch + 4 * g4) = make_float4(tk[4 * g4], tk[4 * g4 + 1], tk[4 * g4 + 2], tk[4 * g4 + 3]);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) r.v[c4] = make_uint4(0u, 0u, 0u, 0u);
    }
    return r;
}

// M'_Z rows of a noisy row (Z K^T in TMEM at taddr; boundary row e of its block, -1 for S0) with
// exact decays, then Z <- Gamma_e Z in place for the state product.
// mz: the M'_Z tile (K-major, 128 rows x 128 B); zq: d-half 0 of the Z tile (d-half 1 16 KB on).
__device__ __noinline__ void mz_rows_exact(uint8_t *mz, uint8_t *zq, uint32_t taddr, int rho, int ch, int e,
                                          const float *s_gam, const float *s_E) {
    float zk[32];
    tmem_ld32(taddr, zk);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const int i = 32 * ch + c;
        zk[c] = (i <= e) ? zk[c] * exp2f(fminf(s_gam[e < 0 ? 0 : e] - s_gam[i], 0.f)) : 0.f;
    }
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
        *reinterpret_cast<uint4 *>(mz + sw128_off(rho, 4 * ch + c4)) = pack8(zk + 8 * c4);
    const float Ge = e >= 0 ? s_E[e] : 1.f;    // Gamma_e (1 for e = -1)
    uint8_t *zrow = zq + ch * 16384;
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
        float f[8];
        unpack8(*reinterpret_cast<const uint4 *>(zrow + sw128_off(rho, c8)), f);
#pragma unroll
        for (int x = 0; x < 8; ++x) f[x] *= Ge;
        *reinterpret_cast<uint4 *>(zrow + sw128_off(rho, c8)) = pack8(f);
    }
}

}  // namespace
}  // namespace gdn
