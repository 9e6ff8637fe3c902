// gdn_attention.cu -- dual-stream softmax attention with the document-blocked causal /
// block-bidirectional mask ("FLARE: Diffusion for Hybrid Language Model", papernotes.org notes,
// Method > Overall framework and Key design 1) on sm_100a, and its C ABI (gdn_attention.h).
//
// One CTA = one (128-row query tile, query head).  The tile's key tiles are 128 clean keys of its
// document each and, for a noisy query tile, one more: the tile's own 128 noisy rows of the same
// view under a block-diagonal mask (B divides 128, so no block straddles a tile).  Per key tile:
//   S = Q K^T           tcgen05, bf16 operands from 128B-swizzled TMA tiles, fp32 in TMEM
//   softmax             thread t owns query row t (TMEM lane t): masked row max, then
//                       P = 2^(s - m) with s = S log2(e) / sqrt(d), written as bf16 pairs over
//                       S's first 64 TMEM columns (the A operand of the next MMA), row sum l
//   O += P V            tcgen05 with A in TMEM, O accumulated in TMEM
// The running max m is a reference that moves only when a tile's max exceeds it by more than
// 8 (log2 units): then O and l are rescaled by 2^(m_old - m_new); otherwise P may reach 2^8,
// harmless in fp32 and bf16.  The output is O / l, rounded once to bf16.
//
// 128 threads, 96 KB of shared memory (Q, K, V tiles) and 256 TMEM columns per CTA, so two CTAs
// share an SM and one's softmax overlaps the other's MMAs.  K of the next key tile is loaded as
// soon as S is computed, V as soon as P V is.  Each CTA derives its (document, head, query tile)
// from its index and per-document prefix tables in the parameter block: documents longest first,
// then heads, then the document's query tiles, so the CTAs that run together read the same key /
// value tiles through L2.  Every mbarrier wait is bounded; a wait that gives up records
// GDN_ERR_TIMEOUT in the workspace and the CTA leaves its loop.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_internal.cuh"
#include "sm100.cuh"
#include "../../include/gdn_attention.h"

namespace gdn {
namespace {

using namespace sm100;

constexpr int AD = 128;                     // head dim
constexpr int AT = 128;                     // query rows / keys per tile
constexpr int kAThreads = 128;              // thread t owns query row t
constexpr uint32_t kAWaitIters = 1u << 24;   // bound of an ordinary wait (the test entry point lowers it)
constexpr int A_OFF_Q = 0, A_OFF_K = 32768, A_OFF_V = 65536;   // [2 d-halves][128 rows][128 B] each
constexpr int A_SMEM = 3 * 32768 + 1024;
constexpr uint32_t TA_S = 0;                // S (fp32, 128 columns); P (bf16 pairs) over its first 64
constexpr uint32_t TA_O = 128;              // O accumulator (fp32, 128 columns)
constexpr float kRescaleLog2 = 8.f;         // move the reference max only past this margin

struct AttnParams {
    int32_t H, Hkv, V, B;
    int64_t TR;
    float scale_log2;                       // log2(e) / sqrt(d)
    uint32_t wait_iters;                    // test instantiation: bound of the mbarrier waits, in polls
    WorkspaceHeader *ws;
    void *out, *out_noisy;
    int32_t N;
    int32_t doc_start[kMaxDocs + 1];
    int32_t doc_prompt[kMaxDocs];
    int32_t resp_off[kMaxDocs + 1];
    int32_t doc_order[kMaxDocs];            // documents, longest first
    int32_t item_off[kMaxDocs + 1];         // first CTA of each document in that order
};

struct AttnMaps {
    CUtensorMap q, k, v, qn, kn, vn;
};

// 2^x by the hardware approximation (ex2.approx.ftz: relative error ~2^-22, 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// TW: the test instantiation, whose waits poll with the caller's bound (gdn_attn_forward_test_wait_limit).
template <bool TW>
__global__ void __launch_bounds__(kAThreads, 2)
gdn_attention_kernel(const __grid_constant__ AttnParams P, const __grid_constant__ AttnMaps M) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_q, bar_k, bar_v, bar_s, bar_o;
    __shared__ uint64_t bar_drain;          // error path: every MMA thread 0 issued has completed
    __shared__ uint32_t s_kflag, s_vflag;   // error path: thread 0's waits of the last tile (see below)
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5;
    // Work item of this CTA: documents longest first; per document, every head in turn; per
    // (document, head) every query tile, clean tiles from the last, then each view's noisy tiles
    // from the last.  The CTAs that run together thus share the (document, head)'s key/value tiles.
    int lo_k = 0, hi_k = P.N;                          // largest k with item_off[k] <= blockIdx.x
    while (hi_k - lo_k > 1) {
        const int mid = (lo_k + hi_k) >> 1;
        if (P.item_off[mid] <= (int)blockIdx.x) lo_k = mid;
        else hi_k = mid;
    }
    const int n = P.doc_order[lo_k];
    const int s = P.doc_start[n], len = P.doc_start[n + 1] - s, Pn = P.doc_prompt[n], R = len - Pn;
    const int nct = (len + AT - 1) / AT, nnt = (R + AT - 1) / AT;
    const int ntile = nct + P.V * nnt;
    const int local = (int)blockIdx.x - P.item_off[lo_k];
    const int h = local / ntile, jt = local % ntile;
    int kind, tile;
    if (jt < nct) {
        kind = 0;
        tile = nct - 1 - jt;
    } else {
        kind = 1 + (jt - nct) / nnt;
        tile = nnt - 1 - (jt - nct) % nnt;
    }
    const int hk = h / (P.H / P.Hkv);
    const int B = P.B;
    const int w = kind - 1;                                   // noisy view (kind > 0)
    const int64_t nrow0 = (int64_t)w * P.TR + P.resp_off[n] + (int64_t)AT * tile;   // noisy tile rows
    int nkc, qrow0;
    if (kind == 0) {
        qrow0 = s + AT * tile;
        nkc = tile + 1;
    } else {
        qrow0 = (int)nrow0;
        const int ilast = min(AT * tile + AT - 1, R - 1);
        nkc = (Pn + (ilast / B) * B + AT - 1) / AT;
    }
    const int nk = nkc + (kind ? 1 : 0);

    if (tid == 0) {
        mbar_init(&bar_q, 1);
        mbar_init(&bar_k, 1);
        mbar_init(&bar_v, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_o, 1);
        mbar_init(&bar_drain, 1);
        s_kflag = s_vflag = 0u;
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
    // Error path (as in the chunked kernel): a wait that gives up records its site, and the CTA
    // leaves the key loop at the next uniform barrier, before another key tile starts.  Thread 0,
    // which issues every TMA load and MMA, decides each issue on the waits of the same tile: it
    // refills a buffer only after seeing its last load arrive and the MMA that read it complete,
    // so no mbarrier ever has two phases outstanding.  It leaves the outcome of its waits of the
    // current tile in shared memory (s_kflag after the S half, s_vflag after the PV half, each
    // tagged with the tile); when the CTA stops, it works out from them which load may still be
    // arriving on each mbarrier, waits for those and, through one more commit, for its MMAs
    // before the CTA frees tensor memory.  (Counting the issued loads in registers instead, or
    // bookkeeping inside the loop's exits, cost about 5 % of the kernel's time.)
    auto wait_ok = [&](uint64_t *bar, uint32_t parity, int where) {
        const bool ok = kwait<TW>(bar, parity, kAWaitIters, P.wait_iters);
        if (!ok) fail(where);
        return ok;
    };
    // key tile j: clean keys [s + 128 j, +128) or (j == nkc) the tile's own noisy rows
    auto issue_tile = [&](uint8_t *dst, const CUtensorMap *clean, const CUtensorMap *noisy, uint64_t *bar, int j) {
        const CUtensorMap *map = j < nkc ? clean : noisy;
        const int row0 = j < nkc ? s + AT * j : (int)nrow0;
        mbar_arrive_expect_tx(bar, 32768u);
        for (int hf = 0; hf < 2; ++hf)
            for (int rh = 0; rh < 2; ++rh)
                tma_load_3d(dst + hf * 16384 + rh * 8192, map, bar, hf * 64, hk, row0 + 64 * rh);
    };
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_q, 32768u);
        const CUtensorMap *qm = kind == 0 ? &M.q : &M.qn;
        for (int hf = 0; hf < 2; ++hf)
            for (int rh = 0; rh < 2; ++rh)
                tma_load_3d(sm + A_OFF_Q + hf * 16384 + rh * 8192, qm, &bar_q, hf * 64, h, qrow0 + 64 * rh);
        issue_tile(sm + A_OFF_K, &M.k, &M.kn, &bar_k, 0);
        issue_tile(sm + A_OFF_V, &M.v, &M.vn, &bar_v, 0);
    }
    const uint64_t dQ = make_sdesc(smem_u32(sm + A_OFF_Q), 16, 1024);      // K-major A
    const uint64_t dK = make_sdesc(smem_u32(sm + A_OFF_K), 16, 1024);      // K-major B (keys x d)
    const uint64_t dV = make_sdesc(smem_u32(sm + A_OFF_V), 16384, 1024);   // MN-major B (keys x d)
    constexpr uint32_t idesc = make_idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_pv = make_idesc_bf16(128, 128, 0, 1);

    // this thread's query row and its visible key range per key tile
    const int r = tid;
    const int i_resp = AT * tile + r;                         // noisy: response index of the row
    const int b0 = kind ? (i_resp / B) * B : 0;
    float m_ref = -INFINITY, l = 0.f;
    const float sl2 = P.scale_log2;
    bool stop = false;        // uniform over the CTA: leave the key loop (a wait gave up)

    int j = 0;
    for (; j < nk; ++j) {
        // ---- S = Q K_j^T
        bool q_ok = true, k_ok = true;    // thread 0: Q and K_j arrived
        if (tid == 0) {
            q_ok = j > 0 || wait_ok(&bar_q, 0, 1);
            k_ok = wait_ok(&bar_k, j & 1, 2) && q_ok;
            if (k_ok) {
                tc_fence_after();
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tb + TA_S, dQ + (off >> 4), dK + (off >> 4), idesc, kk > 0);
                }
                mma_commit(&bar_s);
            }
        }
        __syncwarp();
        const bool s_ok = wait_ok(&bar_s, j & 1, 3);
        __syncwarp();
        tc_fence_after();
        if (tid == 0) {
            const bool kn = k_ok && s_ok && j + 1 < nk;                // K_{j+1} goes out
            if (kn) issue_tile(sm + A_OFF_K, &M.k, &M.kn, &bar_k, j + 1);
            // bit 0 Q missing, bit 1 K_{j+1} issued, bit 2 K_j missing; tile j + 1 above bit 8
            s_kflag = (q_ok ? 0u : 1u) | (kn ? 2u : 0u) | (k_ok ? 0u : 4u) | ((uint32_t)(j + 1) << 8);
        }
        // visible columns of this row in tile j: [lo, hi)
        int lo = 0, hi;
        if (j < nkc) hi = kind == 0 ? AT * (tile - j) + r + 1 : Pn + b0 - AT * j;
        else {
            lo = b0 - AT * tile;
            hi = min(lo + B, R - AT * tile);
        }
        // ---- the row of S (one tensor-memory read), masked row max in log2 units
        float x[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem_addr(tb, warp * 32, TA_S + 32 * c), x[c]);
        tmem_wait_ld();
        const bool full = lo <= 0 && hi >= AT;                  // every key of the tile visible
        float mt = -INFINITY;
        if (full) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) mt = fmaxf(mt, x[c][e]);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int col = 32 * c + e;
                    x[c][e] = (col >= lo && col < hi) ? x[c][e] : -INFINITY;
                    mt = fmaxf(mt, x[c][e]);
                }
        }
        mt *= sl2;                                              // sl2 > 0; -inf stays -inf
        // ---- reference max: move it (and rescale O, l) only past the margin
        float alpha = 1.f;
        if (mt > m_ref + kRescaleLog2) {
            alpha = m_ref == -INFINITY ? 0.f : ex2_approx(m_ref - mt);
            m_ref = mt;
        }
        const float mu = m_ref == -INFINITY ? 0.f : m_ref;
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {     // O holds earlier tiles: rescale
#pragma unroll 1
            for (int c0 = 0; c0 < AD; c0 += 32) {
                float o[32];
                tmem_ld32(tmem_addr(tb, warp * 32, TA_O + c0), o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] *= alpha;
                tmem_st32(tmem_addr(tb, warp * 32, TA_O + c0), o);
            }
        }
        l *= alpha;
        // ---- P = 2^(s - m) (masked scores are -inf: 0) as bf16 pairs over S columns [0, 64)
        float ls = 0.f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float pk[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float p0 = ex2_approx(fmaf(x[2 * hf + e / 16][(2 * e) % 32], sl2, -mu));
                const float p1 = ex2_approx(fmaf(x[2 * hf + e / 16][(2 * e) % 32 + 1], sl2, -mu));
                ls += p0 + p1;
                pk[e] = __uint_as_float(pack_bf2(p0, p1));
            }
            tmem_st32(tmem_addr(tb, warp * 32, TA_S + 32 * hf), pk);
        }
        l += ls;
        tmem_wait_st();
        tc_fence_before();
        if ((stop = __syncthreads_or(*reinterpret_cast<volatile int *>(&s_abort) != 0))) break;
        // ---- O += P V_j
        bool v_ok = true;                 // thread 0: V_j arrived
        if (tid == 0) {
            tc_fence_after();
            v_ok = wait_ok(&bar_v, j & 1, 4);
            if (v_ok) {
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tb + TA_O, tb + TA_S + kk * 8, dV + ((kk * 2048) >> 4), idesc_pv, (j > 0 || kk > 0));
                mma_commit(&bar_o);
            }
        }
        __syncwarp();
        const bool o_ok = wait_ok(&bar_o, j & 1, 5);
        __syncwarp();
        tc_fence_after();
        if (tid == 0) {
            const bool vn = v_ok && o_ok && j + 1 < nk;               // V_{j+1} goes out
            if (vn) issue_tile(sm + A_OFF_V, &M.v, &M.vn, &bar_v, j + 1);
            // bit 1 V_{j+1} issued, bit 2 V_j missing; tile j + 1 above bit 8
            s_vflag = (vn ? 2u : 0u) | (v_ok ? 0u : 4u) | ((uint32_t)(j + 1) << 8);
        }
        if ((stop = __syncthreads_or(*reinterpret_cast<volatile int *>(&s_abort) != 0))) break;
    }

    // ---- out = O / l
    if (!stop) {
        const bool valid = kind == 0 ? (AT * tile + r < len) : (i_resp < R);
        __nv_bfloat16 *orow = kind == 0
            ? static_cast<__nv_bfloat16 *>(P.out) + ((int64_t)(qrow0 + r) * P.H + h) * AD
            : static_cast<__nv_bfloat16 *>(P.out_noisy) + ((nrow0 + r) * P.H + h) * AD;
        const float inv = 1.f / l;
#pragma unroll 1
        for (int c0 = 0; c0 < AD; c0 += 32) {
            float o[32];
            tmem_ld32(tmem_addr(tb, warp * 32, TA_O + c0), o);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 u;
                    u.x = pack_bf2(o[e] * inv, o[e + 1] * inv);
                    u.y = pack_bf2(o[e + 2] * inv, o[e + 3] * inv);
                    u.z = pack_bf2(o[e + 4] * inv, o[e + 5] * inv);
                    u.w = pack_bf2(o[e + 6] * inv, o[e + 7] * inv);
                    *reinterpret_cast<uint4 *>(orow + c0 + e) = u;
                }
            }
        }
    }
    // Drain (only when the CTA stopped early), with the normal limit: the loads that may still be
    // arriving (a completed phase passes at once), then thread 0's MMAs.
    if (stop && tid == 0) {
        const uint32_t lim = kDrainWaitIters;
        // The loop stopped in tile j.  K: K_{j+1} if it went out, else K_j unless it was seen to
        // arrive.  V: after the PV half of tile j (s_vflag tagged j + 1) the same; before it,
        // V_j went out (before the loop or in tile j - 1) and was not waited for.
        const uint32_t kf = s_kflag, vf = s_vflag;
        if (kf & 1u) mbar_wait(&bar_q, 0, lim);
        if (kf & 6u) mbar_wait(&bar_k, ((kf & 2u) ? j + 1 : j) & 1, lim);
        if ((vf >> 8) != (uint32_t)(j + 1)) mbar_wait(&bar_v, j & 1, lim);
        else if (vf & 6u) mbar_wait(&bar_v, ((vf & 2u) ? j + 1 : j) & 1, lim);
        mma_commit(&bar_drain);
        mbar_wait(&bar_drain, 0, lim);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 256);
}

PFN_cuTensorMapEncodeTiled_v12000 attn_encoder() {
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

// [rows, heads, 128] bf16; box = 64 rows x 1 head x 64 columns, 128B swizzle, zero fill past the end
bool attn_map(CUtensorMap *m, const void *ptr, int heads, int64_t rows) {
    auto enc = attn_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)AD, (cuuint64_t)heads, (cuuint64_t)std::max<int64_t>(rows, 1)};
    cuuint64_t strides[2] = {(cuuint64_t)AD * 2, (cuuint64_t)heads * AD * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool attn_desc_ok(const gdn_attn_desc *d) {
    return d && d->num_docs >= 1 && d->num_heads >= 1 && d->num_kv_heads >= 1 && d->head_dim >= 1 &&
           d->num_views >= 0 && d->block_size >= 1 && (d->dtype == GDN_BF16 || d->dtype == GDN_FP32) &&
           d->reserved == 0;
}

bool attn_desc_supported(const gdn_attn_desc *d) {
    return d->head_dim == AD && d->dtype == GDN_BF16 && AT % d->block_size == 0 && d->num_views <= 2 &&
           d->num_heads % d->num_kv_heads == 0 && d->num_docs <= kMaxDocs;
}

// Layout check: documents from offset 0, non-decreasing, prompts inside them, responses in
// whole blocks.
bool attn_layout(const gdn_attn_desc *d, const int32_t *offs, const int32_t *pl, int64_t *T, int64_t *TR) {
    if (!offs || !pl || offs[0] != 0) return false;
    const int N = d->num_docs, B = d->block_size;
    int64_t tr = 0;
    for (int n = 0; n < N; ++n) {
        const int64_t len = (int64_t)offs[n + 1] - offs[n];
        if (len < 0 || pl[n] < 0 || pl[n] > len || (len - pl[n]) % B != 0) return false;
        tr += len - pl[n];
    }
    if (tr > INT32_MAX || offs[N] > INT32_MAX) return false;
    *T = offs[N];
    *TR = tr;
    return true;
}


}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" size_t gdn_attn_workspace_size(const gdn_attn_desc *desc, const int32_t *doc_offsets_host,
                                          const int32_t *prompt_len_host) {
    if (!attn_desc_ok(desc)) return 0;
    int64_t T = 0, TR = 0;
    if (!attn_layout(desc, doc_offsets_host, prompt_len_host, &T, &TR)) return 0;
    return sizeof(WorkspaceHeader);
}

static gdn_status attn_forward_impl(const gdn_attn_desc *desc, const void *q, const void *k, const void *v,
                                    const void *qn, const void *kn, const void *vn,
                                    const int32_t *doc_offsets, const int32_t *prompt_len,
                                    void *out, void *out_noisy, void *workspace, size_t workspace_bytes,
                                    uint32_t wait_iters, gdn_stream_t stream) {
    if (!attn_desc_ok(desc)) return GDN_ERR_INVALID_ARG;
    int64_t T = 0, TR = 0;
    if (!attn_layout(desc, doc_offsets, prompt_len, &T, &TR)) return GDN_ERR_INVALID_ARG;
    const int V = TR > 0 ? desc->num_views : 0;
    if (T > 0 && (!q || !k || !v || !out)) return GDN_ERR_INVALID_ARG;
    if (V > 0 && (!qn || !kn || !vn || !out_noisy)) return GDN_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < sizeof(WorkspaceHeader)) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, qn, kn, vn, out, out_noisy, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    if (!attn_desc_supported(desc)) return GDN_ERR_UNSUPPORTED;

    AttnParams P;
    std::memset(&P, 0, sizeof(P));
    P.H = desc->num_heads;
    P.Hkv = desc->num_kv_heads;
    P.V = V;
    P.B = desc->block_size;
    P.TR = TR;
    P.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)desc->head_dim));
    P.ws = static_cast<WorkspaceHeader *>(workspace);
    P.wait_iters = wait_iters;
    P.out = out;
    P.out_noisy = out_noisy;
    const int N = desc->num_docs;
    P.N = N;
    int64_t roff = 0;
    for (int n = 0; n <= N; ++n) {
        P.doc_start[n] = doc_offsets[n];
        P.resp_off[n] = (int32_t)roff;
        if (n < N) {
            P.doc_prompt[n] = prompt_len[n];
            roff += (int64_t)doc_offsets[n + 1] - doc_offsets[n] - prompt_len[n];
        }
    }
    // documents longest first; each takes H x (its query tiles) CTAs
    std::vector<int> order(N);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
        return doc_offsets[a + 1] - doc_offsets[a] > doc_offsets[b + 1] - doc_offsets[b];
    });
    int64_t items = 0;
    for (int k = 0; k < N; ++k) {
        const int n = order[k];
        const int64_t len = (int64_t)doc_offsets[n + 1] - doc_offsets[n], R = len - prompt_len[n];
        P.doc_order[k] = n;
        P.item_off[k] = (int32_t)std::min<int64_t>(items, INT32_MAX);
        items += (int64_t)desc->num_heads * ((len + AT - 1) / AT + (int64_t)V * ((R + AT - 1) / AT));
    }
    P.item_off[N] = (int32_t)std::min<int64_t>(items, INT32_MAX);
    if (items > INT32_MAX) return GDN_ERR_UNSUPPORTED;
    if (items == 0) return GDN_OK;
    AttnMaps maps;
    const int H = desc->num_heads, Hkv = desc->num_kv_heads;
    if (!attn_map(&maps.q, q, H, T) || !attn_map(&maps.k, k, Hkv, T) || !attn_map(&maps.v, v, Hkv, T))
        return GDN_ERR_CUDA;
    if (V > 0) {
        if (!attn_map(&maps.qn, qn, H, (int64_t)V * TR) || !attn_map(&maps.kn, kn, Hkv, (int64_t)V * TR) ||
            !attn_map(&maps.vn, vn, Hkv, (int64_t)V * TR))
            return GDN_ERR_CUDA;
    } else {
        maps.qn = maps.q;
        maps.kn = maps.k;
        maps.vn = maps.v;
    }
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(gdn_attention_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, A_SMEM);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(gdn_attention_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, A_SMEM);
    });
    if (attr_err != cudaSuccess) return GDN_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, sizeof(WorkspaceHeader), st) != cudaSuccess) return GDN_ERR_CUDA;
    if (wait_iters < kAWaitIters) gdn_attention_kernel<true><<<(unsigned)items, kAThreads, A_SMEM, st>>>(P, maps);
    else gdn_attention_kernel<false><<<(unsigned)items, kAThreads, A_SMEM, st>>>(P, maps);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" gdn_status gdn_attn_forward(const gdn_attn_desc *desc, const void *q, const void *k, const void *v,
                                       const void *qn, const void *kn, const void *vn,
                                       const int32_t *doc_offsets, const int32_t *prompt_len,
                                       void *out, void *out_noisy, void *workspace, size_t workspace_bytes,
                                       gdn_stream_t stream) {
    return attn_forward_impl(desc, q, k, v, qn, kn, vn, doc_offsets, prompt_len, out, out_noisy, workspace,
                             workspace_bytes, kAWaitIters, stream);
}

extern "C" gdn_status gdn_attn_forward_test_wait_limit(const gdn_attn_desc *desc, const void *q, const void *k,
                                                       const void *v, const void *qn, const void *kn,
                                                       const void *vn, const int32_t *doc_offsets,
                                                       const int32_t *prompt_len, void *out, void *out_noisy,
                                                       void *workspace, size_t workspace_bytes,
                                                       uint32_t wait_iters, gdn_stream_t stream) {
    if (wait_iters < 1) return GDN_ERR_INVALID_ARG;
    return attn_forward_impl(desc, q, k, v, qn, kn, vn, doc_offsets, prompt_len, out, out_noisy, workspace,
                             workspace_bytes, wait_iters, stream);
}
