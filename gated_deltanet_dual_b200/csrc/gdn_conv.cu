// gdn_conv.cu -- the ShortConv prologue of the dual-stream forward as a pass of its own (sm_100a).
//
// "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes), Method > Key design 3: a
// depthwise causal conv of width 4 on q, k and v (tap 3 is the current token, the same weights for
// both streams); a noisy tap that reaches before its block's start reads the clean raw input, and
// no tap crosses a document start.  This pass writes the convolved q, k, v and their noisy twins
// (fp32 arithmetic, one bf16 rounding, as the chunked kernel's in-place prologue does) into the
// workspace; the chunked kernel then runs without its prologue.  The pass is bound by HBM and runs
// on every SM, where the prologue ran on the few CTAs that carry the documents' state chains.
//
// Work is tiled by document position: a tile is kTile consecutive positions of one document and a
// 256-channel slice of each of q, k, v.  The block stages into shared memory (cp.async, so the bytes
// in flight hold no registers) the clean rows at positions [a - 3, a + kTile) and, one view at a
// time, the noisy rows at the same positions; every tap of every output row of the tile is then a
// window row, clean or noisy: a noisy tap that reaches before its block's start lands on the clean
// window row of the same position.  So each raw row leaves HBM once (the 3-row halo is the
// neighbouring tile's, from L2), and each convolved row is written once.  A warp computes two rows
// of the tile per stream, a lane 8 channels (16-byte shared reads, conflict-free; 16-byte global
// stores, 512 contiguous bytes per warp).  Consecutive blocks take consecutive tiles of one slice,
// so a block restages its weights only when its slice changes.
#include <algorithm>
#include <cstring>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kTaps = 4;
constexpr int kPassThreads = 256;               // 8 warps
constexpr int kPassWarps = kPassThreads / 32;
constexpr int kTile = 16;                       // document positions per tile (two per warp)
constexpr int kWin = kTile + kTaps - 1;         // window rows: 3 halo rows, then the tile
constexpr int kSliceGroups = 32;                // 8-channel groups per slice: one per lane
constexpr size_t kWinBytes = (size_t)kWin * 3 * kSliceGroups * 16;
constexpr size_t kWeightBytes = (size_t)3 * kTaps * 2 * kSliceGroups * 16;
constexpr size_t kPassSmem = kWeightBytes + 2 * kWinBytes;

struct ConvPassParams {
    const __nv_bfloat16 *x[3], *xn[3];     // raw clean [T, H, d] and noisy [V, T_R, H, d]
    __nv_bfloat16 *y[3], *yn[3];           // convolved (disjoint from the raw inputs)
    const float *w;                        // [3, H d, 4]
    WorkspaceHeader *ws;                   // status words (range-checking build)
    int64_t T, TR;
    int32_t N, H, d, V, B;
    int32_t doc_start[kMaxDocs + 1];
    int32_t doc_prompt[kMaxDocs];
    int32_t resp_off[kMaxDocs + 1];
    int32_t tile_off[kMaxDocs + 1];        // first tile of each document (kTile positions a tile)
    int32_t slices;                        // 256-channel slices per row
};

// the last n with starts[n] <= p < starts[n + 1] (empty documents skipped)
__device__ __forceinline__ int doc_index(const int32_t *starts, int N, int64_t p) {
    int lo = 0, hi = N;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (starts[mid] <= p) lo = mid;
        else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ void unpack_bf16x8(uint4 u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float *f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// one output row: four taps from window rows k, k-1, k-2, k-3 (clean or noisy as `noisy_tap` says)
__device__ __forceinline__ void conv_row(const uint4 (*cw)[3][kSliceGroups], const uint4 (*nw)[3][kSliceGroups],
                                         const float4 (*w_s)[kTaps][2][kSliceGroups], int lane, int k,
                                         const int *tap_kind, __nv_bfloat16 *const *dst) {
#pragma unroll
    for (int X = 0; X < 3; ++X) {
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
        for (int j = 0; j < kTaps; ++j) {
            if (tap_kind[j] < 0) continue;
            float f[8];
            unpack_bf16x8(tap_kind[j] ? nw[k - j][X][lane] : cw[k - j][X][lane], f);
            const float4 wa = w_s[X][kTaps - 1 - j][0][lane], wb = w_s[X][kTaps - 1 - j][1][lane];
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = fmaf(wv[c], f[c], acc[c]);
        }
        *reinterpret_cast<uint4 *>(dst[X]) = pack_bf16x8(acc);   // dst checked by the caller
    }
}

__global__ void __launch_bounds__(kPassThreads) conv_pass_kernel(const __grid_constant__ ConvPassParams P) {
    extern __shared__ __align__(16) uint8_t smem[];
    // weights of the slice's 32 groups: [X][weight tap][channel half][lane] x 4 channels
    auto w_s = reinterpret_cast<float4 (*)[kTaps][2][kSliceGroups]>(smem);
    auto cw = reinterpret_cast<uint4 (*)[3][kSliceGroups]>(smem + kWeightBytes);              // clean window
    auto nw = reinterpret_cast<uint4 (*)[3][kSliceGroups]>(smem + kWeightBytes + kWinBytes);  // noisy window
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g8 = P.H * P.d / 8;
    const int64_t hd = (int64_t)P.H * P.d;
    const int64_t tiles = P.tile_off[P.N];
    const int64_t items = tiles * P.slices;
    int cur_slice = -1;
    for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
        const int slice = (int)(item / tiles);
        const int64_t g = item - (int64_t)slice * tiles;
        const int grp = slice * kSliceGroups + lane;
        const bool lane_on = grp < g8;
        const int64_t col = (int64_t)grp * 8;           // first channel (h d + c) of this lane
        if (slice != cur_slice) {
            __syncthreads();                             // the previous tile is done with w_s
            for (int idx = threadIdx.x; idx < 3 * kTaps * 2 * kSliceGroups; idx += kPassThreads) {
                const int ln = idx & 31, half = (idx >> 5) & 1, t = (idx >> 6) & 3, X = idx >> 8;
                const int gg = slice * kSliceGroups + ln;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (gg < g8) {
                    const float *w = P.w + ((int64_t)X * hd + gg * 8 + half * 4) * kTaps + t;
                    v = make_float4(w[0], w[kTaps], w[2 * kTaps], w[3 * kTaps]);
                }
                w_s[X][t][half][ln] = v;
            }
            cur_slice = slice;
        }
        const int n = doc_index(P.tile_off, P.N, g);
        const int a = (int)(g - P.tile_off[n]) * kTile;          // first document position of the tile
        const int64_t s = P.doc_start[n];
        const int len = P.doc_start[n + 1] - P.doc_start[n];
        const int prompt = P.doc_prompt[n];
        const int L = len - prompt;                               // response length
        const int i0 = a - prompt;                                // response index of position a
        const int nlo = i0 > 0 ? i0 : 0, nhi = i0 + kTile < L ? i0 + kTile : L;
        // clean window: row k holds position a - 3 + k
        for (int t = warp; t < kWin * 3; t += kPassWarps) {
            const int k = t / 3, X = t - 3 * (t / 3), pos = a - (kTaps - 1) + k;
            if (lane_on && pos >= 0 && pos < len && GDN_IN_RANGE(P.ws, s + pos < P.T, 301))
                cp_async16(&cw[k][X][lane], P.x[X] + (s + pos) * hd + col);
        }
        for (int vw = 0; vw < P.V && nlo < nhi; ++vw) {
            if (vw > 0) __syncthreads();                          // view vw-1 is done with nw
            const int64_t vbase = (int64_t)vw * P.TR + P.resp_off[n];
            // noisy window: row k holds response index i0 - 3 + k
            for (int t = warp; t < kWin * 3; t += kPassWarps) {
                const int k = t / 3, X = t - 3 * (t / 3), i = i0 - (kTaps - 1) + k;
                if (lane_on && i >= 0 && i < L && GDN_IN_RANGE(P.ws, vbase + i < (int64_t)P.V * P.TR, 302))
                    cp_async16(&nw[k][X][lane], P.xn[X] + (vbase + i) * hd + col);
            }
            cp_async_commit();
            cp_async_wait_all();
            __syncthreads();
            if (lane_on) {
                if (vw == 0) {
                    for (int r = warp; r < kTile && a + r < len; r += kPassWarps) {
                        int kind[kTaps];
#pragma unroll
                        for (int j = 0; j < kTaps; ++j) kind[j] = a + r - j >= 0 ? 0 : -1;
                        __nv_bfloat16 *dst[3];
#pragma unroll
                        for (int X = 0; X < 3; ++X) dst[X] = P.y[X] + (s + a + r) * hd + col;
                        if (GDN_IN_RANGE(P.ws, s + a + r < P.T, 303)) conv_row(cw, nw, w_s, lane, r + kTaps - 1, kind, dst);
                    }
                }
                for (int r = warp; r < kTile; r += kPassWarps) {
                    const int i = i0 + r;
                    if (i < nlo || i >= nhi) continue;
                    const int bs = (i / P.B) * P.B;
                    int kind[kTaps];
#pragma unroll
                    for (int j = 0; j < kTaps; ++j) kind[j] = i - j >= bs ? 1 : (prompt + i - j >= 0 ? 0 : -1);
                    __nv_bfloat16 *dst[3];
#pragma unroll
                    for (int X = 0; X < 3; ++X) dst[X] = P.yn[X] + (vbase + i) * hd + col;
                    if (GDN_IN_RANGE(P.ws, vbase + i < (int64_t)P.V * P.TR, 304)) conv_row(cw, nw, w_s, lane, r + kTaps - 1, kind, dst);
                }
            }
        }
        if (nlo >= nhi || P.V == 0) {                             // a tile with clean rows only
            cp_async_commit();
            cp_async_wait_all();
            __syncthreads();
            if (lane_on)
                for (int r = warp; r < kTile && a + r < len; r += kPassWarps) {
                    int kind[kTaps];
#pragma unroll
                    for (int j = 0; j < kTaps; ++j) kind[j] = a + r - j >= 0 ? 0 : -1;
                    __nv_bfloat16 *dst[3];
#pragma unroll
                    for (int X = 0; X < 3; ++X) dst[X] = P.y[X] + (s + a + r) * hd + col;
                    if (GDN_IN_RANGE(P.ws, s + a + r < P.T, 303)) conv_row(cw, nw, w_s, lane, r + kTaps - 1, kind, dst);
                }
        }
        __syncthreads();                                          // windows free for the next tile
    }
}

}  // namespace

size_t conv_pass_bytes(int64_t T, int64_t TR, int H, int d, int V) {
    const size_t clean = (size_t)T * H * d * 2, noisy = (size_t)V * TR * H * d * 2;
    return ((3 * (clean + noisy) + 255) / 256) * 256;
}

cudaError_t launch_conv_pass(const Params &p, void *buf, cudaStream_t stream) {
    ConvPassParams C;
    std::memset(&C, 0, sizeof(C));
    const int64_t clean = p.T * p.H * p.dk, noisy = (int64_t)p.V * p.TR * p.H * p.dk;
    __nv_bfloat16 *b = static_cast<__nv_bfloat16 *>(buf);
    const void *xs[3] = {p.q, p.k, p.v}, *xns[3] = {p.qn, p.kn, p.vn};
    for (int X = 0; X < 3; ++X) {
        C.x[X] = static_cast<const __nv_bfloat16 *>(xs[X]);
        C.xn[X] = static_cast<const __nv_bfloat16 *>(xns[X]);
        C.y[X] = b + X * clean;
        C.yn[X] = b + 3 * clean + X * noisy;
    }
    C.w = p.conv_w;
    C.ws = p.ws;
    C.T = p.T; C.TR = p.TR; C.N = p.N; C.H = p.H; C.d = p.dk; C.V = p.V; C.B = p.B;
    std::memcpy(C.doc_start, p.doc_start, sizeof(C.doc_start));
    std::memcpy(C.doc_prompt, p.doc_prompt, sizeof(C.doc_prompt));
    std::memcpy(C.resp_off, p.resp_off, sizeof(C.resp_off));
    const int g8 = p.H * p.dk / 8;
    int64_t tiles = 0;
    for (int n = 0; n < p.N; ++n) {
        C.tile_off[n] = (int32_t)tiles;
        tiles += (p.doc_start[n + 1] - p.doc_start[n] + kTile - 1) / kTile;
    }
    C.tile_off[p.N] = (int32_t)tiles;
    C.slices = (g8 + kSliceGroups - 1) / kSliceGroups;
    if (tiles == 0 || g8 == 0) return cudaSuccess;
    static int per_sm = 0;                                 // resident blocks per SM, asked once
    if (per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(conv_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPassSmem);
        if (e != cudaSuccess) return e;
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, conv_pass_kernel, kPassThreads, kPassSmem) != cudaSuccess ||
            nb < 1)
            nb = 1;
        per_sm = nb;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = std::min<int64_t>((int64_t)sms * per_sm, tiles * C.slices);
    conv_pass_kernel<<<(unsigned)grid, kPassThreads, kPassSmem, stream>>>(C);
    return cudaGetLastError();
}

}  // namespace gdn
