/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the dual-stream Gated
 * DeltaNet forward.  TEST INFRASTRUCTURE ONLY: it is used by the tests, by the
 * smoke check and by the benchmark's CPU-baseline leg.  The product path never
 * links or calls it, and it shares no code with the CUDA library.
 *
 * What it computes, token by token, exactly as the method is stated in
 * "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes):
 *
 *  - Method > Key design 2 (hybrid-attention state scheduling):
 *      clean causal stream  S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 *                           o_t = S_t^T q_t / sqrt(d_k)          (read after the update at t)
 *      noisy stream         for response block b: S~ := S_{e(b-1)} (the clean state just before
 *                           the block), the same update over the block's B noisy tokens, then
 *                           every position of the block reads the block-END state:
 *                           o~_l = S~_{e(b)}^T q~_l / sqrt(d_k).
 *  - Method > Key design 3 (ShortConv anti-leak, document packing):
 *      optional width-W depthwise causal convolution on q, k, v; a noisy tap that reaches
 *      before the block start reads the CLEAN raw input; no tap crosses a document start;
 *      the state restarts from zero at every document, so a packed run equals separate runs.
 *  - Method > Overall framework: the prompt is causal context only; the response is cut
 *    into blocks of B tokens; each block has two complementary noisy views (V views here).
 *
 * Readings where the notes leave a step open (each listed in the design notes):
 *  - S is d_k x d_v, alpha_t = exp(g_t), the erase term is decayed by alpha as written.
 *  - Conv: x'_p = sum_{j=0}^{W-1} w[c][W-1-j] * x_{p-j}; no bias, no activation, no
 *    re-normalisation; same weights for both streams; taps before the document start are 0.
 *  - Noisy tensors are packed over response tokens only (docs in order).
 *
 * All arithmetic is IEEE fp64.  Inputs arrive already rounded to the I/O dtype and widened.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NOMEM 2

/* Depthwise causal conv of one channel series for the clean stream.
 * x[p] for p in [0, len) of one document; taps before the document start read 0. */
static double conv_clean_tap(const double *w, int W, const double *x_doc, long stride, int p)
{
    double acc = 0.0;
    for (int j = 0; j < W; ++j) {
        int src = p - j;
        if (src < 0) continue;
        acc += w[W - 1 - j] * x_doc[(long)src * stride];
    }
    return acc;
}

/* Noisy conv tap at document-local position p inside the block starting at blk_start:
 * tap src >= blk_start reads the noisy input, 0 <= src < blk_start reads the clean raw
 * input, src < 0 (before the document) reads 0 (Key design 3, anti-leak rule). */
static double conv_noisy_tap(const double *w, int W, const double *x_doc, long stride,
                             const double *xn_resp, long nstride, int resp_start,
                             int blk_start, int p)
{
    double acc = 0.0;
    for (int j = 0; j < W; ++j) {
        int src = p - j;
        double val;
        if (src >= blk_start)
            val = xn_resp[(long)(src - resp_start) * nstride];
        else if (src >= 0)
            val = x_doc[(long)src * stride];
        else
            val = 0.0;
        acc += w[W - 1 - j] * val;
    }
    return acc;
}

/* One step of the gated delta rule on a dk x dv state (row-major S[i*dv + j]):
 *   u = S^T k ;  S <- alpha * (S - beta * k u^T) + beta * k v^T
 * i.e. S <- alpha (I - beta k k^T) S + beta k v^T. */
static void delta_step(double *S, double *u, int dk, int dv,
                       const double *k, const double *v, double alpha, double beta)
{
    for (int j = 0; j < dv; ++j) u[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double ki = k[i];
        const double *row = S + (long)i * dv;
        for (int j = 0; j < dv; ++j) u[j] += ki * row[j];
    }
    for (int i = 0; i < dk; ++i) {
        const double ki = k[i];
        double *row = S + (long)i * dv;
        for (int j = 0; j < dv; ++j)
            row[j] = alpha * (row[j] - beta * ki * u[j]) + beta * ki * v[j];
    }
}

/* o = S^T q / sqrt(dk) */
static void readout(const double *S, int dk, int dv, const double *q, double *o)
{
    const double scale = 1.0 / sqrt((double)dk);
    for (int j = 0; j < dv; ++j) o[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double qi = q[i];
        const double *row = S + (long)i * dv;
        for (int j = 0; j < dv; ++j) o[j] += qi * row[j];
    }
    for (int j = 0; j < dv; ++j) o[j] *= scale;
}

/*
 * Full forward.  Shapes (row-major):
 *   q,k [T,H,dk]  v [T,H,dv]  g,beta [T,H]
 *   qn,kn [V,TR,H,dk]  vn [V,TR,H,dv]  gn,betan [V,TR,H]
 *   conv_w: q weights [H*dk][W], then k weights [H*dk][W], then v weights [H*dv][W]
 *           (NULL or conv_width == 0: no conv)
 *   out [T,H,dv]  out_noisy [V,TR,H,dv]  final_state [N,H,dk,dv]
 *   noisy_state (optional, may be NULL) [V, TR/B, H, dk, dv]: block-end noisy states,
 *           blocks numbered over the packed response rows.
 * Returns 0, or a nonzero code for inconsistent metadata.
 */
int gdn_oracle_forward(int N, int H, int dk, int dv, int V, int B, int conv_width,
                       const int32_t *doc_offsets, const int32_t *prompt_len,
                       const double *q, const double *k, const double *v,
                       const double *g, const double *beta,
                       const double *qn, const double *kn, const double *vn,
                       const double *gn, const double *betan,
                       const double *conv_w,
                       double *out, double *out_noisy, double *final_state,
                       double *noisy_state, int num_threads)
{
    if (N < 1 || H < 1 || dk < 1 || dv < 1 || V < 0 || B < 1 || conv_width < 0) return ORACLE_BAD_ARG;
    if (conv_width > 0 && conv_w == NULL) return ORACLE_BAD_ARG;
    long *resp_off = (long *)malloc(sizeof(long) * (N + 1));
    if (!resp_off) return ORACLE_NOMEM;
    resp_off[0] = 0;
    for (int n = 0; n < N; ++n) {
        int len = doc_offsets[n + 1] - doc_offsets[n];
        int P = prompt_len[n];
        if (len < 0 || P < 0 || P > len || (len - P) % B != 0) { free(resp_off); return ORACLE_BAD_ARG; }
        resp_off[n + 1] = resp_off[n] + (len - P);
    }
    const long T = doc_offsets[N];
    const long TR = resp_off[N];
    const int W = conv_width;
    const long sq = (long)H * dk, sv = (long)H * dv; /* token strides */
    int status = ORACLE_OK;

#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
    for (long unit = 0; unit < (long)N * H; ++unit) {
        const int n = (int)(unit / H), h = (int)(unit % H);
        const int s0 = doc_offsets[n];
        const int len = doc_offsets[n + 1] - s0;
        const int P = prompt_len[n];
        const int R = len - P;
        const long rbase = resp_off[n];

        double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
        double *St = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        double *qc = (double *)malloc(sizeof(double) * (size_t)dk);
        double *kc = (double *)malloc(sizeof(double) * (size_t)dk);
        double *vc = (double *)malloc(sizeof(double) * (size_t)dv);
        /* conv'd noisy rows of one block for one view: [B][dk|dv] */
        double *qb = (double *)malloc(sizeof(double) * (size_t)B * dk);
        double *kb = (double *)malloc(sizeof(double) * (size_t)B * dk);
        double *vb = (double *)malloc(sizeof(double) * (size_t)B * dv);
        if (!S || !St || !u || !qc || !kc || !vc || !qb || !kb || !vb) {
#pragma omp atomic write
            status = ORACLE_NOMEM;
            free(S); free(St); free(u); free(qc); free(kc); free(vc); free(qb); free(kb); free(vb);
            continue;
        }
        /* document-local base pointers for head h */
        const double *qd = q + (long)s0 * sq + (long)h * dk;
        const double *kd = k + (long)s0 * sq + (long)h * dk;
        const double *vd = v + (long)s0 * sv + (long)h * dv;
        const double *wq = W ? conv_w + (long)h * dk * W : NULL;
        const double *wk = W ? conv_w + (long)H * dk * W + (long)h * dk * W : NULL;
        const double *wv = W ? conv_w + 2L * H * dk * W + (long)h * dv * W : NULL;

        for (int p = 0; p < len; ++p) {
            /* --- noisy stream: block b starts here; S currently holds S_{e(b-1)} --- */
            if (p >= P && (p - P) % B == 0 && V > 0) {
                const int blk_start = p;               /* document-local */
                const int b0 = p - P;                  /* response-local row of the block start */
                for (int view = 0; view < V; ++view) {
                    const double *qnv = qn + ((long)view * TR + rbase) * sq + (long)h * dk;
                    const double *knv = kn + ((long)view * TR + rbase) * sq + (long)h * dk;
                    const double *vnv = vn + ((long)view * TR + rbase) * sv + (long)h * dv;
                    const double *gnv = gn + ((long)view * TR + rbase) * H + h;
                    const double *bnv = betan + ((long)view * TR + rbase) * H + h;
                    /* noisy rows of this block (conv applied with the anti-leak rule) */
                    for (int l = 0; l < B; ++l) {
                        const int pl = blk_start + l;
                        for (int i = 0; i < dk; ++i) {
                            if (W) {
                                qb[l * dk + i] = conv_noisy_tap(wq + (long)i * W, W, qd + i, sq, qnv + i, sq, P, blk_start, pl);
                                kb[l * dk + i] = conv_noisy_tap(wk + (long)i * W, W, kd + i, sq, knv + i, sq, P, blk_start, pl);
                            } else {
                                qb[l * dk + i] = qnv[(long)(b0 + l) * sq + i];
                                kb[l * dk + i] = knv[(long)(b0 + l) * sq + i];
                            }
                        }
                        for (int j = 0; j < dv; ++j) {
                            if (W)
                                vb[l * dv + j] = conv_noisy_tap(wv + (long)j * W, W, vd + j, sv, vnv + j, sv, P, blk_start, pl);
                            else
                                vb[l * dv + j] = vnv[(long)(b0 + l) * sv + j];
                        }
                    }
                    /* S~ := S_{e(b-1)}, then B steps of the same rule */
                    memcpy(St, S, sizeof(double) * (size_t)dk * dv);
                    for (int l = 0; l < B; ++l) {
                        const long r = b0 + l;
                        delta_step(St, u, dk, dv, kb + (long)l * dk, vb + (long)l * dv,
                                   exp(gnv[r * H]), bnv[r * H]);
                    }
                    /* every position of the block reads the block-end state */
                    for (int l = 0; l < B; ++l) {
                        const long row = (long)view * TR + rbase + b0 + l;
                        readout(St, dk, dv, qb + (long)l * dk, out_noisy + row * sv + (long)h * dv);
                    }
                    if (noisy_state) {
                        const long blk = (rbase + b0) / B;
                        double *dst = noisy_state + (((long)view * (TR / B) + blk) * H + h) * (long)dk * dv;
                        memcpy(dst, St, sizeof(double) * (size_t)dk * dv);
                    }
                }
            }
            /* --- clean causal stream, token p --- */
            for (int i = 0; i < dk; ++i) {
                qc[i] = W ? conv_clean_tap(wq + (long)i * W, W, qd + i, sq, p) : qd[(long)p * sq + i];
                kc[i] = W ? conv_clean_tap(wk + (long)i * W, W, kd + i, sq, p) : kd[(long)p * sq + i];
            }
            for (int j = 0; j < dv; ++j)
                vc[j] = W ? conv_clean_tap(wv + (long)j * W, W, vd + j, sv, p) : vd[(long)p * sv + j];
            const long tok = (long)s0 + p;
            delta_step(S, u, dk, dv, kc, vc, exp(g[tok * H + h]), beta[tok * H + h]);
            readout(S, dk, dv, qc, out + tok * sv + (long)h * dv);
        }
        (void)R;
        memcpy(final_state + ((long)n * H + h) * (long)dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(St); free(u); free(qc); free(kc); free(vc); free(qb); free(kb); free(vb);
    }
    free(resp_off);
    (void)T;
    return status;
}

/*
 * Decode-side steps (the serving paragraph of the same notes: Diffusion-Trust commits a finished
 * block with one causal replay that writes its final state into the state pool; AR-Trust's
 * verify forward runs the clean stream over the K candidate tokens and keeps every step's state
 * so that accepting the first r candidates is a gather of state r).  Per sequence n and head h:
 *   S := S0[n, h];  for t = 0..L-1:  S <- alpha_t (I - beta_t k_t k_t^T) S + beta_t k_t v_t^T,
 *                                     o_t = S^T q_t / sqrt(dk),  states[n, t, h] = S (optional);
 *   S_final[n, h] := S.
 * Shapes: S0, S_final [Nseq, H, dk, dv]; q,k [Nseq, L, H, dk]; v [Nseq, L, H, dv];
 *         g, beta [Nseq, L, H]; out [Nseq, L, H, dv]; states (may be NULL) [Nseq, L, H, dk, dv].
 */
int gdn_oracle_decode_steps(int Nseq, int H, int L, int dk, int dv,
                            const double *S0, const double *q, const double *k, const double *v,
                            const double *g, const double *beta,
                            double *out, double *S_final, double *states, int num_threads)
{
    if (Nseq < 0 || H < 1 || L < 0 || dk < 1 || dv < 1) return ORACLE_BAD_ARG;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
    int status = ORACLE_OK;
    const long units = (long)Nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long unit = 0; unit < units; ++unit) {
        const long n = unit / H, h = unit % H;
        const long sz = (long)dk * dv;
        double *S = (double *)malloc(sizeof(double) * (size_t)sz);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!S || !u) {
            free(S); free(u);
#pragma omp atomic write
            status = ORACLE_NOMEM;
            continue;
        }
        memcpy(S, S0 + unit * sz, sizeof(double) * (size_t)sz);
        for (int t = 0; t < L; ++t) {
            const long row = (n * L + t) * H + h;          /* (n, t, h) */
            delta_step(S, u, dk, dv, k + row * dk, v + row * dv, exp(g[row]), beta[row]);
            readout(S, dk, dv, q + row * dk, out + row * dv);
            if (states) memcpy(states + row * sz, S, sizeof(double) * (size_t)sz);
        }
        memcpy(S_final + unit * sz, S, sizeof(double) * (size_t)sz);
        free(S); free(u);
    }
    return status;
}

/* Threads the oracle would use (for reporting). */
int gdn_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
