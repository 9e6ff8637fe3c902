/*
 * gdn_decode.h -- C ABI of the decode-side Gated DeltaNet state kernels (B200, sm_100a).
 *
 * The serving paragraph of "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes)
 * describes two state operations of the GDN layers at inference time, both on the clean
 * recurrence of Method > Key design 2:
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  alpha_t = exp(g_t),
 *     o_t = S_t^T q_t / sqrt(d_k).
 *   - Diffusion-Trust: the denoising forwards of a block never touch the state pool; once the
 *     block is final, one causal replay runs its tokens from the sequence's pooled state and
 *     writes the final state back  ->  gdn_decode_replay.
 *   - AR-Trust: the noisy stream drafts K candidates, the clean stream verifies them in one
 *     forward that also stores the state after every candidate step (Cache); once the first r
 *     candidates are accepted, a gather-scatter copies the state after step r into the pool,
 *     with no recomputation  ->  gdn_decode_verify, then gdn_decode_commit.
 *
 * Layouts (row-major, contiguous, caller-owned device memory):
 *   state_pool   [P, H, d_k, d_v] fp32   pooled states; row `slots[n]` belongs to sequence n
 *   slots        [N] int32 (device)      distinct pool rows, 0 <= slots[n] < P
 *   q, k         [N, L, H, d_k]          dtype = desc->dtype (bf16 or fp32)
 *   v, out       [N, L, H, d_v]
 *   g, beta      [N, L, H] fp32
 *   state_cache  [N, L, H, d_k, d_v] fp32  state after each of the L steps (verify)
 *   accepted     [N] int32 (device)      accepted candidates r, 0 <= r <= L (commit)
 *   device_status  optional device int32 (may be NULL): cleared on `stream` at the start of each
 *                  call; set to GDN_ERR_INVALID_ARG by a kernel that meets a slot or accepted
 *                  count out of range (that sequence is then left untouched).
 *
 * All calls validate sizes and pointers on the host (no partial launch on error), then enqueue
 * on `stream` and return; nothing is allocated, nothing synchronises.  Calls whose sequences
 * share a pool row race.  Errors: GDN_ERR_INVALID_ARG (sizes, NULL), GDN_ERR_ALIGNMENT (a
 * tensor not 16-byte aligned), GDN_ERR_UNSUPPORTED (d not in {32, 64, 128}, d_k != d_v,
 * L > 64), GDN_ERR_CUDA (launch failure).
 */
#ifndef GDN_DECODE_H
#define GDN_DECODE_H

#include "gdn_dual.h"

#ifdef __cplusplus
extern "C" {
#endif

/* num_seqs N >= 1; num_heads H >= 1; d_k == d_v in {32, 64, 128}; num_tokens L in [1, 64];
 * pool_slots P >= 1; dtype a gdn_dtype; reserved must be 0. */
typedef struct {
    int32_t num_seqs;
    int32_t num_heads;
    int32_t d_k;
    int32_t d_v;
    int32_t num_tokens;
    int32_t pool_slots;
    int32_t dtype;
    int32_t reserved;
} gdn_decode_desc;

/* Causal replay of a committed block (Diffusion-Trust): for every sequence n and head h,
 * S := state_pool[slots[n], h], then the L tokens in order (o_t written to out), then
 * state_pool[slots[n], h] := S. */
gdn_status gdn_decode_replay(const gdn_decode_desc *desc, float *state_pool, const int32_t *slots,
                             const void *q, const void *k, const void *v, const float *g, const float *beta,
                             void *out, int32_t *device_status, gdn_stream_t stream);

/* Verify forward with state cache (AR-Trust): as the replay, but the pool is only read; the
 * state after step t is written to state_cache[n, t, h]. */
gdn_status gdn_decode_verify(const gdn_decode_desc *desc, const float *state_pool, const int32_t *slots,
                             const void *q, const void *k, const void *v, const float *g, const float *beta,
                             void *out, float *state_cache, int32_t *device_status, gdn_stream_t stream);

/* Commit the accepted prefix (AR-Trust rollback by gather-scatter): for every sequence n with
 * r = accepted[n] >= 1, state_pool[slots[n]] := state_cache[n, r - 1]; r = 0 leaves the row. */
gdn_status gdn_decode_commit(const gdn_decode_desc *desc, float *state_pool, const int32_t *slots,
                             const float *state_cache, const int32_t *accepted, int32_t *device_status,
                             gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_DECODE_H */
