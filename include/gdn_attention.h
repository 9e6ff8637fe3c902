/*
 * gdn_attention.h -- C ABI of the dual-stream softmax attention with the document-blocked
 * causal / block-bidirectional mask (B200, sm_100a).
 *
 * "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes), Method > Overall
 * framework: in the hybrid model's softmax-attention layers the clean stream and the noisy
 * stream share one document-blocked mask that is causal for the clean stream and bidirectional
 * inside every noisy block; Method > Key design 1: a noisy block b is predicted from its own
 * noisy tokens and the clean tokens before it (x^{<b}).  Per document n (tokens [s_n, s_{n+1}),
 * prompt length P_n, response cut into blocks of B tokens) and query head h, with key/value
 * head h / (H / H_kv):
 *
 *   clean query at position p:       keys = clean tokens [s_n, p]
 *   noisy query of view v, block b:  keys = clean tokens [s_n, s_n + P_n + (b-1)B)
 *                                          + the B noisy tokens of block b in view v
 *   o = softmax(q K^T / sqrt(d)) V over those keys.
 *
 * Layouts (row-major, contiguous, caller-owned device memory, bf16):
 *   q, out        [T, H, d]           clean stream
 *   k, v          [T, H_kv, d]
 *   qn, out_noisy [V, T_R, H, d]      noisy stream, packed over response tokens (documents in
 *   kn, vn        [V, T_R, H_kv, d]   order), the layout of gdn_dual_forward's noisy twins
 *   doc_offsets   [N+1] int32, HOST   doc_offsets[0] = 0, non-decreasing, T = doc_offsets[N]
 *   prompt_len    [N] int32, HOST     0 <= P_n <= len_n, (len_n - P_n) % B == 0
 *   workspace     device, >= gdn_attn_workspace_size(...) bytes (256), 16-byte aligned: the
 *                 device status word (GDN_ERR_TIMEOUT if a bounded wait gave up; read it with
 *                 gdn_dual_read_device_status), cleared on `stream` by each call.
 *
 * gdn_attn_forward validates on the host (no partial launch on error), enqueues on `stream`
 * and returns; nothing is allocated and nothing synchronises.  Errors: GDN_ERR_INVALID_ARG
 * (sizes, layout, NULL, workspace too small), GDN_ERR_ALIGNMENT (a pointer not 16-byte
 * aligned), GDN_ERR_UNSUPPORTED (d != 128, dtype not bf16, 128 % B != 0, V > 2, H % H_kv != 0,
 * more than 1024 documents), GDN_ERR_CUDA (launch failure).
 */
#ifndef GDN_ATTENTION_H
#define GDN_ATTENTION_H

#include "gdn_dual.h"

#ifdef __cplusplus
extern "C" {
#endif

/* num_docs N >= 1, num_heads H >= 1, num_kv_heads H_kv >= 1 dividing H, head_dim d,
 * num_views V >= 0, block_size B >= 1, dtype a gdn_dtype, reserved = 0. */
typedef struct {
    int32_t num_docs;
    int32_t num_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t num_views;
    int32_t block_size;
    int32_t dtype;
    int32_t reserved;
} gdn_attn_desc;

/* Workspace bytes for a call with this descriptor and document layout (host arrays); 0 when
 * the descriptor or the layout is invalid. */
size_t gdn_attn_workspace_size(const gdn_attn_desc *desc, const int32_t *doc_offsets_host,
                               const int32_t *prompt_len_host);

/* out = clean-stream attention, out_noisy = noisy-stream attention (see above).  With V = 0 or
 * no response tokens, qn/kn/vn/out_noisy may be NULL. */
gdn_status gdn_attn_forward(const gdn_attn_desc *desc, const void *q, const void *k, const void *v,
                            const void *qn, const void *kn, const void *vn,
                            const int32_t *doc_offsets, const int32_t *prompt_len,
                            void *out, void *out_noisy, void *workspace, size_t workspace_bytes,
                            gdn_stream_t stream);

/* FOR TESTS of the bounded-wait error path only: gdn_attn_forward with every device-side wait
 * bounded by `wait_iters` non-blocking polls (>= 1).  A wait that gives up records
 * GDN_ERR_TIMEOUT in the workspace; the kernel then waits with the normal bound for every copy
 * and MMA it issued before it leaves; outputs are unspecified.  (No counterpart in the notes.) */
gdn_status gdn_attn_forward_test_wait_limit(const gdn_attn_desc *desc, const void *q, const void *k,
                                            const void *v, const void *qn, const void *kn, const void *vn,
                                            const int32_t *doc_offsets, const int32_t *prompt_len,
                                            void *out, void *out_noisy, void *workspace, size_t workspace_bytes,
                                            uint32_t wait_iters, gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_ATTENTION_H */
