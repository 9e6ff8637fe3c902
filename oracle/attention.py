"""fp64 CPU oracle for the dual-stream softmax attention with the document-blocked
causal / block-bidirectional mask.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline leg
may import this module.  It shares no code with the CUDA library.

What it computes ("FLARE: Diffusion for Hybrid Language Model", papernotes.org notes, Method >
Overall framework: the softmax layers see the two streams through one document-blocked mask that
is causal for the clean stream and bidirectional inside each noisy block; Method > Key design 1:
a noisy block b is predicted from its own noisy tokens and the clean tokens before it,
x^{<b}).  Per document n (tokens [s_n, s_{n+1}), prompt length P_n, response cut into blocks of
B tokens) and query head h (key/value head h // (H / H_kv)):

  clean query at position p:           keys/values = clean tokens [s_n, p]          (causal)
  noisy query of view v, block b:      keys/values = clean tokens [s_n, l_b)        (the clean
                                       prefix before the block, l_b = s_n + P_n + (b-1)B)
                                       + the B noisy tokens of block b in view v    (bidirectional)

  o = softmax(q K^T / sqrt(d)) V  over exactly those keys.

No key crosses a document boundary and no noisy query sees another block or another view.
Each function evaluates that definition directly with dense fp64 matrix products per document
(or per block); there is no blocking, online softmax or reordering.
"""
from __future__ import annotations

import numpy as np


def _softmax_rows(s: np.ndarray) -> np.ndarray:
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def _as64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def dual_attention(q, k, v, qn, kn, vn, doc_offsets, prompt_len, block_size):
    """Outputs (out [T, H, d], out_noisy [V, T_R, H, d]) in fp64.

    q [T, H, d], k and v [T, H_kv, d]; qn [V, T_R, H, d], kn and vn [V, T_R, H_kv, d] (noisy
    rows packed over response tokens, documents in order); doc_offsets [N+1], prompt_len [N]."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    qn, kn, vn = _as64(qn), _as64(kn), _as64(vn)
    offs = np.asarray(doc_offsets, dtype=np.int64)
    pl = np.asarray(prompt_len, dtype=np.int64)
    T, H, d = q.shape
    Hkv = k.shape[1]
    V = qn.shape[0]
    B = int(block_size)
    grp = H // Hkv
    scale = 1.0 / np.sqrt(d)
    out = np.zeros((T, H, v.shape[2]))
    out_n = np.zeros((V, qn.shape[1], H, vn.shape[3]))
    roff = 0
    for n in range(len(pl)):
        s, e = int(offs[n]), int(offs[n + 1])
        L, P = e - s, int(pl[n])
        R = L - P
        for h in range(H):
            hk = h // grp
            if L > 0:
                Q, K, Vv = q[s:e, h], k[s:e, hk], v[s:e, hk]
                S = (Q @ K.T) * scale
                S[np.triu_indices(L, 1)] = -np.inf          # key position > query position
                out[s:e, h] = _softmax_rows(S) @ Vv
            for w in range(V):
                for b0 in range(0, R, B):
                    pre = P + b0                              # clean keys [s, s + pre)
                    rows = slice(roff + b0, roff + b0 + B)
                    Kc = np.concatenate([k[s:s + pre, hk], kn[w, rows, hk]], axis=0)
                    Vc = np.concatenate([v[s:s + pre, hk], vn[w, rows, hk]], axis=0)
                    S = (qn[w, rows, h] @ Kc.T) * scale
                    out_n[w, rows, h] = _softmax_rows(S) @ Vc
        roff += R
    return out, out_n


def dual_attention_rows(q, k, v, qn, kn, vn, doc_offsets, prompt_len, block_size, clean_rows, noisy_rows):
    """The same definition evaluated only at the given query rows: clean_rows = [(p, h)],
    noisy_rows = [(view, packed row, h)].  Returns two lists of d-vectors (fp64)."""
    offs = np.asarray(doc_offsets, dtype=np.int64)
    pl = np.asarray(prompt_len, dtype=np.int64)
    H, Hkv = q.shape[1], k.shape[1]
    grp = H // Hkv
    d = q.shape[2]
    scale = 1.0 / np.sqrt(d)
    roffs = np.concatenate([[0], np.cumsum(np.diff(offs) - pl)])
    B = int(block_size)

    def one(qv, K, Vv):
        s = (K @ qv) * scale
        w = np.exp(s - s.max())
        return (w / w.sum()) @ Vv

    res_c = []
    for p, h in clean_rows:
        n = int(np.searchsorted(offs, p, side="right") - 1)
        s = int(offs[n])
        hk = h // grp
        res_c.append(one(_as64(q[p, h]), _as64(k[s:p + 1, hk]), _as64(v[s:p + 1, hk])))
    res_n = []
    for w, r, h in noisy_rows:
        n = int(np.searchsorted(roffs, r, side="right") - 1)
        s, P = int(offs[n]), int(pl[n])
        b0 = ((r - int(roffs[n])) // B) * B
        rows = slice(int(roffs[n]) + b0, int(roffs[n]) + b0 + B)
        hk = h // grp
        K = np.concatenate([_as64(k[s:s + P + b0, hk]), _as64(kn[w, rows, hk])], axis=0)
        Vv = np.concatenate([_as64(v[s:s + P + b0, hk]), _as64(vn[w, rows, hk])], axis=0)
        res_n.append(one(_as64(qn[w, r, h]), K, Vv))
    return res_c, res_n
