"""Independent brute-force formulations used to pin the oracle (test code only).

Nothing here is shared with the oracle or with the CUDA library.  Each function
restates a definition from "FLARE: Diffusion for Hybrid Language Model"
(papernotes.org notes) in a different form from the oracle's token loop:
explicit d x d transition matrices and explicit matrix products for the gated
delta rule (Key design 2), and explicit tap matrices for the ShortConv
anti-leak rule (Key design 3).
"""
from __future__ import annotations

import numpy as np


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_problem(rng, lens, prompts, H=2, dk=8, dv=8, V=2, B=4, conv=0, g_lo=-0.3, beta_std=1.0):
    """Seeded random inputs as fp64 numpy arrays, layout as in the library header."""
    lens = np.asarray(lens, dtype=np.int64)
    prompts = np.asarray(prompts, dtype=np.int64)
    T = int(lens.sum())
    TR = int((lens - prompts).sum())
    offs = np.zeros(len(lens) + 1, dtype=np.int32)
    offs[1:] = np.cumsum(lens)

    def stream(n):
        return (unit_rows(rng.standard_normal((n, H, dk))), unit_rows(rng.standard_normal((n, H, dk))),
                rng.standard_normal((n, H, dv)), rng.uniform(g_lo, 0.0, (n, H)),
                1.0 / (1.0 + np.exp(-beta_std * rng.standard_normal((n, H)))))

    q, k, v, g, beta = stream(T)
    views = [stream(TR) for _ in range(V)]
    P = dict(q=q, k=k, v=v, g=g, beta=beta,
             qn=np.stack([w[0] for w in views]) if V else np.zeros((0, TR, H, dk)),
             kn=np.stack([w[1] for w in views]) if V else np.zeros((0, TR, H, dk)),
             vn=np.stack([w[2] for w in views]) if V else np.zeros((0, TR, H, dv)),
             gn=np.stack([w[3] for w in views]) if V else np.zeros((0, TR, H)),
             betan=np.stack([w[4] for w in views]) if V else np.zeros((0, TR, H)),
             doc_offsets=offs, prompt_len=prompts.astype(np.int32), block_size=B, conv_w=None)
    if conv:
        assert dk == dv
        P["conv_w"] = 0.5 * rng.standard_normal((3, H * dk, conv))
    return P


def copy_problem(P):
    return {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in P.items()}


def response_offsets(P):
    lens = np.diff(P["doc_offsets"].astype(np.int64)) - P["prompt_len"]
    out = np.zeros(len(lens) + 1, dtype=np.int64)
    out[1:] = np.cumsum(lens)
    return out


def transition(alpha, beta, k):
    """A = alpha * (I - beta k k^T) as an explicit matrix."""
    d = k.shape[0]
    return alpha * (np.eye(d) - beta * np.outer(k, k))


def clean_states_brute(k, v, g, beta):
    """All clean states S_0..S_{L-1} of one (doc, head) by the explicit sum
    S_t = sum_{i<=t} (A_t ... A_{i+1}) beta_i k_i v_i^T  (zero initial state)."""
    L, dk = k.shape
    dv = v.shape[1]
    As = [transition(np.exp(g[j]), beta[j], k[j]) for j in range(L)]
    states = []
    for t in range(L):
        S = np.zeros((dk, dv))
        for i in range(t + 1):
            M = np.eye(dk)
            for j in range(t, i, -1):       # A_t A_{t-1} ... A_{i+1}
                M = M @ As[j]
            S = S + M @ (beta[i] * np.outer(k[i], v[i]))
        states.append(S)
    return states


def block_end_brute(S_e, kb, vb, gb, bb):
    """Noisy block-end state from the boundary state by the explicit product form
    S~ = (A~_B ... A~_1) S_e + sum_l (A~_B ... A~_{l+1}) beta~_l k~_l v~_l^T."""
    Bn = kb.shape[0]
    As = [transition(np.exp(gb[j]), bb[j], kb[j]) for j in range(Bn)]
    M = np.eye(S_e.shape[0])
    for j in range(Bn - 1, -1, -1):
        M = M @ As[j]
    S = M @ S_e
    for l in range(Bn):
        M = np.eye(S_e.shape[0])
        for j in range(Bn - 1, l, -1):
            M = M @ As[j]
        S = S + M @ (bb[l] * np.outer(kb[l], vb[l]))
    return S


def conv_matrices(w_row, L, P, B):
    """Explicit tap matrices for one channel of one document of length L with prompt P.
    Returns (Cc, Cn_clean, Cn_noisy): clean x' = Cc @ x; noisy x~' = Cn_clean @ x + Cn_noisy @ x~
    where x~ holds the document's response rows (length L-P).  Tap W-1 is the current token."""
    W = w_row.shape[0]
    R = L - P
    Cc = np.zeros((L, L))
    for p in range(L):
        for j in range(W):
            if p - j >= 0:
                Cc[p, p - j] = w_row[W - 1 - j]
    Cn_clean = np.zeros((R, L))
    Cn_noisy = np.zeros((R, R))
    for r in range(R):
        p = P + r
        blk = P + (r // B) * B
        for j in range(W):
            src = p - j
            if src >= blk:
                Cn_noisy[r, src - P] = w_row[W - 1 - j]
            elif src >= 0:
                Cn_clean[r, src] = w_row[W - 1 - j]
    return Cc, Cn_clean, Cn_noisy


def apply_conv_brute(P):
    """Return a copy of the problem with the ShortConv prologue applied to q, k, v (both
    streams) through explicit tap matrices, and conv_w removed."""
    cw = P["conv_w"]
    out = copy_problem(P)
    out["conv_w"] = None
    offs = P["doc_offsets"]
    pl = P["prompt_len"]
    roff = response_offsets(P)
    H = P["q"].shape[1]
    B = P["block_size"]
    for which, name in enumerate(("q", "k", "v")):
        x = P[name]
        xn = P[name + "n"]
        d = x.shape[2]
        for n in range(len(pl)):
            s0, s1 = offs[n], offs[n + 1]
            L, Pn = s1 - s0, pl[n]
            r0, r1 = roff[n], roff[n + 1]
            for h in range(H):
                for c in range(d):
                    Cc, Cnc, Cnn = conv_matrices(cw[which, h * d + c], L, Pn, B)
                    xc = x[s0:s1, h, c]
                    out[name][s0:s1, h, c] = Cc @ xc
                    for view in range(xn.shape[0]):
                        out[name + "n"][view, r0:r1, h, c] = Cnc @ xc + Cnn @ xn[view, r0:r1, h, c]
    return out


def forward_brute(P):
    """Brute-force forward (no conv) for small problems: outputs and noisy block-end states."""
    q, k, v, g, beta = P["q"], P["k"], P["v"], P["g"], P["beta"]
    offs, pl, B = P["doc_offsets"], P["prompt_len"], P["block_size"]
    T, H, dk = q.shape
    dv = v.shape[2]
    V, TR = P["qn"].shape[:2]
    roff = response_offsets(P)
    out = np.zeros((T, H, dv))
    out_noisy = np.zeros((V, TR, H, dv))
    final = np.zeros((len(pl), H, dk, dv))
    nstate = np.zeros((V, TR // B, H, dk, dv))
    sc = 1.0 / np.sqrt(dk)
    for n in range(len(pl)):
        s0, s1 = offs[n], offs[n + 1]
        Pn = pl[n]
        for h in range(H):
            states = clean_states_brute(k[s0:s1, h], v[s0:s1, h], g[s0:s1, h], beta[s0:s1, h])
            for t in range(s1 - s0):
                out[s0 + t, h] = states[t].T @ q[s0 + t, h] * sc
            final[n, h] = states[-1] if s1 > s0 else 0.0
            for r in range(0, s1 - s0 - Pn, B):
                e = Pn + r - 1
                S_e = states[e] if e >= 0 else np.zeros((dk, dv))
                rows = slice(roff[n] + r, roff[n] + r + B)
                for view in range(V):
                    S_end = block_end_brute(S_e, P["kn"][view, rows, h], P["vn"][view, rows, h],
                                            P["gn"][view, rows, h], P["betan"][view, rows, h])
                    nstate[view, (roff[n] + r) // B, h] = S_end
                    for l in range(B):
                        out_noisy[view, roff[n] + r + l, h] = S_end.T @ P["qn"][view, roff[n] + r + l, h] * sc
    return dict(out=out, out_noisy=out_noisy, final_state=final, noisy_state=nstate)
