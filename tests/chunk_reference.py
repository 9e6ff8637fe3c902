"""fp64 numpy evaluation of the chunked (WY / UT) factorisation that the tensor-core kernel
uses, for checking the derivation against the sequential oracle (test code only).

Derivation (from the gated delta rule of "FLARE: Diffusion for Hybrid Language Model",
papernotes.org notes, Method > Key design 2).  Write the update as
    S_t = alpha_t S_{t-1} + k_t u_t^T,   u_t = beta_t v_t - alpha_t beta_t S_{t-1}^T k_t .
Inside a chunk with start state S0, gamma = inclusive cumsum of g, Gamma = exp(gamma):
    S_t = Gamma_t S0 + sum_{i<=t} e^{gamma_t - gamma_i} k_i u_i^T
    (I + A) U = diag(beta) V - diag(beta Gamma) K S0,  A_ti = beta_t e^{gamma_t-gamma_i} k_t.k_i (i<t)
    O = [diag(Gamma) Q S0 + (Q K^T o D) U] / sqrt(d),   D_ti = e^{gamma_t-gamma_i} (i<=t)
    S_C = Gamma_C S0 + (diag(e^{gamma_C - gamma}) K)^T U
Noisy rows of a block whose boundary e lies in the chunk (e = -1 means S0 itself):
    x S_e = Gamma_e x S0 + sum_{i<=e} e^{gamma_e-gamma_i} (x.k_i) u_i
and the block's own B-step recurrence from S_e has the same form with its own T~:
    U~ = T~ (diag(b~) V~ - diag(b~ Gamma~) K~ S_e)
    O~ = [Gamma~_B Q~ S_e + (Q~ K~^T o D~) U~] / sqrt(d),  D~_lj = e^{gamma~_B - gamma~_j} (all j)
The chunk grid of a document is anchored at its response start so that no block straddles
a chunk (chunk size a multiple of B).
"""
from __future__ import annotations

import numpy as np

import brute


def chunk_bounds(s0, s1, r, C):
    """Chunks [a, b) covering [s0, s1) on the grid r + m*C."""
    first = r - ((r - s0 + C - 1) // C) * C if r > s0 else r
    out = []
    a = max(first, s0)
    nxt = first + C
    while a < s1:
        b = min(nxt, s1)
        out.append((a, b))
        a = b
        nxt += C
    return out


def forward_chunked(P, C=64):
    if P.get("conv_w") is not None:
        P = brute.apply_conv_brute(P)
    q, k, v, g, beta = P["q"], P["k"], P["v"], P["g"], P["beta"]
    offs, pl, B = P["doc_offsets"], P["prompt_len"], P["block_size"]
    assert C % B == 0
    T, H, dk = q.shape
    dv = v.shape[2]
    V, TR = P["qn"].shape[:2]
    roff = brute.response_offsets(P)
    out = np.zeros((T, H, dv))
    out_noisy = np.zeros((V, TR, H, dv))
    final = np.zeros((len(pl), H, dk, dv))
    sc = 1.0 / np.sqrt(dk)
    for n in range(len(pl)):
        s0, s1 = int(offs[n]), int(offs[n + 1])
        r = s0 + int(pl[n])
        for h in range(H):
            S0 = np.zeros((dk, dv))
            for (a, b) in chunk_bounds(s0, s1, r, C):
                Q, K, Vv = q[a:b, h], k[a:b, h], v[a:b, h]
                gam = np.cumsum(g[a:b, h])
                bet = beta[a:b, h]
                Gam = np.exp(gam)
                L = b - a
                lower = np.tril(np.ones((L, L))) > 0
                strict = np.tril(np.ones((L, L)), -1) > 0
                decay = np.exp(np.where(lower, gam[:, None] - gam[None, :], 0.0))   # e^{gamma_t-gamma_i}
                A = np.where(strict, bet[:, None] * decay * (K @ K.T), 0.0)
                Tm = np.linalg.inv(np.eye(L) + A)
                U = Tm @ (bet[:, None] * Vv - (bet * Gam)[:, None] * (K @ S0))
                D = np.where(lower, decay, 0.0)
                out[a:b, h] = (Gam[:, None] * (Q @ S0) + ((Q @ K.T) * D) @ U) * sc
                # noisy blocks inside this chunk
                for blk_start in range(max(a, r), b, B):
                    e = blk_start - 1 - a           # chunk-local boundary index, -1 = S0
                    rrow = roff[n] + (blk_start - r)
                    for view in range(V):
                        Qn = P["qn"][view, rrow:rrow + B, h]
                        Kn = P["kn"][view, rrow:rrow + B, h]
                        Vn = P["vn"][view, rrow:rrow + B, h]
                        gn = np.cumsum(P["gn"][view, rrow:rrow + B, h])
                        bn = P["betan"][view, rrow:rrow + B, h]

                        def at_boundary(X):
                            if e < 0:
                                return X @ S0
                            w = np.exp(gam[e] - gam[:e + 1])
                            return Gam[e] * (X @ S0) + ((X @ K[:e + 1].T) * w[None, :]) @ U[:e + 1]

                        QS, KS = at_boundary(Qn), at_boundary(Kn)
                        sn = np.tril(np.ones((B, B)), -1) > 0
                        dn = np.exp(np.where(sn, gn[:, None] - gn[None, :], 0.0))
                        An = np.where(sn, bn[:, None] * dn * (Kn @ Kn.T), 0.0)
                        Tn = np.linalg.inv(np.eye(B) + An)
                        Un = Tn @ (bn[:, None] * Vn - (bn * np.exp(gn))[:, None] * KS)
                        Dn = np.exp(gn[-1] - gn)[None, :]
                        out_noisy[view, rrow:rrow + B, h] = (np.exp(gn[-1]) * QS + ((Qn @ Kn.T) * Dn) @ Un) * sc
                S0 = Gam[-1] * S0 + (np.exp(gam[-1] - gam)[:, None] * K).T @ U
            final[n, h] = S0
    return dict(out=out, out_noisy=out_noisy, final_state=final)


def forward_chunked_folded(P, C=64):
    """The factorisation the tensor-core kernel evaluates, in fp64.  Clean stream as in
    forward_chunked but with U from [P T; T] R (R = beta V - beta Gamma K S0).  Noisy rows are
    folded per block: with y_j = P~_j T~ (one row of the block's readout times its WY inverse),
        Z_j  = Gamma~_B q~_j - sum_l y_l beta~_l Gamma~_l k~_l
        WV_j = sum_l y_l beta~_l v~_l
        o~_j = Gamma_e Z_j S0 + (Z_j K^T o M_j) U + WV_j,   M_ji = e^{gamma_e - gamma_i} [i <= e]
    so each noisy row needs one product with S0 and one with the chunk's U."""
    if P.get("conv_w") is not None:
        P = brute.apply_conv_brute(P)
    q, k, v, g, beta = P["q"], P["k"], P["v"], P["g"], P["beta"]
    offs, pl, B = P["doc_offsets"], P["prompt_len"], P["block_size"]
    T_, H, dk = q.shape
    dv = v.shape[2]
    V, TR = P["qn"].shape[:2]
    roff = brute.response_offsets(P)
    out = np.zeros((T_, H, dv))
    out_noisy = np.zeros((V, TR, H, dv))
    final = np.zeros((len(pl), H, dk, dv))
    sc = 1.0 / np.sqrt(dk)
    for n in range(len(pl)):
        s0, s1 = int(offs[n]), int(offs[n + 1])
        r = s0 + int(pl[n])
        for h in range(H):
            S0 = np.zeros((dk, dv))
            for (a, b) in chunk_bounds(s0, s1, r, C):
                Q, K, Vv = q[a:b, h], k[a:b, h], v[a:b, h]
                gam = np.cumsum(g[a:b, h])
                bet = beta[a:b, h]
                Gam = np.exp(gam)
                L = b - a
                lower = np.tril(np.ones((L, L))) > 0
                strict = np.tril(np.ones((L, L)), -1) > 0
                decay = np.exp(np.where(lower, gam[:, None] - gam[None, :], 0.0))
                A = np.where(strict, bet[:, None] * decay * (K @ K.T), 0.0)
                Tm = np.linalg.inv(np.eye(L) + A)
                Pm = np.where(lower, (Q @ K.T) * decay, 0.0)
                R = bet[:, None] * Vv - (bet * Gam)[:, None] * (K @ S0)
                Y = np.vstack([Pm @ Tm, Tm]) @ R                    # [P U ; U]
                PU, U = Y[:L], Y[L:]
                out[a:b, h] = (Gam[:, None] * (Q @ S0) + PU) * sc
                for blk_start in range(max(a, r), b, B):
                    e = blk_start - 1 - a
                    rrow = roff[n] + (blk_start - r)
                    Ge = np.exp(gam[e]) if e >= 0 else 1.0
                    Mrow = np.zeros(L)
                    if e >= 0:
                        Mrow[:e + 1] = np.exp(gam[e] - gam[:e + 1])
                    for view in range(V):
                        Qn = P["qn"][view, rrow:rrow + B, h]
                        Kn = P["kn"][view, rrow:rrow + B, h]
                        Vn = P["vn"][view, rrow:rrow + B, h]
                        gn = np.cumsum(P["gn"][view, rrow:rrow + B, h])
                        bn = P["betan"][view, rrow:rrow + B, h]
                        An = np.zeros((B, B))
                        for jj in range(B):
                            for ll in range(jj):
                                An[jj, ll] = bn[jj] * np.exp(gn[jj] - gn[ll]) * (Kn[jj] @ Kn[ll])
                        for jj in range(B):
                            Pt = (Qn[jj] @ Kn.T) * np.exp(gn[-1] - gn)
                            y = np.zeros(B)
                            for ll in range(B - 1, -1, -1):          # y (I + A~) = P~_j
                                y[ll] = Pt[ll] - sum(y[m] * An[m, ll] for m in range(ll + 1, B))
                            Z = np.exp(gn[-1]) * Qn[jj] - (y * bn * np.exp(gn)) @ Kn
                            WV = (y * bn) @ Vn
                            o = Ge * (Z @ S0) + ((Z @ K.T) * Mrow) @ U + WV
                            out_noisy[view, rrow + jj, h] = o * sc
                S0 = Gam[-1] * S0 + (np.exp(gam[-1] - gam)[:, None] * K).T @ U
            final[n, h] = S0
    return dict(out=out, out_noisy=out_noisy, final_state=final)
