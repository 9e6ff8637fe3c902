"""fp64 numpy evaluation of the backward of the chunked (WY / UT) factorisation, for checking
the derivation a tensor-core backward would use against the token-by-token backward oracle
(test code only).

Forward per chunk (start state S0, gamma = inclusive cumsum of g, Gamma = e^gamma,
D_ti = e^{gamma_t - gamma_i} for i <= t; the notation of tests/chunk_reference.py):
    A  = strict(beta_t D_ti k_t.k_i),  T = (I + A)^-1
    R  = diag(beta) V - diag(beta Gamma) K S0,   U = T R
    O  = s [diag(Gamma) Q S0 + M U],  M = (Q K^T) o D (i <= t),  s = 1 / sqrt(d)
    S_C = Gamma_C S0 + Khat^T U,  Khat = diag(e^{gamma_C - gamma}) K
Backward with dO and dS_C (the adjoint at the chunk end), by the chain rule through each line:
    dU  = s M^T dO + Khat dS_C,     dR = T^T dU,     dA = -(dR U^T) on the strict lower part
    dS0 = Gamma_C dS_C + s Q^T diag(Gamma) dO - K^T diag(beta Gamma) dR      (adjoint at the start)
    dV  = diag(beta) dR
    dQ  = s [diag(Gamma) dO S0^T + (dM o D) K],   dM = s dO U^T
    dK  = (dM o D)^T Q + diag(e^{gamma_C-gamma}) U dS_C^T - diag(beta Gamma) dR S0^T + G K + G^T K,
          G = dA o beta_t D_ti (strict)
    dbeta_t = dR_t.V_t - Gamma_t dR_t.(K S0)_t + sum_i G'_ti,  G' = dA o D o (K K^T) (strict)
    dgamma from Gamma (O, R, S_C) and from every e^{gamma_t - gamma_i} (M, A, Khat);
    dg = reverse cumulative sum of dgamma inside the chunk.
Noisy blocks: the views' initial-state gradient Lam_e of a block whose boundary state is
    S_e = Gamma_e S0 + sum_{i<=e} e^{gamma_e - gamma_i} k_i u_i^T
enters the chunk backward like one more read-out of the chunk, at row e instead of C:
    dS0 += Gamma_e Lam_e,  du_i += e^{gamma_e-gamma_i} Lam_e^T k_i,  dk_i += e^{gamma_e-gamma_i} Lam_e u_i  (i <= e)
plus the matching decay terms; Lam_e has rank B per view (the block's B queries carried back
through its B steps), the backward mirror of the forward's Z rows.
"""
from __future__ import annotations

import numpy as np

# Operand rounding of the matrix products (identity: exact fp64).  The precision study sets it
# to bf16 rounding to emulate tensor-core products with bf16 operands and wide accumulation.
_ROUND = None


def set_operand_rounding(fn):
    global _ROUND
    _ROUND = fn


def mm(a, b):
    if _ROUND is not None:
        a, b = _ROUND(a), _ROUND(b)
    return a @ b


def clean_backward_chunked(q, k, v, g, beta, doc_offsets, d_out, d_final_state, C=64):
    """Clean-stream gradients (dq, dk, dv, dg, dbeta) by chunks of C tokens from each document
    start; fp64."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    do = np.asarray(d_out, dtype=np.float64)
    dsf = np.asarray(d_final_state, dtype=np.float64)
    offs = np.asarray(doc_offsets, dtype=np.int64)
    T, H, dk = q.shape
    dv = v.shape[2]
    s = 1.0 / np.sqrt(dk)
    res = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("dbeta", beta))}
    for n in range(len(offs) - 1):
        s0, s1 = int(offs[n]), int(offs[n + 1])
        chunks = [(a, min(a + C, s1)) for a in range(s0, s1, C)]
        for h in range(H):
            # forward: chunk start states
            starts = []
            S = np.zeros((dk, dv))
            for a, b in chunks:
                starts.append(S.copy())
                f = _chunk_forward(q[a:b, h], k[a:b, h], v[a:b, h], g[a:b, h], beta[a:b, h], S, s)
                S = f["SC"]
            lam = dsf[n, h].copy()
            for (a, b), S0 in reversed(list(zip(chunks, starts))):
                f = _chunk_forward(q[a:b, h], k[a:b, h], v[a:b, h], g[a:b, h], beta[a:b, h], S0, s)
                gr = _chunk_backward(f, do[a:b, h], lam, s)
                for name in ("dq", "dk", "dv", "dg", "dbeta"):
                    res[name][a:b, h] = gr[name]
                lam = gr["dS0"]
    return res


def _chunk_forward(Q, K, V, g, beta, S0, s):
    L = Q.shape[0]
    gam = np.cumsum(g)
    Gam = np.exp(gam)
    lower = np.tril(np.ones((L, L))) > 0
    strict = np.tril(np.ones((L, L)), -1) > 0
    D = np.where(lower, np.exp(np.where(lower, gam[:, None] - gam[None, :], 0.0)), 0.0)
    KK = mm(K, K.T)
    A = np.where(strict, beta[:, None] * D * KK, 0.0)
    Tm = np.linalg.inv(np.eye(L) + A)
    KS0 = mm(K, S0)
    R = beta[:, None] * V - (beta * Gam)[:, None] * KS0
    U = mm(Tm, R)
    M = mm(Q, K.T) * D
    ec = np.exp(gam[-1] - gam)                    # e^{gamma_C - gamma_i}
    Khat = ec[:, None] * K
    O = s * (Gam[:, None] * mm(Q, S0) + mm(M, U))
    SC = Gam[-1] * S0 + mm(Khat.T, U)
    return dict(Q=Q, K=K, V=V, beta=beta, S0=S0, gam=gam, Gam=Gam, lower=lower, strict=strict, D=D, KK=KK,
                A=A, Tm=Tm, KS0=KS0, R=R, U=U, M=M, ec=ec, Khat=Khat, O=O, SC=SC)


def chunk_state(f, e):
    """S_e (the state after chunk-local token e; e = -1: S0) = Gamma_e S0 + sum_{i<=e} e^{gamma_e-gamma_i} k_i u_i^T."""
    if e < 0:
        return f["S0"].copy()
    w = np.exp(f["gam"][e] - f["gam"][:e + 1])
    return f["Gam"][e] * f["S0"] + mm((w[:, None] * f["K"][:e + 1]).T, f["U"][:e + 1])


def _chunk_backward(f, dO, dSC, s, inject=(), rows=None):
    """inject: (e, Lam_e) pairs, gradients dL/dS_e of block-boundary states inside the chunk
    (the views' initial-state gradients of the noisy block starting after token e).
    rows: the same injections in rank-B form, (X, dOx, e) with X [n, d_k] the carried-back
    queries, dOx [n, d_v] their upstream gradients and e [n] their boundary rows: each row reads
    S_e^T x like an output row with its decay boundary at e, as the forward's Z rows do."""
    Q, K, V, beta, S0 = f["Q"], f["K"], f["V"], f["beta"], f["S0"]
    Gam, D, KK, Tm, U, R, M, ec, Khat = f["Gam"], f["D"], f["KK"], f["Tm"], f["U"], f["R"], f["M"], f["ec"], f["Khat"]
    strict, lower, KS0, gam = f["strict"], f["lower"], f["KS0"], f["gam"]
    L = Q.shape[0]
    dU = s * mm(M.T, dO) + mm(Khat, dSC)
    dS0_inj = np.zeros_like(S0)
    dK_inj = np.zeros_like(K)
    dgam_inj = np.zeros(L)
    if rows is not None and len(rows[0]):
        X, dOx, e = rows
        e = np.asarray(e)
        ge = np.where(e >= 0, gam[np.maximum(e, 0)], 0.0)          # gamma at the boundary (0 for S0)
        Ge = np.where(e >= 0, Gam[np.maximum(e, 0)], 1.0)
        vis = np.arange(L)[None, :] <= e[:, None]                    # key i visible from boundary e
        DX = np.where(vis, np.exp(np.where(vis, ge[:, None] - gam[None, :], 0.0)), 0.0)
        XK = mm(X, K.T)
        MX = XK * DX                                                 # the rows' masked X K^T (like M'_Z)
        dS0_inj += mm(X.T, Ge[:, None] * dOx)
        dU += mm(MX.T, dOx)
        dMX = mm(dOx, U.T)
        dK_inj += mm((dMX * DX).T, X)
        W = dMX * XK * DX                                            # d(decay) terms
        dgam_inj -= W.sum(axis=0)
        tot = W.sum(axis=1) + Ge * np.sum(mm(X, S0) * dOx, axis=1)   # towards gamma at each boundary
        np.add.at(dgam_inj, np.maximum(e, 0), np.where(e >= 0, tot, 0.0))
    for e, lam_e in inject:
        if e < 0:
            dS0_inj += lam_e
            continue
        w = np.exp(gam[e] - gam[:e + 1])                       # e^{gamma_e - gamma_i}, i <= e
        dS0_inj += Gam[e] * lam_e
        dU[:e + 1] += w[:, None] * mm(K[:e + 1], lam_e)
        dK_inj[:e + 1] += w[:, None] * mm(U[:e + 1], lam_e.T)
        t = w * np.sum((K[:e + 1] @ lam_e) * U[:e + 1], axis=1)
        dgam_inj[e] += Gam[e] * np.sum(lam_e * S0) + t.sum()
        dgam_inj[:e + 1] -= t
    dR = mm(Tm.T, dU)
    dA = np.where(strict, -mm(dR, U.T), 0.0)
    dS0 = Gam[-1] * dSC + s * mm(Q.T, Gam[:, None] * dO) - mm(K.T, (beta * Gam)[:, None] * dR) + dS0_inj
    dV = beta[:, None] * dR
    dM = s * mm(dO, U.T)
    dMD = np.where(lower, dM * D, 0.0)
    dQ = s * Gam[:, None] * mm(dO, S0.T) + mm(dMD, K)
    G = np.where(strict, dA * beta[:, None] * D, 0.0)
    dK = mm(dMD.T, Q) + ec[:, None] * mm(U, dSC.T) - (beta * Gam)[:, None] * mm(dR, S0.T) + mm(G, K) + mm(G.T, K) + dK_inj
    dbeta = np.sum(dR * V, axis=1) - Gam * np.sum(dR * KS0, axis=1) + np.sum(np.where(strict, dA * D * KK, 0.0), axis=1)
    # d gamma: through Gamma_t (O and R), Gamma_C (S_C), and the pairwise decays e^{gamma_t-gamma_i}
    dgam = Gam * (s * np.sum(dO * (Q @ S0), axis=1) - beta * np.sum(dR * KS0, axis=1))
    dgam[-1] += Gam[-1] * np.sum(dSC * S0)
    W = np.where(lower, dM * (Q @ K.T) * D, 0.0) + np.where(strict, dA * beta[:, None] * KK * D, 0.0)
    dgam += W.sum(axis=1) - W.sum(axis=0)
    e_term = ec * np.sum((K @ dSC) * U, axis=1)   # d/d(e^{gamma_C - gamma_i}) times the decay
    dgam[-1] += e_term.sum()
    dgam -= e_term
    dgam += dgam_inj
    dg = np.cumsum(dgam[::-1])[::-1]
    return dict(dq=dQ, dk=dK, dv=dV, dg=dg, dbeta=dbeta, dS0=dS0)


def dual_backward_chunked(q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, block_size,
                          d_out, d_out_noisy, d_final_state, C=64, rank_rows=False, checkpoint_round=None):
    """All gradients of the dual-stream forward by chunks of C tokens anchored at each document's
    response start (C a multiple of B, so no block straddles a chunk).  Per chunk: the clean
    forward quantities, the boundary state S_e of every block starting in the chunk, each view's
    B-step block backward from S_e (small dense products), then the chunk backward with the
    views' initial-state gradients injected at their boundaries."""
    import chunk_reference as cr
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    qn, kn, vn, gn, betan = (np.asarray(x, dtype=np.float64) for x in (qn, kn, vn, gn, betan))
    do, don = np.asarray(d_out, dtype=np.float64), np.asarray(d_out_noisy, dtype=np.float64)
    dsf = np.asarray(d_final_state, dtype=np.float64)
    offs = np.asarray(doc_offsets, dtype=np.int64)
    pl = np.asarray(prompt_len, dtype=np.int64)
    B = int(block_size)
    assert C % B == 0
    T, H, dk = q.shape
    V = qn.shape[0]
    s = 1.0 / np.sqrt(dk)
    res = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("dbeta", beta),
                                            ("dqn", qn), ("dkn", kn), ("dvn", vn), ("dgn", gn), ("dbetan", betan))}
    step = lambda S, kk, vv, gg, bb: np.exp(gg) * (S - bb * np.outer(kk, kk @ S)) + bb * np.outer(kk, vv)

    def step_grads(Lam, Sp, kk, vv, gg, bb):
        a = np.exp(gg)
        ks, kl = Sp.T @ kk, Lam.T @ kk
        return (bb * (Lam @ vv) - a * bb * (Lam @ ks + Sp @ kl), bb * kl, a * (np.sum(Lam * Sp) - bb * (ks @ kl)),
                kl @ vv - a * (ks @ kl), a * (Lam - bb * np.outer(kk, kl)))

    roff = 0
    for n in range(len(pl)):
        s0, s1 = int(offs[n]), int(offs[n + 1])
        r = s0 + int(pl[n])
        R = s1 - r
        chunks = cr.chunk_bounds(s0, s1, r, C)
        for h in range(H):
            starts, S = [], np.zeros((dk, dk))
            for a, b in chunks:
                # the chunk-start state as the backward reads it back (checkpoint precision)
                starts.append(S.copy() if checkpoint_round is None else checkpoint_round(S))
                S = _chunk_forward(q[a:b, h], k[a:b, h], v[a:b, h], g[a:b, h], beta[a:b, h], S, s)["SC"]
            lam = dsf[n, h].copy()
            for (a, b), S0 in reversed(list(zip(chunks, starts))):
                f = _chunk_forward(q[a:b, h], k[a:b, h], v[a:b, h], g[a:b, h], beta[a:b, h], S0, s)
                inject = []
                rx, rdo, re_ = [], [], []                       # rank-B rows (rank_rows=True)
                for p in range(max(a, r), b, B):                # blocks starting in this chunk
                    e = p - 1 - a
                    Se = chunk_state(f, e) if (p > s0) else np.zeros_like(S0)
                    rr = roff + (p - r)
                    total = np.zeros_like(S0)
                    for w in range(V):
                        states = [Se]
                        for i in range(B):
                            states.append(step(states[-1], kn[w, rr + i, h], vn[w, rr + i, h], gn[w, rr + i, h],
                                               betan[w, rr + i, h]))
                        Lt = sum(np.outer(qn[w, rr + i, h], don[w, rr + i, h]) for i in range(B)) * s
                        for i in range(B):
                            res["dqn"][w, rr + i, h] = states[B] @ don[w, rr + i, h] * s
                        for i in range(B - 1, -1, -1):
                            dkk, dvv, dgg, dbb, Lt = step_grads(Lt, states[i], kn[w, rr + i, h], vn[w, rr + i, h],
                                                                gn[w, rr + i, h], betan[w, rr + i, h])
                            res["dkn"][w, rr + i, h] = dkk
                            res["dvn"][w, rr + i, h] = dvv
                            res["dgn"][w, rr + i, h] = dgg
                            res["dbetan"][w, rr + i, h] = dbb
                        total += Lt
                        if p > s0 and rank_rows:
                            for i in range(B):                  # x = A~_1^T ... A~_B^T q~ s
                                xv = qn[w, rr + i, h] * s
                                for j in range(B - 1, -1, -1):
                                    kj = kn[w, rr + j, h]
                                    xv = np.exp(gn[w, rr + j, h]) * (xv - betan[w, rr + j, h] * kj * (kj @ xv))
                                rx.append(xv)
                                rdo.append(don[w, rr + i, h])
                                re_.append(e)
                    if p > s0 and not rank_rows:                # a document's first block starts from zero
                        inject.append((e, total))
                rows = (np.array(rx).reshape(-1, dk), np.array(rdo).reshape(-1, v.shape[2]),
                        np.array(re_, dtype=np.int64)) if rank_rows else None
                gr = _chunk_backward(f, do[a:b, h], lam, s, inject, rows)
                for name in ("dq", "dk", "dv", "dg", "dbeta"):
                    res[name][a:b, h] = gr[name]
                lam = gr["dS0"]
        roff += R
    return res
