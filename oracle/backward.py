"""fp64 CPU oracle for the backward pass of the dual-stream Gated DeltaNet forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline leg
may import this module.  It shares no code with the CUDA library.

What it differentiates ("FLARE: Diffusion for Hybrid Language Model", papernotes.org notes,
Method > Key design 2): per document and head, the clean chain
    S_t = A_t S_{t-1} + beta_t k_t v_t^T,   A_t = alpha_t (I - beta_t k_t k_t^T),  alpha_t = e^{g_t},
    o_t = S_t^T q_t / sqrt(d_k),            S = 0 before the document,
and for every response block b and view the noisy block started from the clean state just
before it, S~_0 = S_{e(b-1)} (zero for the first block of a document without prompt), run over
the block's B noisy tokens with the same rule, every position reading the block-end state:
o~_l = S~_B^T q~_l / sqrt(d_k).  The scalar being differentiated is
    L = sum <do, out> + sum <do~, out_noisy> + sum <dS, final_state>
for given upstream gradients.  The notes' backward injects each noisy block's gradient into the
causal chain; here that is the adjoint recurrence written out: with Lam_t = dL/dS_t,
    Lam_t   = q_t do_t^T / sqrt(d_k) + A_{t+1}^T Lam_{t+1} + sum over views of Lam~_0 of the block
              that starts at t + 1,
    Lam~_B  = sum_l q~_l do~_l^T / sqrt(d_k),   Lam~_{i-1} = A~_i^T Lam~_i,
and, per step with state S_prev before it and Lam after it (A^T = A):
    dv   = beta Lam^T k,
    dk   = beta Lam v - alpha beta (Lam S_prev^T k + S_prev Lam^T k),
    dbeta = k^T Lam v - alpha (k^T S_prev)(Lam^T k),
    dg   = alpha (<Lam, S_prev> - beta (k^T S_prev)(Lam^T k)),
    dq_t = S_t do_t / sqrt(d_k)   (noisy: dq~_l = S~_B do~_l / sqrt(d_k)).
The matrices are formed explicitly in fp64, token by token, in the pages' order; no chunking.
"""
from __future__ import annotations

import numpy as np


def _as64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def dual_backward(q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, block_size,
                  d_out, d_out_noisy, d_final_state=None):
    """Gradients of L with respect to every input, fp64.

    Returns dict(dq, dk, dv, dg, dbeta, dqn, dkn, dvn, dgn, dbetan) with the inputs' shapes."""
    q, k, v, g, beta = (_as64(x) for x in (q, k, v, g, beta))
    qn, kn, vn, gn, betan = (_as64(x) for x in (qn, kn, vn, gn, betan))
    do, don = _as64(d_out), _as64(d_out_noisy)
    dsf = _as64(d_final_state)
    offs = np.asarray(doc_offsets, dtype=np.int64)
    pl = np.asarray(prompt_len, dtype=np.int64)
    T, H, dk_ = q.shape
    dv_ = v.shape[2]
    V = qn.shape[0]
    B = int(block_size)
    sc = 1.0 / np.sqrt(dk_)
    res = {name: np.zeros_like(x) for name, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("dbeta", beta),
                                                    ("dqn", qn), ("dkn", kn), ("dvn", vn), ("dgn", gn),
                                                    ("dbetan", betan))}

    def step(S, kk, vv, gg, bb):
        return np.exp(gg) * (S - bb * np.outer(kk, kk @ S)) + bb * np.outer(kk, vv)

    def step_grads(Lam, Sp, kk, vv, gg, bb):
        """Gradients of one step (state Sp before, Lam = dL/dS after); returns (dk, dv, dg, dbeta, Lam_before)."""
        a = np.exp(gg)
        ks = Sp.T @ kk                    # k^T S_prev  (d_v)
        kl = Lam.T @ kk                   # Lam^T k     (d_v)
        dvv = bb * kl
        dkk = bb * (Lam @ vv) - a * bb * (Lam @ ks + Sp @ kl)
        dbb = kl @ vv - a * (ks @ kl)
        dgg = a * (np.sum(Lam * Sp) - bb * (ks @ kl))
        Lam_prev = a * (Lam - bb * np.outer(kk, kl))
        return dkk, dvv, dgg, dbb, Lam_prev

    roff = 0
    for n in range(len(pl)):
        s, e = int(offs[n]), int(offs[n + 1])
        P, R = int(pl[n]), e - s - int(pl[n])
        for h in range(H):
            # forward: clean states S_t (state after token t), with S before the document = 0
            Ss = np.zeros((e - s + 1, dk_, dv_))          # Ss[i] = state after i tokens of the document
            for i in range(e - s):
                t = s + i
                Ss[i + 1] = step(Ss[i], k[t, h], v[t, h], g[t, h], beta[t, h])
            Lam = np.zeros((dk_, dv_)) if dsf is None else dsf[n, h].copy()
            for i in range(e - s - 1, -1, -1):
                t = s + i
                Lam = Lam + np.outer(q[t, h], do[t, h]) * sc
                res["dq"][t, h] = Ss[i + 1] @ do[t, h] * sc
                # a response block starts right after this token: inject its views' gradients
                # into Lam = dL/dS after token t (the block's initial state)
                rel = i + 1 - P                                # response index of the next token
                if 0 <= rel < R and rel % B == 0:
                    Lam = Lam + _noisy_block(res, Ss[i + 1], qn, kn, vn, gn, betan, don, roff + rel, B, h, sc,
                                             step, step_grads)
                dkk, dvv, dgg, dbb, Lam = step_grads(Lam, Ss[i], k[t, h], v[t, h], g[t, h], beta[t, h])
                res["dk"][t, h] += dkk
                res["dv"][t, h] += dvv
                res["dg"][t, h] += dgg
                res["dbeta"][t, h] += dbb
            if P == 0 and R > 0:
                # first block of a document without prompt: it starts from the hard zero state,
                # whose gradient goes nowhere
                _noisy_block(res, np.zeros((dk_, dv_)), qn, kn, vn, gn, betan, don, roff, B, h, sc, step, step_grads)
        roff += R
    return res


def _noisy_block(res, S0, qn, kn, vn, gn, betan, don, r0, B, h, sc, step, step_grads):
    """Backward of every view of the noisy block whose packed rows are [r0, r0 + B), started
    from S0; accumulates its input gradients and returns the sum over views of dL/dS0."""
    V = qn.shape[0]
    total = np.zeros_like(S0)
    for w in range(V):
        states = [S0]
        for i in range(B):
            r = r0 + i
            states.append(step(states[-1], kn[w, r, h], vn[w, r, h], gn[w, r, h], betan[w, r, h]))
        Lam = np.zeros_like(S0)
        for i in range(B):
            r = r0 + i
            Lam = Lam + np.outer(qn[w, r, h], don[w, r, h]) * sc
            res["dqn"][w, r, h] = states[B] @ don[w, r, h] * sc
        for i in range(B - 1, -1, -1):
            r = r0 + i
            dkk, dvv, dgg, dbb, Lam = step_grads(Lam, states[i], kn[w, r, h], vn[w, r, h], gn[w, r, h],
                                                 betan[w, r, h])
            res["dkn"][w, r, h] += dkk
            res["dvn"][w, r, h] += dvv
            res["dgn"][w, r, h] += dgg
            res["dbetan"][w, r, h] += dbb
        total += Lam
    return total


def _conv_taps(L, P, B, W):
    """Source of every tap of the width-W ShortConv (Key design 3 of the FLARE notes) for one
    document of L tokens with prompt P: tap j of output position i reads position i - j.
    Clean position i: the clean input at i - j, or 0 before the document.  Noisy response
    position r (block start b0 = B floor(r / B)): the noisy input at r - j inside the block,
    else the clean raw input at P + r - j, else 0.  Returns two lists of (out, j, kind, src)
    with kind 'c' (clean source) or 'n' (noisy source)."""
    clean = [(i, j, "c", i - j) for i in range(L) for j in range(W) if i - j >= 0]
    noisy = []
    for r in range(L - P):
        b0 = (r // B) * B
        for j in range(W):
            src = r - j
            if src >= b0:
                noisy.append((r, j, "n", src))
            elif P + src >= 0:
                noisy.append((r, j, "c", P + src))
    return clean, noisy


def dual_backward_conv(q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, block_size, conv_w,
                       d_out, d_out_noisy, d_final_state=None):
    """Gradients with the ShortConv prologue on q, k, v (both streams, the same weights
    conv_w [3, H d, W], tap W-1 = the current token: x'_p = sum_j w[W-1-j] x_{p-j}).  The conv is
    linear: apply it, differentiate the rule with respect to the convolved inputs
    (dual_backward), then send every tap's gradient back to its source (the transposed taps; a
    noisy output's taps before its block start feed the CLEAN raw input) and to its weight.
    Returns dual_backward's dict plus dconv_w."""
    q, k, v, g, beta = (_as64(x) for x in (q, k, v, g, beta))
    qn, kn, vn, gn, betan = (_as64(x) for x in (qn, kn, vn, gn, betan))
    w = _as64(conv_w)
    offs = np.asarray(doc_offsets, dtype=np.int64)
    pl = np.asarray(prompt_len, dtype=np.int64)
    B = int(block_size)
    T, H, d = q.shape
    W = w.shape[-1]
    wr = w.reshape(3, H, d, W)
    ins = {"q": q, "k": k, "v": v}
    noisy_in = {"q": qn, "k": kn, "v": vn}
    conv = {n: np.zeros_like(x) for n, x in ins.items()}
    convn = {n: np.zeros_like(x) for n, x in noisy_in.items()}
    taps = []
    roff = 0
    for n in range(len(pl)):
        s0, L, P = int(offs[n]), int(offs[n + 1] - offs[n]), int(pl[n])
        clean, noisy = _conv_taps(L, P, B, W)
        taps.append((s0, roff, clean, noisy))
        for X, name in enumerate(("q", "k", "v")):
            wx = wr[X]                                           # [H, d, W]
            for (i, j, _, src) in clean:
                conv[name][s0 + i] += wx[..., W - 1 - j] * ins[name][s0 + src]
            for view in range(qn.shape[0]):
                for (r, j, kind, src) in noisy:
                    x_src = noisy_in[name][view, roff + src] if kind == "n" else ins[name][s0 + src]
                    convn[name][view, roff + r] += wx[..., W - 1 - j] * x_src
        roff += L - P
    res = dual_backward(conv["q"], conv["k"], conv["v"], g, beta, convn["q"], convn["k"], convn["v"], gn, betan,
                        doc_offsets, prompt_len, B, d_out, d_out_noisy, d_final_state)
    dw = np.zeros_like(wr)
    grads = {"q": np.zeros_like(q), "k": np.zeros_like(k), "v": np.zeros_like(v)}
    gradsn = {"q": np.zeros_like(qn), "k": np.zeros_like(kn), "v": np.zeros_like(vn)}
    for (s0, roff, clean, noisy) in taps:
        for X, name in enumerate(("q", "k", "v")):
            wx = wr[X]
            dc = res["d" + name]                                 # gradient w.r.t. the convolved clean input
            dn = res["d" + name + "n"]
            for (i, j, _, src) in clean:
                grads[name][s0 + src] += wx[..., W - 1 - j] * dc[s0 + i]
                dw[X, ..., W - 1 - j] += ins[name][s0 + src] * dc[s0 + i]
            for view in range(qn.shape[0]):
                for (r, j, kind, src) in noisy:
                    gout = dn[view, roff + r]
                    if kind == "n":
                        gradsn[name][view, roff + src] += wx[..., W - 1 - j] * gout
                        dw[X, ..., W - 1 - j] += noisy_in[name][view, roff + src] * gout
                    else:
                        grads[name][s0 + src] += wx[..., W - 1 - j] * gout
                        dw[X, ..., W - 1 - j] += ins[name][s0 + src] * gout
    out = dict(res)
    for name in ("q", "k", "v"):
        out["d" + name] = grads[name]
        out["d" + name + "n"] = gradsn[name]
    out["dconv_w"] = dw.reshape(w.shape)
    return out
