"""Pins of the fp64 oracle: properties fixed by the method's definition or by mathematics,
each chosen so that a plausible mistake in the oracle (a dropped term, a wrong sign or
index, a transposed operand, the wrong state read by the noisy stream, a leaking conv tap)
fails at least one of them.  Every pin takes a forward callable with the signature of
``oracle.forward`` so that the planted-mistake test can run the same pins on variants.

Definitions from "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes):
Key design 2 (gated delta rule, noisy block state and block-end readout) and Key
design 3 (ShortConv anti-leak rule, document reset).
"""
from __future__ import annotations

import numpy as np

import brute

ATOL = 1e-11


def _run(fwd, P, **kw):
    return fwd(P["q"], P["k"], P["v"], P["g"], P["beta"], P["qn"], P["kn"], P["vn"], P["gn"],
               P["betan"], P["doc_offsets"], P["prompt_len"], P["block_size"], conv_w=P["conv_w"],
               **kw)


def _close(a, b, tol=ATOL, what=""):
    err = float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0
    assert err <= tol * max(1.0, float(np.max(np.abs(b))) if np.size(b) else 1.0), f"{what}: err {err}"


def pin_p1_identity_span(fwd):
    """alpha=1, beta=0 leaves S unchanged: outputs over the span read the state before it;
    from a zero state everything is zero."""
    rng = np.random.default_rng(1)
    P = brute.rand_problem(rng, [24], [8], H=2, dk=6, dv=5, V=1, B=4)
    a, b = 12, 20
    P["g"][a:b] = 0.0
    P["beta"][a:b] = 0.0
    full = _run(fwd, P)
    # state before the span: the final state of the same document cut at a
    Pc = brute.copy_problem(P)
    Pc["doc_offsets"] = np.array([0, a], np.int32)
    Pc["prompt_len"] = np.array([8], np.int32)
    for key in ("q", "k", "v", "g", "beta"):
        Pc[key] = P[key][:a]
    for key in ("qn", "kn", "vn", "gn", "betan"):
        Pc[key] = P[key][:, :a - 8]
    S_a = _run(fwd, Pc)["final_state"][0]
    for t in range(a, b):
        for h in range(2):
            _close(full["out"][t, h], S_a[h].T @ P["q"][t, h] / np.sqrt(6), what="P1 span")
    Z = brute.copy_problem(P)
    Z["g"][:] = 0.0
    Z["beta"][:] = 0.0
    Z["betan"][:] = 0.0
    r = _run(fwd, Z)
    assert np.all(r["out"] == 0.0) and np.all(r["final_state"] == 0.0) and np.all(r["out_noisy"] == 0.0)


def pin_p2_exact_write(fwd):
    """alpha=1, beta=1, |k|=1: the delta rule writes v at key k, so S_t^T k_t = v_t; with
    q_t = k_t the output is v_t / sqrt(d_k)."""
    rng = np.random.default_rng(2)
    P = brute.rand_problem(rng, [20], [4], H=2, dk=7, dv=3, V=1, B=4)
    P["g"][:] = 0.0
    P["beta"][:] = 1.0
    P["q"] = P["k"].copy()
    r = _run(fwd, P)
    _close(r["out"], P["v"] / np.sqrt(7), tol=1e-12, what="P2")
    # the noisy stream obeys the same rule at the block end: the last token of each block
    Pn = brute.copy_problem(P)
    Pn["gn"][:] = 0.0
    Pn["betan"][:] = 1.0
    Pn["qn"] = Pn["kn"].copy()
    rn = _run(fwd, Pn)
    last = np.arange(3, Pn["qn"].shape[1], 4)
    _close(rn["out_noisy"][:, last], Pn["vn"][:, last] / np.sqrt(7), tol=1e-12, what="P2 noisy")


def pin_p3_orthonormal_keys(fwd):
    """Orthonormal keys k_t = e_{t mod d} (t < d): the erase term never acts, and the rule
    reduces to gated linear attention
    o_t = sum_{i<=t} (prod_{j=i+1..t} alpha_j) beta_i (q_t . k_i) v_i / sqrt(d)."""
    rng = np.random.default_rng(3)
    d, L = 12, 12
    P = brute.rand_problem(rng, [L], [4], H=1, dk=d, dv=4, V=1, B=4, g_lo=-0.7)
    P["k"][:, 0, :] = np.eye(d)[np.arange(L) % d]
    r = _run(fwd, P)
    g, b, q, k, v = P["g"][:, 0], P["beta"][:, 0], P["q"][:, 0], P["k"][:, 0], P["v"][:, 0]
    for t in range(L):
        acc = np.zeros(4)
        for i in range(t + 1):
            acc += np.exp(np.sum(g[i + 1:t + 1])) * b[i] * (q[t] @ k[i]) * v[i]
        _close(r["out"][t, 0], acc / np.sqrt(d), what="P3")


def pin_p4_brute_force(fwd):
    """L <= 16 per document: the oracle equals explicit matrix products (clean outputs, final
    states, noisy block-end states and noisy outputs), over two packed documents, one with an
    empty prompt."""
    rng = np.random.default_rng(4)
    P = brute.rand_problem(rng, [16, 12], [4, 0], H=2, dk=5, dv=4, V=2, B=4, g_lo=-0.8)
    r = _run(fwd, P, return_noisy_state=True)
    bf = brute.forward_brute(P)
    for key in ("out", "final_state", "out_noisy", "noisy_state"):
        _close(r[key], bf[key], what=f"P4 {key}")


def pin_p5_doc_reset(fwd):
    """A packed run equals separate runs per document, bit for bit (Key design 3)."""
    rng = np.random.default_rng(5)
    lens, prompts = [12, 20, 8], [4, 8, 0]
    P = brute.rand_problem(rng, lens, prompts, H=2, dk=6, dv=6, V=2, B=4, conv=4)
    r = _run(fwd, P)
    offs, roff = P["doc_offsets"], brute.response_offsets(P)
    for n in range(3):
        Pn = brute.copy_problem(P)
        s0, s1, r0, r1 = offs[n], offs[n + 1], roff[n], roff[n + 1]
        for key in ("q", "k", "v", "g", "beta"):
            Pn[key] = P[key][s0:s1]
        for key in ("qn", "kn", "vn", "gn", "betan"):
            Pn[key] = P[key][:, r0:r1]
        Pn["doc_offsets"] = np.array([0, s1 - s0], np.int32)
        Pn["prompt_len"] = np.array([prompts[n]], np.int32)
        rn = _run(fwd, Pn)
        assert np.array_equal(rn["out"], r["out"][s0:s1]), "P5 out"
        assert np.array_equal(rn["out_noisy"], r["out_noisy"][:, r0:r1]), "P5 out_noisy"
        assert np.array_equal(rn["final_state"][0], r["final_state"][n]), "P5 final"


def pin_p6_noisy_equals_clean(fwd):
    """Noisy inputs equal to the clean ones: the noisy block-end state is the clean state
    S_{e(b)}, so o~_l = S_{e(b)}^T q_l / sqrt(d) for every l of the block; with B = 1, o~ = o."""
    rng = np.random.default_rng(6)
    for B in (4, 1):
        P = brute.rand_problem(rng, [20], [8], H=2, dk=6, dv=5, V=2, B=B)
        for view in range(2):
            for src, dst in (("q", "qn"), ("k", "kn"), ("v", "vn"), ("g", "gn"), ("beta", "betan")):
                P[dst][view] = P[src][8:]
        r = _run(fwd, P, return_noisy_state=True)
        states = brute.clean_states_brute(P["k"][:, 0], P["v"][:, 0], P["g"][:, 0], P["beta"][:, 0])
        for view in range(2):
            for blk in range(12 // B):
                e = 8 + (blk + 1) * B - 1
                _close(r["noisy_state"][view, blk, 0], states[e], what="P6 state")
                for l in range(B):
                    row = blk * B + l
                    _close(r["out_noisy"][view, row, 0],
                           states[e].T @ P["q"][8 + row, 0] / np.sqrt(6), what="P6 readout")
        if B == 1:
            _close(r["out_noisy"][0], r["out"][8:], what="P6 B=1")


def pin_p7_isolation(fwd):
    """o~ of block b is unchanged by clean inputs at positions >= the block start, by other
    blocks' noisy inputs and by the other view; o and final_state ignore all noisy inputs."""
    rng = np.random.default_rng(7)
    P = brute.rand_problem(rng, [28], [8], H=1, dk=6, dv=6, V=2, B=4, conv=4)
    r0 = _run(fwd, P)
    blk = 2                                   # block rows 8..11 in the response, positions 16..19
    start = 8 + blk * 4
    Q = brute.copy_problem(P)
    for key in ("q", "k", "v", "g", "beta"):
        Q[key][start:] = rng.standard_normal(Q[key][start:].shape)
    for key in ("qn", "kn", "vn", "gn", "betan"):
        Q[key][0, :blk * 4] = rng.standard_normal(Q[key][0, :blk * 4].shape)
        Q[key][0, (blk + 1) * 4:] = rng.standard_normal(Q[key][0, (blk + 1) * 4:].shape)
        Q[key][1] = rng.standard_normal(Q[key][1].shape)
    Q["betan"] = np.abs(Q["betan"]) % 1.0
    Q["beta"] = np.abs(Q["beta"]) % 1.0
    Q["gn"] = -np.abs(Q["gn"])
    Q["g"] = -np.abs(Q["g"])
    r1 = _run(fwd, Q)
    rows = slice(blk * 4, blk * 4 + 4)
    assert np.array_equal(r0["out_noisy"][0, rows], r1["out_noisy"][0, rows]), "P7 noisy block isolation"
    Z = brute.copy_problem(P)
    for key in ("qn", "kn", "vn", "gn", "betan"):
        Z[key] = rng.standard_normal(Z[key].shape)
    Z["betan"] = np.abs(Z["betan"]) % 1.0
    Z["gn"] = -np.abs(Z["gn"])
    r2 = _run(fwd, Z)
    assert np.array_equal(r0["out"], r2["out"]) and np.array_equal(r0["final_state"], r2["final_state"]), \
        "P7 clean ignores noisy"


def pin_p8_conv(fwd):
    """ShortConv: the identity filter w = [0,0,0,1] gives the no-conv result; a random filter
    equals explicit tap matrices applied before a no-conv run (noisy taps before the block
    start read clean raw inputs); noisy = clean inputs gives noisy conv = clean conv."""
    rng = np.random.default_rng(8)
    P = brute.rand_problem(rng, [20, 16], [8, 4], H=2, dk=4, dv=4, V=2, B=4, conv=4)
    Pi = brute.copy_problem(P)
    Pi["conv_w"] = np.zeros_like(P["conv_w"])
    Pi["conv_w"][..., 3] = 1.0
    Pn = brute.copy_problem(P)
    Pn["conv_w"] = None
    a, b = _run(fwd, Pi), _run(fwd, Pn)
    for key in ("out", "out_noisy", "final_state"):
        assert np.array_equal(a[key], b[key]), f"P8 identity {key}"
    c = _run(fwd, P)
    d = _run(fwd, brute.apply_conv_brute(P))
    for key in ("out", "out_noisy", "final_state"):
        _close(c[key], d[key], what=f"P8 taps {key}")
    E = brute.copy_problem(P)
    E["doc_offsets"] = np.array([0, 20], np.int32)
    E["prompt_len"] = np.array([8], np.int32)
    for key in ("q", "k", "v", "g", "beta"):
        E[key] = P[key][:20]
    for view in range(2):
        for src, dst in (("q", "qn"), ("k", "kn"), ("v", "vn"), ("g", "gn"), ("beta", "betan")):
            E[dst] = np.stack([E[src][8:]] * 2)
    re = _run(fwd, E, return_noisy_state=True)
    Ec = brute.apply_conv_brute(E)
    states = brute.clean_states_brute(Ec["k"][:, 1], Ec["v"][:, 1], Ec["g"][:, 1], Ec["beta"][:, 1])
    for blk in range(3):
        _close(re["noisy_state"][1, blk, 1], states[8 + 4 * blk + 3], what="P8 noisy=clean conv")


def pin_p9_linearity_in_v(fwd):
    """For fixed q, k, g, beta the map v -> (o, o~, S) is linear: scaling and superposition
    (clean v and noisy v~ together)."""
    rng = np.random.default_rng(9)
    P = brute.rand_problem(rng, [16, 12], [4, 4], H=2, dk=5, dv=3, V=2, B=4)
    P2 = brute.copy_problem(P)
    P2["v"] = rng.standard_normal(P["v"].shape)
    P2["vn"] = rng.standard_normal(P["vn"].shape)
    Ps = brute.copy_problem(P)
    Ps["v"] = P["v"] + P2["v"]
    Ps["vn"] = P["vn"] + P2["vn"]
    Pc = brute.copy_problem(P)
    Pc["v"] = 2.5 * P["v"]
    Pc["vn"] = 2.5 * P["vn"]
    r1, r2, rs, rc = (_run(fwd, x) for x in (P, P2, Ps, Pc))
    for key in ("out", "out_noisy", "final_state"):
        _close(rs[key], r1[key] + r2[key], tol=1e-12, what=f"P9 sum {key}")
        _close(rc[key], 2.5 * r1[key], tol=1e-12, what=f"P9 scale {key}")


ALL_PINS = [pin_p1_identity_span, pin_p2_exact_write, pin_p3_orthonormal_keys, pin_p4_brute_force,
            pin_p5_doc_reset, pin_p6_noisy_equals_clean, pin_p7_isolation, pin_p8_conv,
            pin_p9_linearity_in_v]


def pin_golden_hand_worked(fwd):
    """The hand-worked fixtures under tests/golden (values derived by hand from the rule)."""
    import json
    import os
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    for name in ("gdr_hand_d2.json", "conv_antileak_hand_d1.json"):
        fx = json.load(open(os.path.join(here, name)))
        arr = lambda key: np.array(fx[key], dtype=np.float64)
        conv = None if fx["conv_w"] is None else arr("conv_w")
        r = fwd(arr("q"), arr("k"), arr("v"), np.log(arr("alpha")), arr("beta"),
                arr("qn"), arr("kn"), arr("vn"), np.log(arr("alphan")), arr("betan"),
                fx["doc_offsets"], fx["prompt_len"], fx["block_size"], conv_w=conv)
        sq = np.sqrt(arr("q").shape[2])
        _close(r["out"] * sq, np.array(fx["expect_times_sqrt_dk"]["out"]), tol=1e-12, what=name)
        _close(r["out_noisy"] * sq, np.array(fx["expect_times_sqrt_dk"]["out_noisy"]), tol=1e-12, what=name)
        _close(r["final_state"], np.array(fx["expect_final_state"]), tol=1e-12, what=name)


ALL_PINS.append(pin_golden_hand_worked)
