"""Pins of the fp64 attention oracle (oracle/attention.py) against facts that do not come from the
oracle itself: closed forms of the softmax, invariants of the mask the FLARE notes describe
(Method > Overall framework, Key design 1), and planted mistakes that the pins must catch."""
import os
import types

import numpy as np
import pytest

from oracle import attention as oa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def layout(lens, prompts):
    offs = np.zeros(len(lens) + 1, np.int64)
    offs[1:] = np.cumsum(lens)
    return offs, np.asarray(prompts, np.int64)


def draw(lens, prompts, H=2, Hkv=2, d=8, V=2, seed=0):
    rng = np.random.default_rng(seed)
    offs, pl = layout(lens, prompts)
    T, TR = int(offs[-1]), int(sum(lens) - sum(prompts))
    x = lambda *s: rng.standard_normal(s)
    return dict(q=x(T, H, d), k=x(T, Hkv, d), v=x(T, Hkv, d), qn=x(V, TR, H, d), kn=x(V, TR, Hkv, d),
                vn=x(V, TR, Hkv, d), doc_offsets=offs, prompt_len=pl)


def run(inp, B, mod=oa):
    return mod.dual_attention(inp["q"], inp["k"], inp["v"], inp["qn"], inp["kn"], inp["vn"],
                              inp["doc_offsets"], inp["prompt_len"], B)


CASES = [([12, 20, 9], [4, 0, 1], 4), ([16, 8], [8, 8], 2), ([10], [3], 1), ([24, 7], [8, 3], 4)]


def _pin_zero_query_is_mean(mod):
    for lens, prompts, B in CASES:
        inp = draw(lens, prompts, seed=1)
        inp["q"][:] = 0.0
        inp["qn"][:] = 0.0
        out, outn = run(inp, B, mod)
        offs, pl = inp["doc_offsets"], inp["prompt_len"]
        roff = 0
        for n in range(len(lens)):
            s, e = offs[n], offs[n + 1]
            for p in range(s, e):
                np.testing.assert_allclose(out[p], inp["v"][s:p + 1].mean(axis=0), rtol=1e-12, atol=1e-12)
            R = lens[n] - prompts[n]
            for r in range(R):
                b0 = (r // B) * B
                for w in range(inp["qn"].shape[0]):
                    vis = np.concatenate([inp["v"][s:s + prompts[n] + b0], inp["vn"][w, roff + b0:roff + b0 + B]])
                    np.testing.assert_allclose(outn[w, roff + r], vis.mean(axis=0), rtol=1e-12, atol=1e-12)
            roff += R


def _pin_block1_noisy_equals_clean(mod):
    for lens, prompts, _ in CASES:
        inp = draw(lens, prompts, seed=2, V=1)
        offs, pl = inp["doc_offsets"], inp["prompt_len"]
        roff = 0
        for n in range(len(lens)):
            s, P, R = offs[n], prompts[n], lens[n] - prompts[n]
            for name, cn in (("qn", "q"), ("kn", "k"), ("vn", "v")):
                inp[name][0, roff:roff + R] = inp[cn][s + P:s + P + R]
            roff += R
        out, outn = run(inp, 1, mod)
        roff = 0
        for n in range(len(lens)):
            s, P, R = offs[n], prompts[n], lens[n] - prompts[n]
            np.testing.assert_allclose(outn[0, roff:roff + R], out[s + P:s + P + R], rtol=1e-12, atol=1e-12)
            roff += R


def _pin_isolation(mod):
    lens, prompts, B = [24, 7], [8, 3], 4
    inp = draw(lens, prompts, seed=3)
    out, outn = run(inp, B, mod)
    # block 2 of document 0 starts at clean position 8 + 8 = 16: later clean tokens are invisible
    b = dict(inp)
    for name in ("q", "k", "v"):
        b[name] = inp[name].copy()
        b[name][16:24] += 5.0
    _, outn2 = run(b, B, mod)
    np.testing.assert_allclose(outn2[:, 8:12], outn[:, 8:12], rtol=0, atol=1e-13)
    # other blocks, the other view and the other document's noisy rows are invisible
    c = dict(inp)
    for name in ("qn", "kn", "vn"):
        c[name] = inp[name].copy()
        c[name][0, 0:8] += 3.0          # blocks 0, 1 of view 0
        c[name][1, 8:12] += 3.0         # block 2 of view 1
        c[name][0, 16:20] += 3.0        # document 1
    out3, outn3 = run(c, B, mod)
    np.testing.assert_allclose(outn3[0, 8:16], outn[0, 8:16], rtol=0, atol=1e-13)
    np.testing.assert_allclose(out3, out, rtol=0, atol=0)
    # documents do not see each other: the second document alone gives the same rows
    one = draw([7], [3], seed=4)
    for name in ("q", "k", "v"):
        one[name] = inp[name][24:31]
    for name in ("qn", "kn", "vn"):
        one[name] = inp[name][:, 16:20]
    o1, on1 = run(one, B, mod)
    np.testing.assert_allclose(o1, out[24:31], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(on1, outn[:, 16:20], rtol=1e-13, atol=1e-13)


def _pin_permutation_inside_block(mod):
    lens, prompts, B = [12, 20, 9], [4, 0, 1], 4
    inp = draw(lens, prompts, seed=5)
    out, outn = run(inp, B, mod)
    perm = np.array([2, 0, 3, 1])
    p = dict(inp)
    for name in ("qn", "kn", "vn"):
        p[name] = inp[name].copy()
        p[name][1, 12:16] = inp[name][1, 12 + perm]     # document 1, block 1, view 1
    _, outn2 = run(p, B, mod)
    np.testing.assert_allclose(outn2[1, 12:16], outn[1, 12 + perm], rtol=1e-12, atol=1e-13)


def _pin_first_token_and_shift(mod):
    lens, prompts, B = [12, 20, 9], [4, 0, 1], 4
    inp = draw(lens, prompts, seed=6, H=4, Hkv=2)
    out, outn = run(inp, B, mod)
    for n, s in enumerate(inp["doc_offsets"][:-1]):
        for h in range(4):     # a document's first token sees only itself (grouped key/value heads)
            np.testing.assert_allclose(out[s, h], inp["v"][s, h // 2], rtol=1e-13, atol=1e-13)
    # a key offset u shifts every score of a query by q.u: the softmax does not move
    sh = dict(inp)
    u = np.random.default_rng(7).standard_normal(inp["k"].shape[2])
    sh["k"] = inp["k"] + u
    sh["kn"] = inp["kn"] + u
    o2, on2 = run(sh, B, mod)
    np.testing.assert_allclose(o2, out, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(on2, outn, rtol=1e-10, atol=1e-10)


def _pin_two_key_weights(mod):
    """Second token of a document, d = 4: k_0 = 0 and q.k_1 = 2 ln 3, so with the 1/sqrt(d) scale
    the scores are 0 and ln 3, the weights 1/4 and 3/4: o = (v_0 + 3 v_1) / 4.  The noisy query
    of a one-token prompt with B = 1 and the same keys sees the same two keys."""
    inp = draw([2], [1], H=1, Hkv=1, d=4, V=1, seed=9)
    inp["k"][0, 0] = 0.0
    inp["k"][1, 0] = np.array([2.0, 0.0, 0.0, 0.0])
    inp["q"][1, 0] = np.array([np.log(3.0), 0.0, 0.0, 0.0])
    inp["kn"][0, 0, 0] = inp["k"][1, 0]
    inp["qn"][0, 0, 0] = inp["q"][1, 0]
    out, outn = run(inp, 1, mod)
    expect = (inp["v"][0, 0] + 3.0 * inp["v"][1, 0]) / 4.0
    np.testing.assert_allclose(out[1, 0], expect, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(outn[0, 0, 0], (inp["v"][0, 0] + 3.0 * inp["vn"][0, 0, 0]) / 4.0,
                               rtol=1e-14, atol=1e-14)


PINS = [_pin_two_key_weights, _pin_zero_query_is_mean, _pin_block1_noisy_equals_clean, _pin_isolation,
        _pin_permutation_inside_block, _pin_first_token_and_shift]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__[5:] for p in PINS])
def test_oracle_pins(pin):
    pin(oa)


def test_rows_entry_point_matches_full():
    lens, prompts, B = [24, 7, 13], [8, 3, 1], 4
    inp = draw(lens, prompts, seed=8, H=4, Hkv=1)
    out, outn = run(inp, B)
    cr = [(0, 0), (5, 3), (23, 1), (24, 2), (30, 3), (31, 0), (43, 2)]
    nr = [(0, 0, 0), (1, 15, 3), (0, 16, 1), (1, 19, 2), (0, 20, 0), (1, 31, 3)]
    c, nn = oa.dual_attention_rows(inp["q"], inp["k"], inp["v"], inp["qn"], inp["kn"], inp["vn"],
                                   inp["doc_offsets"], inp["prompt_len"], B, cr, nr)
    for (p, h), x in zip(cr, c):
        np.testing.assert_allclose(x, out[p, h], rtol=1e-12, atol=1e-13)
    for (w, r, h), x in zip(nr, nn):
        np.testing.assert_allclose(x, outn[w, r, h], rtol=1e-12, atol=1e-13)


def _mutant(old, new):
    src = open(os.path.join(ROOT, "oracle", "attention.py")).read()
    assert old in src
    mod = types.ModuleType("attention_mutant")
    exec(compile(src.replace(old, new), "attention_mutant", "exec"), mod.__dict__)
    return mod


MUTANTS = {
    "prefix one token too long": ("pre = P + b0 ", "pre = P + b0 + 1 "),
    "clean stream not causal": ("S[np.triu_indices(L, 1)] = -np.inf", "pass"),
    "clean stream strictly causal": ("np.triu_indices(L, 1)", "np.triu_indices(L, 0)"),
    "noisy block sees the clean block": ("Kc = np.concatenate([k[s:s + pre, hk]", "Kc = np.concatenate([k[s:s + pre + B, hk]"),
    "no 1/sqrt(d)": ("scale = 1.0 / np.sqrt(d)\n    out", "scale = 1.0\n    out"),
    "wrong key head": ("hk = h // grp\n            if L", "hk = h % Hkv\n            if L"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name):
    old, new = MUTANTS[name]
    mod = _mutant(old, new)
    caught = 0
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin catches the mutant '{name}'"
