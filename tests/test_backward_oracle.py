"""Pins of the fp64 backward oracle (oracle/backward.py): every gradient against central finite
differences of the fp64 forward oracle (a different program: the C recurrence), on tiny problems
that cover prompts, empty prompts, several blocks, both views and the final-state gradient; and
planted mistakes that the pin must catch."""
import os
import types

import numpy as np
import pytest

import oracle
from oracle import backward as ob

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NAMES = ("q", "k", "v", "g", "beta", "qn", "kn", "vn", "gn", "betan")


def draw(lens, prompts, B, H=2, d=3, V=2, seed=0):
    rng = np.random.default_rng(seed)
    offs = np.zeros(len(lens) + 1, np.int32)
    offs[1:] = np.cumsum(lens)
    T, TR = int(offs[-1]), int(sum(lens) - sum(prompts))
    x = lambda *s: rng.standard_normal(s)
    unit = lambda a: a / np.linalg.norm(a, axis=-1, keepdims=True)
    inp = dict(q=unit(x(T, H, d)), k=unit(x(T, H, d)), v=x(T, H, d), g=-0.3 * rng.random((T, H)),
               beta=1 / (1 + np.exp(-x(T, H))), qn=unit(x(V, TR, H, d)), kn=unit(x(V, TR, H, d)),
               vn=x(V, TR, H, d), gn=-0.3 * rng.random((V, TR, H)), betan=1 / (1 + np.exp(-x(V, TR, H))))
    up = dict(d_out=x(T, H, d), d_out_noisy=x(V, TR, H, d), d_final_state=x(len(lens), H, d, d))
    return inp, up, offs, np.asarray(prompts, np.int32)


def loss(inp, up, offs, pl, B):
    r = oracle.forward(*(inp[n] for n in NAMES), offs, pl, B)
    return (np.sum(r["out"] * up["d_out"]) + np.sum(r["out_noisy"] * up["d_out_noisy"])
            + np.sum(r["final_state"] * up["d_final_state"]))


def fd_check(mod, lens, prompts, B, seed, eps=1e-6, tol=1e-6):
    inp, up, offs, pl = draw(lens, prompts, B, seed=seed)
    grads = mod.dual_backward(*(inp[n] for n in NAMES), offs, pl, B, up["d_out"], up["d_out_noisy"],
                              up["d_final_state"])
    for n in NAMES:
        x = inp[n]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            keep = x[i]
            x[i] = keep + eps
            lp = loss(inp, up, offs, pl, B)
            x[i] = keep - eps
            lm = loss(inp, up, offs, pl, B)
            x[i] = keep
            fd[i] = (lp - lm) / (2 * eps)
        got = grads["d" + n]
        scale = max(np.abs(fd).max(), 1e-12)
        assert np.abs(got - fd).max() <= tol * scale, f"d{n}: max err {np.abs(got - fd).max():.3e} vs {scale:.3e}"


CASES = [([10, 8], [2, 0], 2), ([9, 8], [5, 4], 4), ([6, 5], [1, 0], 1), ([12], [0], 4)]


@pytest.mark.parametrize("lens,prompts,B", CASES)
def test_gradients_match_finite_differences_of_the_forward_oracle(lens, prompts, B):
    fd_check(ob, lens, prompts, B, seed=len(lens) + B)


def _mutant(old, new):
    src = open(os.path.join(ROOT, "oracle", "backward.py")).read()
    assert old in src, old
    mod = types.ModuleType("backward_mutant")
    exec(compile(src.replace(old, new), "backward_mutant", "exec"), mod.__dict__)
    return mod


MUTANTS = {
    "no injection of the noisy blocks": ("Lam = Lam + _noisy_block(", "_ = Lam + _noisy_block("),
    "adjoint not decayed": ("Lam_prev = a * (Lam - bb * np.outer(kk, kl))", "Lam_prev = Lam - bb * np.outer(kk, kl)"),
    "erase term of dk dropped": ("- a * bb * (Lam @ ks + Sp @ kl)", "- a * bb * (Lam @ ks)"),
    "noisy readout gradient from the wrong state": ("res[\"dqn\"][w, r, h] = states[B] @", "res[\"dqn\"][w, r, h] = states[i] @"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_finite_differences_catch_planted_mistakes(name):
    mod = _mutant(*MUTANTS[name])
    with pytest.raises(AssertionError):
        fd_check(mod, [10, 8], [2, 0], 2, seed=4)


def _conv_fd_check(mod):
    lens, prompts, B = [10, 8], [2, 0], 2
    inp, up, offs, pl = draw(lens, prompts, B, seed=11)
    H, d = inp["q"].shape[1], inp["q"].shape[2]
    w = 0.5 * np.random.default_rng(12).standard_normal((3, H * d, 4))

    def loss_w(inp_, w_):
        r = oracle.forward(*(inp_[n] for n in NAMES), offs, pl, B, conv_w=w_)
        return (np.sum(r["out"] * up["d_out"]) + np.sum(r["out_noisy"] * up["d_out_noisy"])
                + np.sum(r["final_state"] * up["d_final_state"]))

    grads = mod.dual_backward_conv(*(inp[n] for n in NAMES), offs, pl, B, w, up["d_out"], up["d_out_noisy"],
                                   up["d_final_state"])
    eps = 1e-6
    for n, x in [(n, inp[n]) for n in NAMES] + [("conv_w", w)]:
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            keep = x[i]
            x[i] = keep + eps
            lp = loss_w(inp, w)
            x[i] = keep - eps
            lm = loss_w(inp, w)
            x[i] = keep
            fd[i] = (lp - lm) / (2 * eps)
        scale = max(np.abs(fd).max(), 1e-12)
        assert np.abs(grads["d" + n] - fd).max() <= 1e-6 * scale, f"d{n}"


def test_shortconv_mistake_is_caught():
    """Noisy taps that cross the block start into the noisy stream (the leak the anti-leak rule
    forbids) disagree with the finite differences."""
    mod = _mutant("            if src >= b0:", "            if src >= 0:")
    with pytest.raises(AssertionError):
        _conv_fd_check(mod)


def test_shortconv_gradients_match_finite_differences():
    """With the width-4 ShortConv prologue: every input gradient and the weight gradient against
    central differences of the C forward oracle (which convolves internally); with B = 2 every
    noisy position has taps before its block start, which read (and send gradient to) the clean
    raw input."""
    _conv_fd_check(ob)
