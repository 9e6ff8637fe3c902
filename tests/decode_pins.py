"""Pins for the oracle's decode-side steps (test code only).

The serving paragraph of "FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes)
describes two decode-side state operations on top of the gated delta rule of Key design 2:
Diffusion-Trust commits a finished block with one causal replay that writes the block's final
state into the state pool, and AR-Trust's verify forward keeps the state after every candidate
step so that accepting the first r candidates is a gather of the r-th state (Cache-and-Scatter).

Each pin takes `steps(S0, q, k, v, g, beta, record_states)` (the function under test, with the
signature of oracle.decode_steps) and checks it against something other than itself: the pinned
forward oracle, explicit d x d matrix products, or the split-and-resume identity.
"""
from __future__ import annotations

import numpy as np

import brute


def rand_decode(rng, N=3, L=6, H=2, dk=8, dv=8, g_lo=-0.4, s0_scale=0.5):
    """Seeded decode inputs (fp64): a non-zero starting state per (sequence, head) and L tokens."""
    q = brute.unit_rows(rng.standard_normal((N, L, H, dk)))
    k = brute.unit_rows(rng.standard_normal((N, L, H, dk)))
    v = rng.standard_normal((N, L, H, dv))
    g = rng.uniform(g_lo, 0.0, (N, L, H))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((N, L, H))))
    S0 = s0_scale * rng.standard_normal((N, H, dk, dv))
    return S0, q, k, v, g, beta


def pin_d1_zero_state_is_forward(steps, fwd):
    """From a zero state the steps are the clean stream of the pinned forward oracle run on each
    sequence as one document of L prompt tokens (no response, no noisy view)."""
    rng = np.random.default_rng(101)
    S0, q, k, v, g, beta = rand_decode(rng)
    S0[:] = 0.0
    N, L, H, dk = q.shape
    dv = v.shape[3]
    res = steps(S0, q, k, v, g, beta, True)
    offs = np.arange(N + 1, dtype=np.int32) * L
    empty = lambda d: np.zeros((0, 0, H, d))
    ref = fwd(q.reshape(N * L, H, dk), k.reshape(N * L, H, dk), v.reshape(N * L, H, dv),
              g.reshape(N * L, H), beta.reshape(N * L, H), empty(dk), empty(dk), empty(dv),
              np.zeros((0, 0, H)), np.zeros((0, 0, H)), offs, np.full(N, L, dtype=np.int32), 4)
    assert np.allclose(res["out"].reshape(N * L, H, dv), ref["out"], rtol=0, atol=1e-12)
    assert np.allclose(res["final_state"], ref["final_state"], rtol=0, atol=1e-12)


def pin_d2_brute_force_from_state(steps, fwd=None):
    """With a non-zero starting state S0, explicit matrix products give every step:
    S_t = (A_t ... A_1) S0 + sum_{i<=t} (A_t ... A_{i+1}) beta_i k_i v_i^T,  A_j = alpha_j (I - beta_j k_j k_j^T),
    o_t = S_t^T q_t / sqrt(d_k)."""
    rng = np.random.default_rng(102)
    S0, q, k, v, g, beta = rand_decode(rng, N=2, L=5, H=2, dk=6, dv=5)
    res = steps(S0, q, k, v, g, beta, True)
    N, L, H, dk = q.shape
    for n in range(N):
        for h in range(H):
            As = [brute.transition(np.exp(g[n, t, h]), beta[n, t, h], k[n, t, h]) for t in range(L)]
            for t in range(L):
                M = np.eye(dk)
                for j in range(t, -1, -1):
                    M = M @ As[j]
                S = M @ S0[n, h]
                for i in range(t + 1):
                    M = np.eye(dk)
                    for j in range(t, i, -1):
                        M = M @ As[j]
                    S = S + M @ (beta[n, i, h] * np.outer(k[n, i, h], v[n, i, h]))
                assert np.allclose(res["states"][n, t, h], S, rtol=0, atol=1e-12)
                o = S.T @ q[n, t, h] / np.sqrt(dk)
                assert np.allclose(res["out"][n, t, h], o, rtol=0, atol=1e-12)
            assert np.allclose(res["final_state"][n, h], res["states"][n, L - 1, h], rtol=0, atol=0)


def pin_d3_split_and_resume(steps, fwd=None):
    """Running the first a tokens, then resuming from the state they leave, equals one run over
    all L tokens (the pool makes a replay resumable)."""
    rng = np.random.default_rng(103)
    S0, q, k, v, g, beta = rand_decode(rng, N=2, L=7)
    full = steps(S0, q, k, v, g, beta, False)
    for a in (1, 3, 6):
        first = steps(S0, q[:, :a], k[:, :a], v[:, :a], g[:, :a], beta[:, :a], False)
        rest = steps(first["final_state"], q[:, a:], k[:, a:], v[:, a:], g[:, a:], beta[:, a:], False)
        assert np.array_equal(np.concatenate([first["out"], rest["out"]], axis=1), full["out"])
        assert np.array_equal(rest["final_state"], full["final_state"])


def pin_d4_rollback_is_prefix_run(steps, fwd=None):
    """Cache-and-Scatter: the recorded state of step r - 1 is the state a run over only the first
    r candidates leaves, so accepting r candidates commits exactly that run (r = 0 keeps S0)."""
    rng = np.random.default_rng(104)
    S0, q, k, v, g, beta = rand_decode(rng, N=2, L=5)
    rec = steps(S0, q, k, v, g, beta, True)
    for r in range(1, 6):
        pre = steps(S0, q[:, :r], k[:, :r], v[:, :r], g[:, :r], beta[:, :r], False)
        assert np.array_equal(rec["states"][:, r - 1], pre["final_state"])


DECODE_PINS = [pin_d1_zero_state_is_forward, pin_d2_brute_force_from_state, pin_d3_split_and_resume,
               pin_d4_rollback_is_prefix_run]
