"""The chunked (WY / UT) backward of the clean stream (tests/chunk_backward_reference.py, the
derivation a tensor-core backward would use) against the token-by-token fp64 backward oracle."""
import numpy as np
import pytest

from oracle import backward as ob
import chunk_backward_reference as cbr


@pytest.mark.parametrize("C", [16, 64])
@pytest.mark.parametrize("lens", [[150, 70], [64, 1, 129]])
def test_chunked_clean_backward_matches_the_oracle(C, lens):
    rng = np.random.default_rng(C + len(lens))
    H, d = 2, 8
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(offs[-1])
    unit = lambda a: a / np.linalg.norm(a, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((T, H, d))), unit(rng.standard_normal((T, H, d)))
    v = rng.standard_normal((T, H, d))
    g = -0.5 * rng.random((T, H))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    do = rng.standard_normal((T, H, d))
    dsf = rng.standard_normal((len(lens), H, d, d))
    prompts = np.asarray(lens, np.int32)                     # no response: clean stream only
    e = np.zeros((0, 0, H, d))
    e1 = np.zeros((0, 0, H))
    ref = ob.dual_backward(q, k, v, g, beta, e, e, e, e1, e1, offs, prompts, 1, do, e, dsf)
    got = cbr.clean_backward_chunked(q, k, v, g, beta, offs, do, dsf, C=C)
    for name in ("dq", "dk", "dv", "dg", "dbeta"):
        r = ref[name]
        assert np.abs(got[name] - r).max() <= 1e-10 * max(np.abs(r).max(), 1.0), name


@pytest.mark.parametrize("C,B", [(16, 4), (64, 4), (64, 16), (16, 1)])
def test_chunked_dual_backward_matches_the_oracle(C, B):
    """Both streams: the noisy blocks' initial-state gradients enter the chunk backward at their
    boundary states (prompts not on the chunk grid, an empty prompt, two views)."""
    rng = np.random.default_rng(C + B)
    H, d, V = 2, 6, 2
    R = lambda x: (x // B) * B
    lens = [21 + R(80), R(48), 13 + R(16)]
    prompts = [21, 0, 13]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, TR = int(offs[-1]), int(sum(lens) - sum(prompts))
    unit = lambda a: a / np.linalg.norm(a, axis=-1, keepdims=True)
    x = lambda *sh: rng.standard_normal(sh)
    ins = dict(q=unit(x(T, H, d)), k=unit(x(T, H, d)), v=x(T, H, d), g=-0.4 * rng.random((T, H)),
               beta=1 / (1 + np.exp(-x(T, H))), qn=unit(x(V, TR, H, d)), kn=unit(x(V, TR, H, d)),
               vn=x(V, TR, H, d), gn=-0.4 * rng.random((V, TR, H)), betan=1 / (1 + np.exp(-x(V, TR, H))))
    order = ("q", "k", "v", "g", "beta", "qn", "kn", "vn", "gn", "betan")
    do, don, dsf = x(T, H, d), x(V, TR, H, d), x(len(lens), H, d, d)
    ref = ob.dual_backward(*(ins[n] for n in order), offs, prompts, B, do, don, dsf)
    got = cbr.dual_backward_chunked(*(ins[n] for n in order), offs, prompts, B, do, don, dsf, C=C)
    for name in ref:
        r = ref[name]
        assert np.abs(got[name] - r).max() <= 1e-10 * max(np.abs(r).max(), 1.0), name


def test_noisy_injection_is_rank_B_in_carried_back_queries():
    """A block's initial-state gradient sum_l (A~_1^T ... A~_B^T q~_l) do~_l^T / sqrt(d): the
    block's queries carried back through its steps (B rows per view) times their upstream
    gradients, so a kernel can inject it as extra read-out rows instead of a d x d matrix."""
    rng = np.random.default_rng(3)
    d, B = 6, 4
    unit = lambda a: a / np.linalg.norm(a)
    kn = [unit(rng.standard_normal(d)) for _ in range(B)]
    qn = [unit(rng.standard_normal(d)) for _ in range(B)]
    gn = -0.3 * rng.random(B)
    bn = 1 / (1 + np.exp(-rng.standard_normal(B)))
    don = [rng.standard_normal(d) for _ in range(B)]
    s = 1 / np.sqrt(d)
    A = [np.exp(gn[i]) * (np.eye(d) - bn[i] * np.outer(kn[i], kn[i])) for i in range(B)]
    # the adjoint written out: Lam_B = sum_l q_l do_l^T s, Lam_{i-1} = A_i^T Lam_i
    lam = sum(np.outer(qn[l], don[l]) for l in range(B)) * s
    for i in range(B - 1, -1, -1):
        lam = A[i].T @ lam
    # rank-B form: x_l = A_1^T ... A_B^T q_l s
    xs = []
    for l in range(B):
        x = qn[l] * s
        for i in range(B - 1, -1, -1):
            x = A[i].T @ x
        xs.append(x)
    lam_rank = sum(np.outer(xs[l], don[l]) for l in range(B))
    np.testing.assert_allclose(lam_rank, lam, rtol=1e-12, atol=1e-14)
    assert np.linalg.matrix_rank(lam) <= B


@pytest.mark.parametrize("C,B", [(16, 4), (64, 16)])
def test_injection_as_rank_B_rows_matches_the_matrix_form(C, B):
    """The kernel's form of the injection: B carried-back query rows per view and block, read out
    against the chunk like the forward's Z rows, give the same gradients as the d x d matrices."""
    rng = np.random.default_rng(10 + B)
    H, d, V = 1, 6, 2
    R = lambda x: (x // B) * B
    lens = [21 + R(80), R(48)]
    prompts = [21, 0]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, TR = int(offs[-1]), int(sum(lens) - sum(prompts))
    unit = lambda a: a / np.linalg.norm(a, axis=-1, keepdims=True)
    x = lambda *sh: rng.standard_normal(sh)
    ins = (unit(x(T, H, d)), unit(x(T, H, d)), x(T, H, d), -0.4 * rng.random((T, H)), 1 / (1 + np.exp(-x(T, H))),
           unit(x(V, TR, H, d)), unit(x(V, TR, H, d)), x(V, TR, H, d), -0.4 * rng.random((V, TR, H)),
           1 / (1 + np.exp(-x(V, TR, H))))
    do, don, dsf = x(T, H, d), x(V, TR, H, d), x(len(lens), H, d, d)
    a = cbr.dual_backward_chunked(*ins, offs, prompts, B, do, don, dsf, C=C)
    r = cbr.dual_backward_chunked(*ins, offs, prompts, B, do, don, dsf, C=C, rank_rows=True)
    for name in a:
        assert np.abs(a[name] - r[name]).max() <= 1e-11 * max(np.abs(a[name]).max(), 1.0), name
