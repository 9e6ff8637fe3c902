"""Backward pass (gdn_dual_backward) against the fp64 backward oracle, element by element.

Both sides see the same I/O-rounded inputs; the GPU computes in fp32, so every gradient tensor
must agree to 1e-4 max|ref| (the fp32 bar of the forward) for fp32 and bf16 I/O alike."""
import numpy as np
import pytest
import torch

from oracle import backward as ob
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 1e-4
GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dqn", "dkn", "dvn", "dgn", "dbetan")


def problem(lens, prompts, B, d=64, H=2, V=2, dtype="fp32", seed=0, g_lo=-0.1, conv=0):
    offs = np.zeros(len(lens) + 1, np.int32)
    offs[1:] = np.cumsum(lens)
    return synth.make_problem_from_layout(offs, prompts, num_heads=H, d_k=d, d_v=d, block_size=B, num_views=V,
                                          dtype=dtype, seed=seed, g_lo=g_lo, conv_width=conv, device="cuda")


def upstream(pr, seed, final=True):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    x = lambda *s: torch.randn(*s, generator=gen, device="cuda").to(pr.q.dtype)
    do = x(*pr.q.shape[:2], pr.v.shape[2])
    don = x(pr.qn.shape[0], pr.qn.shape[1], pr.q.shape[1], pr.v.shape[2])
    dsf = torch.randn(pr.num_docs, pr.num_heads, pr.d_k, pr.d_v, generator=gen, device="cuda") if final else None
    return do, don, dsf


def check(pr, seed=1, final=True):
    do, don, dsf = upstream(pr, seed, final)
    got = b.backward(pr.q, pr.k, pr.v, pr.g, pr.beta, pr.qn, pr.kn, pr.vn, pr.gn, pr.betan, pr.doc_offsets,
                     pr.prompt_len, pr.block_size, do, don, dsf, conv_w=pr.conv_w)
    torch.cuda.synchronize()
    if pr.conv_w is None:
        ref = ob.dual_backward(pr.q, pr.k, pr.v, pr.g, pr.beta, pr.qn, pr.kn, pr.vn, pr.gn, pr.betan,
                               pr.doc_offsets, pr.prompt_len, pr.block_size, do, don, dsf)
    else:
        ref = ob.dual_backward_conv(pr.q, pr.k, pr.v, pr.g, pr.beta, pr.qn, pr.kn, pr.vn, pr.gn, pr.betan,
                                    pr.doc_offsets, pr.prompt_len, pr.block_size, pr.conv_w, do, don, dsf)
    errs = {}
    for n in GRADS + (("dconv_w",) if pr.conv_w is not None else ()):
        r = ref[n]
        if r.size == 0:
            continue
        e = float(np.abs(got[n].double().cpu().numpy() - r).max() / max(np.abs(r).max(), 1e-30))
        errs[n] = e
    assert all(e <= TOL for e in errs.values()), errs
    return errs


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_head_dims_and_dtypes(d, dtype):
    """Several 16-token checkpoint segments with ragged ends, a prompt, an empty prompt, a
    prompt-only document."""
    check(problem([37, 68, 20], [5, 0, 20], 4, d=d, dtype=dtype, seed=d))


@pytest.mark.parametrize("B", [1, 2, 8, 16, 32])
def test_block_sizes(B):
    check(problem([37, 71, 20], [5, 7, 20], B, seed=B))


@pytest.mark.parametrize("V", [0, 1, 3])
def test_view_counts(V):
    check(problem([40, 33], [8, 1], 4, V=V, seed=10 + V))


def test_without_final_state_gradient_and_strong_gates():
    check(problem([50, 29], [10, 1], 4, seed=20, g_lo=-1.0), final=False)


@pytest.mark.parametrize("name", ["train_8x4096_h16_d128"])
def test_full_size_sampled_units(name):
    """The training workload at full size: two (document, head) units recomputed by the oracle
    on their own (documents and heads are independent)."""
    pr = synth.make_problem(name, seed=2, device="cuda")
    do, don, dsf = upstream(pr, 3)
    got = b.backward(pr.q, pr.k, pr.v, pr.g, pr.beta, pr.qn, pr.kn, pr.vn, pr.gn, pr.betan, pr.doc_offsets,
                     pr.prompt_len, pr.block_size, do, don, dsf)
    torch.cuda.synchronize()
    offs = pr.doc_offsets.astype(np.int64)
    roffs = pr.response_offsets()
    for n, h in ((0, 0), (pr.num_docs - 1, pr.num_heads - 1)):
        s, e, r0, r1 = int(offs[n]), int(offs[n + 1]), int(roffs[n]), int(roffs[n + 1])
        sl = lambda t: t[s:e, h:h + 1].cpu()
        sn = lambda t: t[:, r0:r1, h:h + 1].cpu()
        ref = ob.dual_backward(sl(pr.q), sl(pr.k), sl(pr.v), sl(pr.g), sl(pr.beta), sn(pr.qn), sn(pr.kn), sn(pr.vn),
                               sn(pr.gn), sn(pr.betan), [0, e - s], pr.prompt_len[n:n + 1], pr.block_size,
                               sl(do), sn(don), dsf[n:n + 1, h:h + 1].cpu())
        for g_ in GRADS:
            noisy = g_ in ("dqn", "dkn", "dvn", "dgn", "dbetan")
            mine = got[g_][:, r0:r1, h:h + 1] if noisy else got[g_][s:e, h:h + 1]
            r = ref[g_]
            err = float(np.abs(mine.double().cpu().numpy() - r).max() / max(np.abs(r).max(), 1e-30))
            assert err <= TOL, (n, h, g_, err)


def test_invalid_arguments():
    pr = problem([40, 33], [8, 1], 4, seed=30)
    do, don, dsf = upstream(pr, 4)
    with pytest.raises(b.GdnError) as e:       # a negative prompt length (same total of responses)
        b.backward(pr.q, pr.k, pr.v, pr.g, pr.beta, pr.qn, pr.kn, pr.vn, pr.gn, pr.betan, pr.doc_offsets,
                   [10, -1], 4, do, don, dsf)
    assert e.value.status == b.GDN_ERR_INVALID_ARG


@pytest.mark.parametrize("B", [1, 4, 8, 32])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_shortconv_backward(B, dtype):
    """gdn_dual_backward_conv against the oracle's conv backward (Key design 3): ragged documents, a
    prompt shorter than the conv, an empty prompt (the first block's taps before the document read
    nothing), a prompt-only document; gradients of the raw inputs and of the weights."""
    R = lambda r: (r // B) * B
    lens = [2 + R(40), 69 + R(3), 20]
    prompts = [2, 5, 20]
    lens[1] = 5 + R(64)
    check(problem(lens, prompts, B, d=64, dtype=dtype, seed=40 + B, conv=4))


@pytest.mark.parametrize("conv", [0, 4])
def test_backward_is_deterministic(conv):
    """Two calls on the same inputs give bit-identical gradients (no atomics: per-slice partials
    added in a fixed order)."""
    pr = problem([200, 136], [72, 8], 4, d=128, dtype="bf16", seed=50 + conv, conv=conv)
    do, don, dsf = upstream(pr, 5)
    run = lambda: b.backward(pr.q, pr.k, pr.v, pr.g, pr.beta, pr.qn, pr.kn, pr.vn, pr.gn, pr.betan, pr.doc_offsets,
                             pr.prompt_len, pr.block_size, do, don, dsf, conv_w=pr.conv_w)
    a = {n: t.clone() for n, t in run().items()}
    c = run()
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n], c[n]), n
