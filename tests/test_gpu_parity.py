"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle, element by
element, on the same seeded inputs.  Tolerances (written here, applied per output tensor):
  fp32 I/O: max|gpu - ref| <= 1e-4 * max|ref|
  bf16 I/O: max|gpu - ref| <= 2e-2 * max|ref|   (fp32 accumulation and fp32 state)
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}
ALGOS = {"seq": b.ALGO_SEQUENTIAL, "auto": b.ALGO_AUTO}


def rel_err(got, ref):
    got = got.detach().double().cpu().numpy() if hasattr(got, "detach") else got
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref))) / max(scale, 1e-30)


def check(prob, dtype, algo=b.ALGO_AUTO, tol=None):
    tol = TOL[dtype] if tol is None else tol
    out, out_noisy, fs = b.forward_problem(prob, algo=algo)
    torch.cuda.synchronize()
    ref = oracle.forward_problem(prob)
    errs = {"out": rel_err(out, ref["out"]), "out_noisy": rel_err(out_noisy, ref["out_noisy"]),
            "final_state": rel_err(fs, ref["final_state"])}
    assert all(e <= tol for e in errs.values()), errs
    return errs


def small(lens, prompts, H=2, d=32, B=4, V=2, dtype="fp32", conv=0, seed=0, g_lo=-0.1, beta_std=1.0):
    offs = np.zeros(len(lens) + 1, np.int32)
    offs[1:] = np.cumsum(lens)
    return synth.make_problem_from_layout(offs, prompts, num_heads=H, d_k=d, d_v=d, block_size=B,
                                          num_views=V, dtype=dtype, conv_width=conv, seed=seed,
                                          g_lo=g_lo, beta_std=beta_std, device="cuda")


@pytest.mark.parametrize("algo", list(ALGOS))
def test_tiny_fp32_workload(algo):
    """The tiny fp32 workload (1 x 64 tokens, H=2, d=32, B=4, 2 views) at 1e-4."""
    prob = synth.make_problem("tiny_fp32_1x64_h2_d32", device="cuda")
    check(prob, "fp32", ALGOS[algo])


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_head_dims_and_dtypes(d, dtype):
    prob = small([136, 72], [40, 0], H=2, d=d, dtype=dtype, seed=d)
    check(prob, dtype, b.ALGO_SEQUENTIAL)


def algos_for(conv):
    """The sequential and the in-order chunked kernels implement bf16 d=128 problems with or without
    the ShortConv prologue; the pipelined chunked kernel without it.  With ShortConv, AUTO (with the
    workspace size the library asks for) runs the conv as a pass of its own, then the chunked kernel."""
    return [b.ALGO_SEQUENTIAL, b.ALGO_CHUNKED] + ([b.ALGO_PIPELINED] if conv == 0 else [b.ALGO_AUTO])


@pytest.mark.parametrize("B", [1, 2, 4, 8, 16, 32])
@pytest.mark.parametrize("conv", [0, 4])
def test_block_sizes_and_conv(B, conv):
    """Ragged prompts (not multiples of 64 or B), several chunks, a partial last chunk, a
    response-only document."""
    lens = [37 + 3 * 64, 2 * 64, 96]
    prompts = [37, 0, 32]
    lens = [p + ((l - p) // B) * B for l, p in zip(lens, prompts)]
    prob = small(lens, prompts, H=3, d=128, B=B, dtype="bf16", conv=conv, seed=B + conv)
    for algo in algos_for(conv):
        check(prob, "bf16", algo)


@pytest.mark.parametrize("V", [0, 1, 3])
def test_view_counts(V):
    prob = small([128, 64], [32, 16], H=2, d=64, V=V, dtype="fp32", seed=V)
    check(prob, "fp32", b.ALGO_AUTO)


@pytest.mark.parametrize("algo", [b.ALGO_CHUNKED, b.ALGO_PIPELINED])
@pytest.mark.parametrize("V", [0, 1, 2])
def test_view_counts_chunked(V, algo):
    prob = small([200, 136], [72, 8], H=2, d=128, V=V, dtype="bf16", seed=20 + V)
    check(prob, "bf16", algo)


@pytest.mark.parametrize("V", [3, 8])
@pytest.mark.parametrize("conv", [0, 4])
def test_more_than_two_views_auto(V, conv):
    """V = 3 and V = 8 (the header's maximum) at bf16, d = 128, algo AUTO: the tensor-core kernel
    is selected and runs the views in pairs."""
    prob = small([200, 136], [72, 8], H=2, d=128, V=V, dtype="bf16", conv=conv, seed=30 + V + conv)
    desc = b.make_desc(prob.num_docs, 2, 128, 128, V, 4, b.GDN_BF16, conv)
    assert b.select_algo(desc) == b.ALGO_CHUNKED
    check(prob, "bf16", b.ALGO_AUTO)
    if conv == 0:
        check(prob, "bf16", b.ALGO_PIPELINED)


@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (32, "fp32")])
def test_all_documents_empty(d, dtype):
    """Every document empty (T = 0 with N x H > 0): GDN_OK and zero final states."""
    prob = small([0, 0, 0], [0, 0, 0], H=2, d=d, dtype=dtype)
    fs = torch.full((3, 2, d, d), float("nan"), device="cuda")
    ws = b.Workspace(256)
    _, _, fs = b.forward_problem(prob, final_state=fs, workspace=ws)
    assert b.read_device_status(ws) == b.GDN_OK
    assert bool((fs == 0).all())


@pytest.mark.parametrize("conv", [0, 4])
def test_packed_documents_with_degenerate_lengths(conv):
    """Packed row with an empty document, a prompt-only document, a response-only document and
    one-block documents."""
    lens = [0, 24, 4, 100, 8, 0, 52]
    prompts = [0, 24, 0, 20, 4, 0, 0]
    prob = small(lens, prompts, H=2, d=128, B=4, dtype="bf16", conv=conv, seed=7)
    for algo in algos_for(conv):
        check(prob, "bf16", algo)


def test_strong_gates_and_large_beta():
    """g ~ U(-0.5, 0), beta = sigmoid(N(0, 2)) as in the large workload, over long chunks."""
    prob = small([512 + 256, 640], [256, 128], H=2, d=128, B=4, dtype="bf16", seed=11, g_lo=-0.5, beta_std=2.0)
    for algo in algos_for(0):
        check(prob, "bf16", algo)


@pytest.mark.parametrize("algo", [b.ALGO_CHUNKED, b.ALGO_PIPELINED])
@pytest.mark.parametrize("B", [4, 16, 32])
def test_extreme_gates_take_the_exact_decay_paths(B, algo):
    """g ~ U(-8, 0): a chunk's cumulative decay leaves the range in which e^{gamma_t - gamma_i}
    factorises as E_t F_i (|gamma| >= 100 in log2 units), so the chunked kernel exponentiates every
    difference (P and A rows, M'_Z and, for B >= 16, the noisy block coefficients)."""
    prob = small([640, 384], [128, 64], H=2, d=128, B=B, dtype="bf16", seed=41 + B, g_lo=-8.0)
    check(prob, "bf16", algo)


@pytest.mark.parametrize("algo", [b.ALGO_CHUNKED, b.ALGO_PIPELINED])
def test_chunked_matches_sequential_kernel(algo):
    """The CUDA kernels agree with each other on a multi-unit problem (all fp32 state)."""
    prob = small([1000, 1536, 520], [232, 512, 8], H=4, d=128, B=4, dtype="bf16", seed=31)
    a = [t.float().clone() for t in b.forward_problem(prob, algo=b.ALGO_SEQUENTIAL)]
    c = [t.float().clone() for t in b.forward_problem(prob, algo=algo)]
    torch.cuda.synchronize()
    for x, y in zip(a, c):
        assert float((x - y).abs().max()) <= 2e-2 * float(x.abs().max())


def test_doc_reset_equivalence_on_gpu():
    """A packed run equals separate runs per document (Key design 3), within tolerance."""
    lens, prompts = [72, 40, 96], [8, 0, 32]
    prob = small(lens, prompts, H=2, d=64, B=4, dtype="fp32", conv=4, seed=3)
    out, out_n, fs = (t.clone() for t in b.forward_problem(prob))
    offs = prob.doc_offsets
    roff = prob.response_offsets()
    for n in range(3):
        s0, s1, r0, r1 = offs[n], offs[n + 1], roff[n], roff[n + 1]
        o1, n1, f1 = b.forward(prob.q[s0:s1].contiguous(), prob.k[s0:s1].contiguous(), prob.v[s0:s1].contiguous(),
                               prob.g[s0:s1].contiguous(), prob.beta[s0:s1].contiguous(),
                               prob.qn[:, r0:r1].contiguous(), prob.kn[:, r0:r1].contiguous(),
                               prob.vn[:, r0:r1].contiguous(), prob.gn[:, r0:r1].contiguous(),
                               prob.betan[:, r0:r1].contiguous(), [0, s1 - s0], [prompts[n]], 4,
                               conv_w=prob.conv_w)
        torch.cuda.synchronize()
        scale = float(out.abs().max())
        assert float((o1 - out[s0:s1]).abs().max()) <= 1e-5 * scale
        assert float((n1 - out_n[:, r0:r1]).abs().max()) <= 1e-5 * max(scale, float(out_n.abs().max()))
        assert float((f1[0] - fs[n]).abs().max()) <= 1e-5 * float(fs.abs().max())


def test_noisy_equal_clean_B1_gives_clean_output():
    """Noisy inputs equal to the clean ones and B = 1: o~ equals o."""
    prob = small([96], [32], H=2, d=128, B=1, dtype="bf16", seed=5)
    for view in range(2):
        prob.qn[view].copy_(prob.q[32:])
        prob.kn[view].copy_(prob.k[32:])
        prob.vn[view].copy_(prob.v[32:])
        prob.gn[view].copy_(prob.g[32:])
        prob.betan[view].copy_(prob.beta[32:])
    out, out_n, _ = b.forward_problem(prob)
    torch.cuda.synchronize()
    for view in range(2):
        err = float((out_n[view].float() - out[32:].float()).abs().max())
        assert err <= 2e-2 * float(out.float().abs().max())


def test_isolation_of_noisy_blocks_on_gpu():
    """o~ of a block ignores clean inputs at or after its start and other blocks' noisy inputs;
    o and final_state ignore all noisy inputs."""
    prob = small([160], [32], H=2, d=128, B=4, dtype="bf16", conv=4, seed=9)
    out0, n0, f0 = (t.clone() for t in b.forward_problem(prob))
    blk_row = 40                                   # response row of the checked block
    start = 32 + blk_row
    gen = torch.Generator(device="cuda").manual_seed(1)
    for t in (prob.q, prob.k, prob.v):
        t[start:] = torch.randn(t[start:].shape, generator=gen, device="cuda").to(t.dtype)
    for t in (prob.qn, prob.kn, prob.vn):
        t[:, :blk_row] = torch.randn(t[:, :blk_row].shape, generator=gen, device="cuda").to(t.dtype)
        t[:, blk_row + 4:] = torch.randn(t[:, blk_row + 4:].shape, generator=gen, device="cuda").to(t.dtype)
    _, n1, _ = b.forward_problem(prob)
    torch.cuda.synchronize()
    scale = float(n0.float().abs().max())
    assert float((n1[:, blk_row:blk_row + 4].float() - n0[:, blk_row:blk_row + 4].float()).abs().max()) <= 1e-3 * scale
    prob2 = small([160], [32], H=2, d=128, B=4, dtype="bf16", conv=4, seed=9)
    for t in (prob2.qn, prob2.kn, prob2.vn):
        t.copy_(torch.randn(t.shape, generator=gen, device="cuda").to(t.dtype))
    o2, _, f2 = b.forward_problem(prob2)
    torch.cuda.synchronize()
    assert torch.equal(o2, out0) and torch.equal(f2, f0)


def test_device_status_ok_after_forward():
    prob = small([64], [32], H=2, d=32, dtype="fp32")
    ws = b.Workspace(256)
    b.forward_problem(prob, workspace=ws)
    assert b.read_device_status(ws) == b.GDN_OK


def test_errors_with_real_tensors_do_not_launch():
    """Invalid arguments with real device tensors: a status code, outputs untouched."""
    dev = "cuda"
    T, H, d, TR = 64, 2, 32, 35          # prompt 29 leaves 35 response tokens: not a multiple of B=2
    mk = lambda *s: torch.randn(*s, device=dev)
    q, k, v = mk(T, H, d), mk(T, H, d), mk(T, H, d)
    g, beta = -mk(T, H).abs(), mk(T, H).sigmoid()
    qn, kn, vn = mk(2, TR, H, d), mk(2, TR, H, d), mk(2, TR, H, d)
    gn, betan = -mk(2, TR, H).abs(), mk(2, TR, H).sigmoid()
    out = torch.full((T, H, d), 7.0, device=dev)
    with pytest.raises(b.GdnError) as e:
        b.forward(q, k, v, g, beta, qn, kn, vn, gn, betan, [0, 64], [29], 2, out=out)
    assert e.value.status == b.GDN_ERR_INVALID_ARG
    sl = lambda t: t[:, :34].contiguous()          # prompt 30: 34 response rows, but an invalid algo
    with pytest.raises(b.GdnError) as e:
        b.forward(q, k, v, g, beta, sl(qn), sl(kn), sl(vn), sl(gn), sl(betan), [0, 64], [30], 2, algo=9, out=out)
    assert e.value.status == b.GDN_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
