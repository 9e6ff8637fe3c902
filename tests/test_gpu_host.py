"""gdn_dual_forward_host (the forward from and to host buffers, document groups pipelined across
the host link) against gdn_dual_forward on device copies of the same inputs: the same kernels run
on each group's documents, so the outputs must be bit-identical; one case also against the fp64
oracle.  Every algorithm family: the chunked kernel (with and without ShortConv), the sequential
kernel, Route I."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "beta", "qn", "kn", "vn", "gn", "betan"]


def _host_run(prob, algo, groups):
    desc = b.make_desc(prob.num_docs, prob.num_heads, prob.d_k, prob.d_v, prob.num_views, prob.block_size,
                       b._dtype_code(prob.q), prob.conv_width, algo)
    host = {n: getattr(prob, n).cpu().pin_memory() for n in NAMES}
    cw = None if prob.conv_w is None else prob.conv_w.cpu().pin_memory()
    T, H, d = prob.q.shape
    V, TR = prob.qn.shape[0], prob.qn.shape[1]
    out = torch.full((T, H, d), float("nan"), dtype=prob.q.dtype).pin_memory()
    outn = torch.full((V, TR, H, d), float("nan"), dtype=prob.q.dtype).pin_memory()
    fs = torch.full((prob.num_docs, H, d, d), float("nan"), dtype=torch.float32).pin_memory()
    nbytes = b.host_staging_size(desc, prob.doc_offsets, prob.prompt_len, groups)
    assert nbytes > 0
    staging = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    st = b.forward_host_raw(desc, *[host[n] for n in NAMES], prob.doc_offsets, prob.prompt_len, cw, out, outn, fs,
                            staging, groups)
    assert st == b.GDN_OK, b.status_string(st)
    torch.cuda.synchronize()
    assert b.read_host_device_status(staging)[0] == b.GDN_OK
    return out, outn, fs


def _same(prob, algo, groups):
    ref = b.forward_problem(prob, algo=algo)
    torch.cuda.synchronize()
    got = _host_run(prob, algo, groups)
    for name, x, y in zip(("out", "out_noisy", "final_state"), got, ref):
        assert torch.equal(x, y.cpu()), f"{name} differs (groups={groups})"
    return got


LENS, PROMPTS = [200, 0, 72, 136, 64, 520], [8, 0, 72, 0, 32, 264]   # an empty and a prompt-only document


@pytest.mark.parametrize("groups", [1, 2, 3, 6, 64])
def test_host_forward_matches_device_forward_chunked(groups):
    offs = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)
    prob = synth.make_problem_from_layout(offs, PROMPTS, num_heads=3, d_k=128, d_v=128, block_size=4, num_views=2,
                                          dtype="bf16", seed=100 + groups, device="cuda")
    _same(prob, b.ALGO_AUTO, groups)


@pytest.mark.parametrize("groups", [2, 4])
def test_host_forward_shortconv(groups):
    offs = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)
    prob = synth.make_problem_from_layout(offs, PROMPTS, num_heads=2, d_k=128, d_v=128, block_size=8, num_views=2,
                                          dtype="bf16", conv_width=4, seed=110 + groups, device="cuda")
    _same(prob, b.ALGO_AUTO, groups)


def test_host_forward_sequential_fp32_against_oracle():
    offs = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)
    prob = synth.make_problem_from_layout(offs, PROMPTS, num_heads=2, d_k=32, d_v=32, block_size=8, num_views=3,
                                          dtype="fp32", seed=120, device="cuda")
    out, outn, fs = _same(prob, b.ALGO_AUTO, 3)
    ref = oracle.forward_problem(prob)
    for name, got in (("out", out), ("out_noisy", outn), ("final_state", fs)):
        r = ref[name]
        err = float(np.max(np.abs(got.double().numpy() - r)))
        assert err <= 1e-4 * max(float(np.max(np.abs(r))), 1e-30), f"{name}: {err:.3e}"


@pytest.mark.parametrize("conv", [0, 4])
def test_host_forward_route1(conv):
    offs = np.concatenate([[0], np.cumsum([96, 160, 64])]).astype(np.int32)
    prob = synth.make_problem_from_layout(offs, [32, 0, 64], num_heads=2, d_k=128, d_v=128, block_size=16,
                                          num_views=2, dtype="bf16", conv_width=conv, seed=130 + conv, device="cuda")
    _same(prob, b.ALGO_ROUTE1, 2)


def test_host_forward_eight_views():
    """Eight views: the chunked path runs one launch per pair of views inside every group."""
    offs = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)
    prob = synth.make_problem_from_layout(offs, PROMPTS, num_heads=2, d_k=128, d_v=128, block_size=4, num_views=8,
                                          dtype="bf16", seed=140, device="cuda")
    _same(prob, b.ALGO_AUTO, 3)


def test_host_forward_empty_documents_and_more_groups_than_documents():
    """Degenerate layouts: every document empty (only the zero final states come back), and more
    groups asked for than there are documents (one document per group)."""
    offs = np.zeros(4, np.int32)
    prob = synth.make_problem_from_layout(offs, [0, 0, 0], num_heads=2, d_k=128, d_v=128, block_size=4,
                                          num_views=2, dtype="bf16", seed=150, device="cuda")
    out, outn, fs = _same(prob, b.ALGO_AUTO, 5)
    assert torch.count_nonzero(fs) == 0
    offs = np.concatenate([[0], np.cumsum([64, 0, 96])]).astype(np.int32)
    prob = synth.make_problem_from_layout(offs, [32, 0, 0], num_heads=2, d_k=128, d_v=128, block_size=8,
                                          num_views=1, dtype="bf16", seed=151, device="cuda")
    _same(prob, b.ALGO_AUTO, 64)


def test_host_forward_full_training_shape():
    """The training shape through the host path in eight groups, bit-identical to the device call."""
    prob = synth.make_problem("train_8x4096_h16_d128", device="cuda")
    _same(prob, b.ALGO_AUTO, 8)
