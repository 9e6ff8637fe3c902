"""GPU parity at the benchmark workloads' full sizes, in the launch configuration bench.py times
(algo auto, one call over all documents and heads).  The oracle recomputes sampled
(document, head) units one by one from the same inputs; each sampled unit's clean outputs,
noisy outputs and final state must be within the bf16 tolerance 2e-2 x max|ref| of that unit.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

WORKLOADS = (["train_8x4096_h16_d128", "packed_32768_h16_d128"]
             + [f"conv_4x8192_h16_d128_B{bs}" for bs in synth.BLOCK_SWEEP]
             + ["large_32x8192_h32_d128"])
TOL = 2e-2


def unit_problem(prob, n, h):
    s0, s1 = int(prob.doc_offsets[n]), int(prob.doc_offsets[n + 1])
    roff = prob.response_offsets()
    r0, r1 = int(roff[n]), int(roff[n + 1])
    d = prob.d_k
    cut = lambda t: t[s0:s1, h:h + 1].cpu()
    cutn = lambda t: t[:, r0:r1, h:h + 1].cpu()
    conv = None if prob.conv_w is None else prob.conv_w[:, h * d:(h + 1) * d, :].cpu()
    args = (cut(prob.q), cut(prob.k), cut(prob.v), cut(prob.g), cut(prob.beta),
            cutn(prob.qn), cutn(prob.kn), cutn(prob.vn), cutn(prob.gn), cutn(prob.betan),
            [0, s1 - s0], [int(prob.prompt_len[n])], prob.block_size)
    return args, conv, (s0, s1, r0, r1)


def rel(got, ref):
    return float(np.max(np.abs(got - ref))) / max(float(np.max(np.abs(ref))), 1e-30) if ref.size else 0.0


@pytest.mark.parametrize("name", WORKLOADS)
def test_full_size_sampled_units(name):
    prob = synth.make_problem(name, device="cuda")
    out, out_n, fs = b.forward_problem(prob)
    torch.cuda.synchronize()
    N, H = prob.num_docs, prob.num_heads
    rng = np.random.default_rng(0)
    units = sorted({(0, 0), (N - 1, H - 1)} | {(int(rng.integers(N)), int(rng.integers(H))) for _ in range(4)})
    jobs = []
    for n, h in units:
        args, conv, (s0, s1, r0, r1) = unit_problem(prob, n, h)
        jobs.append((n, h, args, conv, out[s0:s1, h].double().cpu().numpy(),
                     out_n[:, r0:r1, h].double().cpu().numpy(), fs[n, h].double().cpu().numpy()))

    def run(job):
        n, h, args, conv, o, on, f = job
        ref = oracle.forward(*args, conv_w=conv, num_threads=1)
        return (n, h, rel(o, ref["out"][:, 0]), rel(on, ref["out_noisy"][:, :, 0]), rel(f, ref["final_state"][0, 0]))

    with ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        results = list(ex.map(run, jobs))
    bad = [r for r in results if max(r[2:]) > TOL]
    assert not bad, bad


def test_maximum_document_count():
    """1024 documents (the per-call maximum), each one prompt token block plus one response block."""
    N = 1024
    offs = np.arange(0, 8 * (N + 1), 8, dtype=np.int32)
    prob = synth.make_problem_from_layout(offs, [4] * N, num_heads=1, d_k=32, d_v=32, block_size=4,
                                          num_views=2, dtype="fp32", seed=3, device="cuda")
    out, out_n, fs = b.forward_problem(prob)
    torch.cuda.synchronize()
    ref = oracle.forward_problem(prob)
    assert rel(out.double().cpu().numpy(), ref["out"]) <= 1e-4
    assert rel(out_n.double().cpu().numpy(), ref["out_noisy"]) <= 1e-4
    assert rel(fs.double().cpu().numpy(), ref["final_state"]) <= 1e-4
