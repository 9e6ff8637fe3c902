"""Route I (chunk-then-refine, GDN_ALGO_ROUTE1) against the fp64 oracle, element by element.

The clean pass materialises the state before every response block; each (view, block) is then
refined from its stored state.  Same outputs as the fused kernels by construction (Key design 2
of the FLARE notes: the noisy block starts from S_{e(b-1)} and every position reads the block-end
state); bf16 I/O within 2e-2 max|ref| per tensor, fp32 within 1e-4."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu


def _check(prob, tol):
    out, out_n, fs = b.forward_problem(prob, algo=b.ALGO_ROUTE1)
    torch.cuda.synchronize()
    ref = oracle.forward_problem(prob)
    for name, got in (("out", out), ("out_noisy", out_n), ("final_state", fs)):
        r = ref[name]
        if r.size == 0:
            continue
        err = float(np.max(np.abs(got.double().cpu().numpy() - r)))
        assert err <= tol * max(float(np.max(np.abs(r))), 1e-30), f"{name}: {err:.3e}"


@pytest.mark.parametrize("dtype,d,tol", [("fp32", 32, 1e-4), ("bf16", 64, 2e-2), ("bf16", 128, 2e-2), ("fp32", 128, 1e-4)])
@pytest.mark.parametrize("B", [1, 4, 16, 32])
def test_route1_matches_oracle(dtype, d, tol, B):
    offs = np.array([0, 96 + 2 * B, 96 + 2 * B + 4 * B], np.int32)      # prompts 96 and 0
    prob = synth.make_problem_from_layout(offs, [96, 0], num_heads=2, d_k=d, d_v=d, block_size=B, num_views=2,
                                          dtype=dtype, seed=B + d, device="cuda")
    _check(prob, tol)


@pytest.mark.parametrize("V", [0, 1, 2])
def test_route1_views_and_packed_docs(V):
    offs = np.array([0, 64, 64, 200, 264, 300], np.int32)             # an empty document, unequal lengths
    prob = synth.make_problem_from_layout(offs, [0, 0, 72, 64, 4], num_heads=3, d_k=128, d_v=128, block_size=8,
                                          num_views=V, dtype="bf16", seed=7, device="cuda")
    _check(prob, 2e-2)


def test_route1_long_document_tiles():
    """Several 32-token tiles per document and blocks crossing tile boundaries."""
    offs = np.array([0, 1000], np.int32)
    prob = synth.make_problem_from_layout(offs, [232], num_heads=2, d_k=128, d_v=128, block_size=16, num_views=2,
                                          dtype="bf16", seed=9, device="cuda")
    _check(prob, 2e-2)


@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("V", [1, 3, 8])
def test_route1_tensor_cores_odd_views_and_prompts(B, V):
    """bf16, d = 128, B = 16 / 32: Route I on tensor cores (the chunked kernel exporting the state
    before every response block, then the refine kernel by pairs of views; V odd leaves a pair with
    one view, V = 8 gives four pairs per block).  Prompts that are not whole chunks, an empty response, and few units (split over two
    CTAs)."""
    lens, prompts = [40 + 4 * B, 96 + 6 * B, 72, 3 * B], [40, 96, 72, 0]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    prob = synth.make_problem_from_layout(offs, prompts, num_heads=2, d_k=128, d_v=128, block_size=B, num_views=V,
                                          dtype="bf16", seed=60 + B + V, device="cuda")
    _check(prob, 2e-2)


@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("V", [1, 2])
def test_route1_tensor_cores_shortconv(B, V):
    """Route I on tensor cores with the width-4 ShortConv (Key design 3 of the FLARE notes): the
    conv pass writes the convolved inputs into the workspace, then both stages run on them.
    Prompts of every kind, so that noisy taps before a block start read clean raw inputs and no
    tap crosses a document start."""
    lens, prompts = [40 + 4 * B, 2 * B, 96 + 3 * B], [40, 0, 96]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    prob = synth.make_problem_from_layout(offs, prompts, num_heads=2, d_k=128, d_v=128, block_size=B, num_views=V,
                                          dtype="bf16", conv_width=4, seed=80 + B + V, device="cuda")
    _check(prob, 2e-2)


@pytest.mark.parametrize("wl", ["train_8x4096_h16_d128_B16", "train_8x4096_h16_d128_B32",
                                "conv_4x8192_h16_d128_B16", "conv_4x8192_h16_d128_B32"])
def test_route1_tensor_cores_match_fused_kernel_full_size(wl):
    """The full training and ShortConv shapes: Route I on tensor cores against the fused chunked
    kernel (both checked against the oracle elsewhere), every output element, within the bf16
    bar."""
    prob = synth.make_problem(wl, device="cuda")
    r1 = b.forward_problem(prob, algo=b.ALGO_ROUTE1)
    r2 = b.forward_problem(prob, algo=b.ALGO_CHUNKED)
    torch.cuda.synchronize()
    for name, x, y in zip(("out", "out_noisy", "final_state"), r1, r2):
        scale = float(y.abs().max())
        err = float((x.float() - y.float()).abs().max())
        assert err <= 2e-2 * scale, f"{name}: {err:.3e} vs {scale:.3e}"
