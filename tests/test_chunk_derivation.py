"""The chunked WY/UT factorisation used by the tensor-core kernel equals the sequential
oracle (fp64, CPU).  This checks the derivation, not the oracle."""
import numpy as np
import pytest

import brute
import chunk_reference
import oracle
import pins


@pytest.mark.parametrize("B,C", [(4, 8), (2, 8), (8, 16), (1, 4), (4, 4)])
@pytest.mark.parametrize("conv", [0, 4])
def test_chunked_equals_sequential(B, C, conv):
    rng = np.random.default_rng(100 + B * 10 + C + conv)
    # ragged prompts (first chunk partial), response not a multiple of C (last chunk partial),
    # an empty prompt and a response-only tail document
    lens = [37 + (B * 5 - 37 % B) % B + 3 * B, 4 * B, 29 + B * 3]
    prompts = [13, 0, 29]
    lens = [p + ((l - p) // B) * B for l, p in zip(lens, prompts)]
    P = brute.rand_problem(rng, lens, prompts, H=2, dk=6, dv=5 if not conv else 6, V=2, B=B,
                           conv=conv, g_lo=-0.6)
    ref = pins._run(oracle.forward, P)
    got = chunk_reference.forward_chunked(P, C=C)
    for key in ("out", "out_noisy", "final_state"):
        err = np.max(np.abs(got[key] - ref[key]))
        assert err < 1e-10 * max(1.0, np.max(np.abs(ref[key]))), (key, err)


def test_chunk_bounds_anchor_at_response_start():
    b = chunk_reference.chunk_bounds(100, 300, 150, 64)
    assert b[0] == (100, 150 - 64 * 0) or b[0][1] == 150 - 0
    starts = [x for x, _ in b]
    assert 150 in starts and all((s - 150) % 64 == 0 for s in starts[1:])
    assert b[-1][1] == 300 and all(y == x2 for (_, y), (x2, _) in zip(b, b[1:]))


@pytest.mark.parametrize("B", [1, 2, 4, 8])
@pytest.mark.parametrize("conv", [0, 4])
def test_folded_noisy_rows_equal_sequential(B, conv):
    """The folded per-row form of the noisy stream (Z rows, W~V~ term, masked Z K^T) used by
    the tensor-core kernel equals the sequential oracle."""
    rng = np.random.default_rng(200 + B + conv)
    lens, prompts = [13 + 6 * B, 5 * B, 29 + 3 * B], [13, 0, 29]
    P = brute.rand_problem(rng, lens, prompts, H=2, dk=6, dv=6, V=2, B=B, conv=conv, g_lo=-0.6)
    ref = pins._run(oracle.forward, P)
    got = chunk_reference.forward_chunked_folded(P, C=max(8, 2 * B))
    for key in ("out", "out_noisy", "final_state"):
        err = np.max(np.abs(got[key] - ref[key]))
        assert err < 1e-10 * max(1.0, np.max(np.abs(ref[key]))), (key, err)
