"""Host-side work models of bench.py: the visible-pair count behind the attention roofline and
the algorithmic byte counts, checked against explicit enumeration (CPU only)."""
import numpy as np
import pytest

import bench
from gated_deltanet_dual_b200 import synth


def brute_pairs(offs, pl, B, V):
    """Count (query, key) pairs of the document-blocked mask one query at a time."""
    n_pairs = 0
    for n in range(len(pl)):
        L, P = offs[n + 1] - offs[n], pl[n]
        for p in range(L):
            n_pairs += p + 1                       # clean query: keys [0, p]
        for r in range(L - P):
            b0 = (r // B) * B
            n_pairs += V * (P + b0 + B)           # noisy query: clean prefix + its block
    return n_pairs


@pytest.mark.parametrize("B", [1, 2, 4, 8])
def test_attention_pairs_match_enumeration(B):
    rng = np.random.default_rng(B)
    lens = [int(x) for x in rng.integers(0, 60, 5)]
    prompts = []
    for ln in lens:
        p = int(rng.integers(0, ln + 1))
        p += (ln - p) % B                          # response in whole blocks
        prompts.append(p)
    offs = np.concatenate([[0], np.cumsum(lens)])
    for V in (0, 1, 2):
        assert bench.attn_pairs(offs, prompts, B, V) == brute_pairs(offs, prompts, B, V)


@pytest.fixture(scope="module")
def train_problem():
    return synth.make_problem("train_8x4096_h16_d128", seed=0, device="cpu")


def test_backward_bytes_of_the_training_workload(train_problem):
    prob = train_problem
    toks = (32768 + 2 * 24576) * 16
    # bf16 q, k, v, upstream grad (4 x 256 B), g and beta (8 B); fp32 dq, dk, dv (3 x 512 B),
    # dg and dbeta (8 B); one fp32 128 x 128 final-state gradient per (document, head)
    expect = toks * (4 * 256 + 8 + 3 * 512 + 8) + 8 * 16 * 128 * 128 * 4
    assert bench.backward_bytes(prob) == expect


def test_forward_bytes_per_token_head(train_problem):
    w = bench.algorithmic_work(train_problem)
    assert w["bytes_per_token_head"] == 1032
