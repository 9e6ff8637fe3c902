"""Dual-stream softmax attention (include/gdn_attention.h) against the fp64 oracle, element by
element, through the C ABI.  Tolerance: bf16 I/O, max|gpu - ref| <= 2e-2 max|ref| per output
tensor (one bf16 rounding of the output plus bf16 probabilities in the P V product)."""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 2e-2


def rel(gpu, ref):
    gpu = gpu.detach().double().cpu().numpy()
    if ref.size == 0:
        return 0.0
    return float(np.abs(gpu - ref).max() / max(np.abs(ref).max(), 1e-30))


def problem(lens, prompts, H=2, Hkv=2, B=4, V=2, seed=0):
    offs = np.zeros(len(lens) + 1, np.int32)
    offs[1:] = np.cumsum(lens)
    return synth.make_attn_problem_from_layout(offs, prompts, num_heads=H, num_kv_heads=Hkv, d=128, block_size=B,
                                               num_views=V, seed=seed, device="cuda")


def check(pr):
    out, outn = b.attention_forward(pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets, pr.prompt_len,
                                    pr.block_size)
    torch.cuda.synchronize()
    ref, refn = oa.dual_attention(pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets, pr.prompt_len,
                                  pr.block_size)
    e = (rel(out, ref), rel(outn, refn))
    assert max(e) <= TOL, e
    return e


@pytest.mark.parametrize("B", [1, 2, 4, 8, 16, 32])
def test_block_sizes_ragged_documents(B):
    """Documents shorter and longer than a 128-row tile, a ragged last tile, a prompt-only and a
    response-only document, several key tiles per query tile."""
    R = lambda r: (r // B) * B
    lens = [300, 129, 40 + R(64), 512 + R(96), 7]
    prompts = [300 - R(200), 129 - R(128), 40, 0, 7]
    check(problem(lens, prompts, B=B, seed=B))


@pytest.mark.parametrize("V", [0, 1, 2])
def test_view_counts(V):
    check(problem([260, 390], [100, 6], V=V, seed=10 + V))


@pytest.mark.parametrize("H,Hkv", [(4, 1), (4, 2), (3, 3)])
def test_grouped_key_value_heads(H, Hkv):
    check(problem([333, 200], [77, 32], H=H, Hkv=Hkv, seed=20 + H + Hkv))


def test_empty_document_and_single_tokens():
    check(problem([0, 1, 4, 0, 131], [0, 1, 0, 0, 3], seed=30))


def test_long_document_many_key_tiles():
    check(problem([1600], [400], H=1, Hkv=1, seed=31))


def test_large_scores_keep_the_softmax_stable():
    """q scaled by 8: scores up to ~ +-40; the reference max must move and rescale O."""
    pr = problem([700, 300], [200, 100], seed=32)
    pr.q.mul_(8.0)
    pr.qn.mul_(8.0)
    check(pr)


@pytest.mark.parametrize("name", sorted(synth.ATTN_WORKLOADS))
def test_full_size_sampled_rows(name):
    """The benchmarked shapes: sampled rows (tile edges, document edges, block edges, random) of
    the full-size call against the oracle evaluated row by row."""
    pr = synth.make_attn_problem(name, seed=1, device="cuda")
    out, outn = b.attention_forward(pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets, pr.prompt_len,
                                    pr.block_size)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    T, H = pr.q.shape[0], pr.q.shape[1]
    V, TR = pr.qn.shape[0], pr.qn.shape[1]
    offs = pr.doc_offsets.astype(np.int64)
    edges = [int(o) for o in offs[:-1]] + [int(o) - 1 for o in offs[1:]] + [127, 128, 255, 4095]
    cr = [(p, int(rng.integers(H))) for p in edges if 0 <= p < T]
    cr += [(int(p), int(rng.integers(H))) for p in rng.integers(0, T, 24)]
    nr = [(int(rng.integers(V)), int(r), int(rng.integers(H))) for r in rng.integers(0, TR, 32)]
    nr += [(0, 0, 0), (V - 1, TR - 1, H - 1), (0, 127, 1), (1 % V, 128, 2)]
    qc, kc, vc = (t.cpu() for t in (pr.q, pr.k, pr.v))
    qnc, knc, vnc = (t.cpu() for t in (pr.qn, pr.kn, pr.vn))
    c, nn = oa.dual_attention_rows(qc, kc, vc, qnc, knc, vnc, pr.doc_offsets, pr.prompt_len, pr.block_size, cr, nr)
    ref_c = np.stack(c)
    ref_n = np.stack(nn)
    got_c = torch.stack([out[p, h] for p, h in cr]).double().cpu().numpy()
    got_n = torch.stack([outn[w, r, h] for w, r, h in nr]).double().cpu().numpy()
    assert np.abs(got_c - ref_c).max() <= TOL * np.abs(ref_c).max()
    assert np.abs(got_n - ref_n).max() <= TOL * np.abs(ref_n).max()


def test_invalid_arguments_launch_nothing():
    pr = problem([260, 390], [100, 6], seed=40)
    out = torch.full_like(pr.q, 7.0)
    with pytest.raises(b.GdnError) as e:     # response 162 not a multiple of B = 4
        b.attention_forward(pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets, [98, 8], 4, out=out)
    assert e.value.status == b.GDN_ERR_INVALID_ARG
    p3 = problem([260, 390], [101, 9], B=3, seed=41)
    out3 = torch.full_like(p3.q, 7.0)
    with pytest.raises(b.GdnError) as e:     # valid layout for B = 3, but 128 % 3 != 0
        b.attention_forward(p3.q, p3.k, p3.v, p3.qn, p3.kn, p3.vn, p3.doc_offsets, p3.prompt_len, 3, out=out3)
    assert e.value.status == b.GDN_ERR_UNSUPPORTED
    with pytest.raises(ValueError):          # noisy rows do not match the layout
        b.attention_forward(pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets, [104, 6], 4, out=out)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()) and bool((out3 == 7.0).all())
