"""Failure detection on the GPU without a fault: every device-side mbarrier wait of the
tensor-core kernels is bounded.  Through the test-only entry points each wait is bounded by one
try-wait, so a wait gives up while the copy or MMA it waits for is still in flight.  The kernel
must record GDN_ERR_TIMEOUT and the site of the wait in the workspace, wait (with the normal
bound) for every copy and MMA it had already issued, free its tensor memory and leave; the
context stays usable, and the next ordinary call on the same workspace returns GDN_OK with
oracle-correct outputs.  Nothing here waits on a flag that is never set, traps or faults."""
import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 2e-2


def rel(got, ref):
    got = got.detach().double().cpu().numpy()
    return float(np.max(np.abs(got - ref))) / max(float(np.max(np.abs(ref))), 1e-30)


@pytest.mark.parametrize("algo,conv", [(b.ALGO_CHUNKED, 0), (b.ALGO_CHUNKED, 4), (b.ALGO_PIPELINED, 0)])
def test_forward_wait_gives_up_then_next_call_is_correct(algo, conv):
    offs = np.array([0, 200, 328], np.int32)
    prob = synth.make_problem_from_layout(offs, [72, 0], num_heads=2, d_k=128, d_v=128, block_size=4,
                                          num_views=2, dtype="bf16", conv_width=conv, seed=60 + conv, device="cuda")
    desc = b.make_desc(2, 2, 128, 128, 2, 4, b.GDN_BF16, conv, algo)
    ws = b.Workspace(256)
    out = torch.empty(prob.T, 2, 128, dtype=torch.bfloat16, device="cuda")
    out_n = torch.empty(2, prob.T_R, 2, 128, dtype=torch.bfloat16, device="cuda")
    fs = torch.empty(2, 2, 128, 128, device="cuda")
    for attempt in range(2):          # twice: the context and the workspace stay usable
        st = b.forward_test_wait_limit_raw(desc, prob.q, prob.k, prob.v, prob.g, prob.beta, prob.qn, prob.kn,
                                           prob.vn, prob.gn, prob.betan, prob.doc_offsets, prob.prompt_len,
                                           prob.conv_w, out, out_n, fs, ws.tensor, 1)
        assert st == b.GDN_OK, b.status_string(st)       # the call itself enqueues normally
        status, where = b.read_device_status_where(ws.tensor)
        assert status == b.GDN_ERR_TIMEOUT and where > 0, (attempt, status, where)
    out, out_n, fs = b.forward_problem(prob, workspace=ws, algo=algo)
    assert b.read_device_status_where(ws.tensor) == (b.GDN_OK, 0)
    ref = oracle.forward_problem(prob)
    errs = (rel(out, ref["out"]), rel(out_n, ref["out_noisy"]), rel(fs, ref["final_state"]))
    assert max(errs) <= TOL, errs


def test_attention_wait_gives_up_then_next_call_is_correct():
    offs = np.array([0, 300, 429], np.int32)
    pr = synth.make_attn_problem_from_layout(offs, [100, 1], num_heads=2, num_kv_heads=2, d=128, block_size=4,
                                             num_views=2, seed=70, device="cuda")
    desc = b.make_attn_desc(2, 2, 2, 128, 2, 4, b.GDN_BF16)
    ws = b.Workspace(256)
    out = torch.empty_like(pr.q)
    out_n = torch.empty_like(pr.qn)
    for attempt in range(2):
        st = b.attention_forward_test_wait_limit_raw(desc, pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets,
                                                     pr.prompt_len, out, out_n, ws.tensor, 1)
        assert st == b.GDN_OK, b.status_string(st)
        status, where = b.read_device_status_where(ws.tensor)
        assert status == b.GDN_ERR_TIMEOUT and where > 0, (attempt, status, where)
    out, out_n = b.attention_forward(pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets, pr.prompt_len,
                                     pr.block_size, workspace=ws.tensor)
    assert b.read_device_status_where(ws.tensor) == (b.GDN_OK, 0)
    ref, refn = oa.dual_attention(pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets, pr.prompt_len,
                                  pr.block_size)
    assert max(rel(out, ref), rel(out_n, refn)) <= TOL
