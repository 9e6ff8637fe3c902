"""gdn_dual_forward_noalloc: the entry point for callers that cannot allocate device memory (an
engine whose memory is all pre-reserved by its own pool, or a plugin host without a device
allocator).  It runs the same kernels as gdn_dual_forward, with the library's fixed scratch
array in place of a caller-owned workspace, so on the same inputs its outputs must be
bit-identical to gdn_dual_forward's, call after call, while the array is reused; and both must
match the fp64 oracle within the I/O dtype's tolerance.  After each call the device status read
from the array must be GDN_OK.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    # (lens, prompts, H, d, B, dtype, conv, tolerance against the oracle) -- bf16 d=128 runs the
    # tensor-core kernel (with and without the ShortConv prologue), fp32 d=32 the CUDA-core kernel
    ([200, 136], [72, 8], 2, 128, 4, "bf16", 0, 2e-2),
    ([200, 136], [72, 8], 2, 128, 4, "bf16", 4, 2e-2),
    ([64], [32], 2, 32, 4, "fp32", 0, 1e-4),
]


def rel(got, want):
    want = np.asarray(want)
    return float(np.max(np.abs(got.double().cpu().numpy() - want))) / max(float(np.max(np.abs(want))), 1e-30)


@pytest.mark.parametrize("lens,prompts,H,d,B,dtype,conv,tol", CASES)
def test_noalloc_matches_forward_on_two_calls(lens, prompts, H, d, B, dtype, conv, tol):
    offs = np.zeros(len(lens) + 1, np.int32)
    offs[1:] = np.cumsum(lens)
    prob = synth.make_problem_from_layout(offs, prompts, num_heads=H, d_k=d, d_v=d, block_size=B,
                                          num_views=2, dtype=dtype, conv_width=conv, seed=5, device="cuda")
    # the reference call gets a workspace of the same 256-byte class, so both calls take the same
    # path (with ShortConv: the chunked kernel's prologue rather than the separate conv pass)
    ref = [t.clone() for t in b.forward_problem(prob, workspace=b.Workspace(256))]
    torch.cuda.synchronize()
    want = oracle.forward_problem(prob)
    desc = b.make_desc(prob.num_docs, H, d, d, prob.num_views, B, b._dtype_code(prob.q), conv)
    for call in range(2):
        out = torch.full_like(ref[0], float("nan"))
        out_n = torch.full_like(ref[1], float("nan"))
        fs = torch.full_like(ref[2], float("nan"))
        st = b.forward_noalloc_raw(desc, prob.q, prob.k, prob.v, prob.g, prob.beta, prob.qn, prob.kn, prob.vn,
                                   prob.gn, prob.betan, prob.doc_offsets, prob.prompt_len, prob.conv_w,
                                   out, out_n, fs)
        assert st == b.GDN_OK, b.status_string(st)
        assert b.noalloc_read_device_status() == b.GDN_OK, f"call {call}"
        for got, same, key in zip((out, out_n, fs), ref, ("out", "out_noisy", "final_state")):
            assert torch.equal(got, same), f"call {call}: {key} differs from gdn_dual_forward"
            assert rel(got, want[key]) <= tol, f"call {call}: {key} against the oracle"
