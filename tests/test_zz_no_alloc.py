"""gdn_dual_forward_noalloc: the entry point for callers that cannot allocate device memory
(an engine whose memory is all pre-reserved by its own pool, or a plugin host without a device
allocator).  It must give the same results as gdn_dual_forward with a caller-owned workspace,
call after call, while the library's fixed scratch array is reused.  This file is collected
last on purpose."""
import numpy as np
import pytest
import torch

from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    # (lens, prompts, H, d, B, dtype, tolerance)  -- bf16 d=128 runs the tensor-core kernel,
    # fp32 d=32 the CUDA-core kernel
    ([200, 136], [72, 8], 2, 128, 4, "bf16", 2e-2),
    ([64], [32], 2, 32, 4, "fp32", 1e-4),
]


@pytest.mark.parametrize("lens,prompts,H,d,B,dtype,tol", CASES)
def test_noalloc_matches_forward_on_two_calls(lens, prompts, H, d, B, dtype, tol):
    offs = np.zeros(len(lens) + 1, np.int32)
    offs[1:] = np.cumsum(lens)
    prob = synth.make_problem_from_layout(offs, prompts, num_heads=H, d_k=d, d_v=d, block_size=B,
                                          num_views=2, dtype=dtype, seed=5, device="cuda")
    ref = [t.clone() for t in b.forward_problem(prob)]
    torch.cuda.synchronize()
    desc = b.make_desc(prob.num_docs, H, d, d, prob.num_views, B, b._dtype_code(prob.q))
    for call in range(2):
        out = torch.full_like(ref[0], float("nan"))
        out_n = torch.full_like(ref[1], float("nan"))
        fs = torch.full_like(ref[2], float("nan"))
        st = b.forward_noalloc_raw(desc, prob.q, prob.k, prob.v, prob.g, prob.beta, prob.qn, prob.kn, prob.vn,
                                   prob.gn, prob.betan, prob.doc_offsets, prob.prompt_len, None,
                                   out, out_n, fs)
        assert st == b.GDN_OK, b.status_string(st)
        torch.cuda.synchronize()
        for got, want in zip((out, out_n, fs), ref):
            scale = float(want.float().abs().max())
            assert float((got.float() - want.float()).abs().max()) <= tol * scale, f"call {call}"
