"""Run a fixed set of forward problems through one build of the library and save what they
produce (test infrastructure for tests/test_gpu_debug_bounds.py).

    python tests/debug_bounds_run.py <library .so> <output .pt>

Each problem runs with the workspace gdn_dual_workspace_size asks for (so the ShortConv pass
runs) and, for the ShortConv ones, again with a 256-byte workspace (the fused prologue); the
outputs and the device status words after each call are saved."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from gated_deltanet_dual_b200 import binding as b  # noqa: E402
from gated_deltanet_dual_b200 import synth  # noqa: E402


def problems():
    """(name, problem): block sizes, views, ShortConv on and off, degenerate documents, few units
    (split over two CTAs), chunks that straddle document edges, and one full-size workload."""
    def layout(lens, prompts, **kw):
        offs = np.zeros(len(lens) + 1, np.int32)
        offs[1:] = np.cumsum(lens)
        return synth.make_problem_from_layout(offs, prompts, device="cuda", **kw)
    for B in (1, 4, 32):
        for conv in (0, 4):
            yield f"ragged_B{B}_conv{conv}", layout([200, 136, 96], [72, 8, 32], num_heads=3, d_k=128, d_v=128,
                                                    block_size=B, num_views=2, dtype="bf16", conv_width=conv,
                                                    seed=B + conv)
    for V in (0, 1, 3):
        yield f"views{V}", layout([192, 128], [64, 0], num_heads=2, d_k=128, d_v=128, block_size=4, num_views=V,
                                  dtype="bf16", conv_width=4, seed=40 + V)
    yield "degenerate", layout([0, 64, 5, 0, 300, 4, 64], [0, 64, 1, 0, 100, 0, 0], num_heads=2, d_k=128, d_v=128,
                               block_size=4, num_views=2, dtype="bf16", conv_width=4, seed=7)
    yield "train_8x4096_h16_d128", synth.make_problem("train_8x4096_h16_d128", device="cuda")


def main(lib, path):
    b.load_library(lib)
    res = {}
    for name, prob in problems():
        desc = b.make_desc(prob.num_docs, prob.num_heads, prob.d_k, prob.d_v, prob.num_views, prob.block_size,
                           b._dtype_code(prob.q), prob.conv_width)
        sizes = [b.workspace_size(desc, prob.doc_offsets)] + ([256] if prob.conv_width else [])
        for size in sizes:
            ws = b.Workspace(size)
            out, out_n, fs = b.forward_problem(prob, workspace=ws)
            status, where = b.read_device_status_where(ws.tensor)
            res[f"{name}/ws{size}"] = {"status": status, "where": where, "out": out.cpu(), "out_noisy": out_n.cpu(),
                                       "final_state": fs.cpu()}
    torch.save(res, path)


if __name__ == "__main__":
    main(sys.argv[1], sys.argv[2])
