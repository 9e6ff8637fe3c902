"""The range-checking build (libgdn_dual_debug.so: the chunked kernel and the ShortConv pass
compiled with GDN_DEBUG_BOUNDS, every computed global index checked before its access) on the
problems of tests/debug_bounds_run.py: no check may fail (status GDN_OK), and the outputs must
be bit-identical to the normal build's, since the checks do not change the arithmetic.  Each
build runs in a process of its own (one library per process)."""
import os
import subprocess
import sys

import pytest
import torch

from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import build as gbuild

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def run(lib, path):
    subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_run.py"), lib, path], check=True, timeout=600)
    return torch.load(path)


def test_range_checking_build_passes_and_matches(tmp_path):
    dbg_lib = gbuild.build_debug()
    normal = run(gbuild.LIB, str(tmp_path / "normal.pt"))
    checked = run(dbg_lib, str(tmp_path / "debug.pt"))
    assert normal.keys() == checked.keys()
    for key, r in checked.items():
        assert (r["status"], r["where"]) == (b.GDN_OK, 0), (key, r["status"], r["where"])
        assert normal[key]["status"] == b.GDN_OK, key
        for t in ("out", "out_noisy", "final_state"):
            assert torch.equal(r[t], normal[key][t]), (key, t)
