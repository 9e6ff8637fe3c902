"""The oracle's decode-side steps against their pins, and planted mistakes in them (CPU only)."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import decode_pins
import oracle

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")).read()


def _steps(lib=None):
    def steps(S0, q, k, v, g, beta, record):
        return oracle.decode_steps(S0, q, k, v, g, beta, record_states=record, _lib=lib)
    return steps


@pytest.mark.parametrize("pin", decode_pins.DECODE_PINS, ids=lambda p: p.__name__)
def test_decode_pin(pin):
    pin(_steps(), oracle.forward)


def test_commit_definition():
    """commit() is the gather-scatter of its definition: rows of accepted sequences take the
    state after their r-th candidate, r = 0 and slots of other sequences stay as they were."""
    rng = np.random.default_rng(7)
    S0, q, k, v, g, beta = decode_pins.rand_decode(rng, N=3, L=4)
    pool = rng.standard_normal((6,) + S0.shape[1:])
    slots = np.array([4, 0, 2])
    pool[slots] = S0
    rec = oracle.decode_steps(S0, q, k, v, g, beta, record_states=True)
    acc = np.array([0, 4, 2])
    new = oracle.commit(pool, slots, rec["states"], acc)
    assert np.array_equal(new[4], S0[0])                    # r = 0: unchanged
    assert np.array_equal(new[0], rec["final_state"][1])     # r = L: the full run
    pre = oracle.decode_steps(S0[2:3], q[2:3, :2], k[2:3, :2], v[2:3, :2], g[2:3, :2], beta[2:3, :2])
    assert np.array_equal(new[2], pre["final_state"][0])     # r = 2: the two-token run
    for s in (1, 3, 5):
        assert np.array_equal(new[s], pool[s])


DECODE_MUTANTS = {
    "starts_from_zero": ("memcpy(S, S0 + unit * sz, sizeof(double) * (size_t)sz);",
                         "memset(S, 0, sizeof(double) * (size_t)sz);"),
    "records_state_before_update": (
        "            delta_step(S, u, dk, dv, k + row * dk, v + row * dv, exp(g[row]), beta[row]);\n"
        "            readout(S, dk, dv, q + row * dk, out + row * dv);\n"
        "            if (states) memcpy(states + row * sz, S, sizeof(double) * (size_t)sz);",
        "            if (states) memcpy(states + row * sz, S, sizeof(double) * (size_t)sz);\n"
        "            delta_step(S, u, dk, dv, k + row * dk, v + row * dv, exp(g[row]), beta[row]);\n"
        "            readout(S, dk, dv, q + row * dk, out + row * dv);"),
    "final_state_is_start": ("memcpy(S_final + unit * sz, S, sizeof(double) * (size_t)sz);",
                             "memcpy(S_final + unit * sz, S0 + unit * sz, sizeof(double) * (size_t)sz);"),
    "token_major_rows": ("const long row = (n * L + t) * H + h;", "const long row = ((long)t * Nseq + n) * H + h;"),
    "ungated": ("exp(g[row]), beta[row]);", "1.0, beta[row]);"),
}


@pytest.mark.parametrize("name", sorted(DECODE_MUTANTS))
def test_some_decode_pin_rejects_mutant(name):
    old, new = DECODE_MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation anchor for {name} not found"
    with tempfile.TemporaryDirectory() as tmp:
        src, lib = os.path.join(tmp, "m.c"), os.path.join(tmp, "libm.so")
        open(src, "w").write(SRC.replace(old, new))
        subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", lib, src, "-lm"])
        mlib = oracle.open_library(lib)
        failed = []
        for pin in decode_pins.DECODE_PINS:
            try:
                pin(_steps(mlib), oracle.forward)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"no decode pin rejects the planted mistake {name}"
