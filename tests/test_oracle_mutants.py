"""Planted mistakes in the oracle (CPU only): each textual mutation of the oracle's C source
is compiled into a throw-away library, and at least one pin must reject it.  This shows the
pins are sharp enough to catch a dropped term, a wrong sign, a wrong state or a leaking tap."""
import os
import subprocess
import tempfile

import pytest

import oracle
import pins

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")).read()

MUTANTS = {
    "erase_not_decayed": ("row[j] = alpha * (row[j] - beta * ki * u[j]) + beta * ki * v[j];",
                          "row[j] = alpha * row[j] - beta * ki * u[j] + beta * ki * v[j];"),
    "erase_sign": ("row[j] = alpha * (row[j] - beta * ki * u[j]) + beta * ki * v[j];",
                   "row[j] = alpha * (row[j] + beta * ki * u[j]) + beta * ki * v[j];"),
    "write_without_beta": ("row[j] = alpha * (row[j] - beta * ki * u[j]) + beta * ki * v[j];",
                           "row[j] = alpha * (row[j] - beta * ki * u[j]) + ki * v[j];"),
    "scale_by_dv": ("const double scale = 1.0 / sqrt((double)dk);",
                    "const double scale = 1.0 / sqrt((double)dv);"),
    "clean_read_before_update": (
        "            delta_step(S, u, dk, dv, kc, vc, exp(g[tok * H + h]), beta[tok * H + h]);\n"
        "            readout(S, dk, dv, qc, out + tok * sv + (long)h * dv);",
        "            readout(S, dk, dv, qc, out + tok * sv + (long)h * dv);\n"
        "            delta_step(S, u, dk, dv, kc, vc, exp(g[tok * H + h]), beta[tok * H + h]);"),
    "noisy_ungated": ("exp(gnv[r * H]), bnv[r * H]);", "1.0, bnv[r * H]);"),
    "noisy_reads_own_position_state": (
        "                    /* every position of the block reads the block-end state */\n"
        "                    for (int l = 0; l < B; ++l) {",
        "                    memcpy(St, S, sizeof(double) * (size_t)dk * dv);\n"
        "                    for (int l = 0; l < B; ++l) {\n"
        "                        delta_step(St, u, dk, dv, kb + (long)l * dk, vb + (long)l * dv,\n"
        "                                   exp(gnv[(long)(b0 + l) * H]), bnv[(long)(b0 + l) * H]);"),
    "conv_noisy_taps_leak": ("        if (src >= blk_start)\n", "        if (src >= resp_start)\n"),
    "conv_tap_reversed": ("        acc += w[W - 1 - j] * x_doc[(long)src * stride];",
                          "        acc += w[j] * x_doc[(long)src * stride];"),
}


def _build_mutant(name, tmpdir):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, f"mutation anchor for {name} not found"
    src = os.path.join(tmpdir, f"{name}.c")
    lib = os.path.join(tmpdir, f"lib{name}.so")
    open(src, "w").write(SRC.replace(old, new, 1))
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", lib, src, "-lm"])
    return oracle.open_library(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_some_pin_rejects_mutant(name):
    with tempfile.TemporaryDirectory() as tmp:
        lib = _build_mutant(name, tmp)

        def fwd(*a, **kw):
            return oracle.forward(*a, _lib=lib, **kw)

        failed = []
        for pin in pins.ALL_PINS:
            try:
                pin(fwd)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"no pin rejects the planted mistake {name}"
