"""The fp64 oracle against what the method and mathematics fix (CPU only)."""
import json
import os

import numpy as np
import pytest

import oracle
import pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.forward)


@pytest.mark.parametrize("name", ["gdr_hand_d2.json", "conv_antileak_hand_d1.json"])
def test_golden_hand_worked(name):
    fx = json.load(open(os.path.join(GOLDEN, name)))
    arr = lambda key: np.array(fx[key], dtype=np.float64)
    conv = None if fx["conv_w"] is None else arr("conv_w")
    r = oracle.forward(arr("q"), arr("k"), arr("v"), np.log(arr("alpha")), arr("beta"),
                       arr("qn"), arr("kn"), arr("vn"), np.log(arr("alphan")), arr("betan"),
                       fx["doc_offsets"], fx["prompt_len"], fx["block_size"], conv_w=conv)
    sq = np.sqrt(arr("q").shape[2])
    np.testing.assert_allclose(r["out"] * sq, np.array(fx["expect_times_sqrt_dk"]["out"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["out_noisy"] * sq, np.array(fx["expect_times_sqrt_dk"]["out_noisy"]),
                               rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["final_state"], np.array(fx["expect_final_state"]), rtol=0, atol=1e-12)


def test_rejects_misaligned_response():
    import brute
    P = brute.rand_problem(np.random.default_rng(0), [10], [4], V=1, B=4)
    with pytest.raises(ValueError):
        pins._run(oracle.forward, P)


def test_threads_do_not_change_result():
    import brute
    P = brute.rand_problem(np.random.default_rng(11), [40, 24, 36], [8, 0, 12], H=3, dk=8, dv=8, V=2, B=4, conv=4)
    a = pins._run(oracle.forward, P, num_threads=1)
    b = pins._run(oracle.forward, P, num_threads=4)
    for key in a:
        assert np.array_equal(a[key], b[key])
