"""Precision study for a tensor-core backward: the chunked backward of
tests/chunk_backward_reference.py with every chunk-level matrix product taking bf16-rounded
operands (wide accumulation, as tcgen05 kind::f16 does), against the fp64 token-by-token
backward oracle on the same bf16 inputs.  All gradients must stay within the bf16 I/O bar of
2e-2 max|ref| (measured: at most 5.3e-3 at d = 64 and 3.5e-3 at d = 128), so the planned kernel
can keep bf16 operands everywhere, the triangular inverse T included."""
import numpy as np
import pytest

from oracle import backward as ob
import chunk_backward_reference as cbr


def bf16(x):
    """Round to the nearest bfloat16 (ties to even): keep the top 16 bits of the fp32 pattern."""
    x32 = np.ascontiguousarray(x, dtype=np.float32)
    b = x32.view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return b.view(np.float32).astype(np.float64)


def test_bf16_rounding_helper():
    assert bf16(np.array([1.0]))[0] == 1.0
    assert bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0            # tie: to even
    assert bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    assert bf16(np.array([1.0 + 2.0 ** -7]))[0] == 1.0 + 2.0 ** -7


@pytest.mark.parametrize("ckpt", [None, "bf16"])
@pytest.mark.parametrize("d,L,P", [(64, 1024, 256), (128, 1024, 256)])
def test_chunked_backward_with_bf16_operands_meets_the_bf16_bar(d, L, P, ckpt):
    """ckpt = "bf16": the chunk-start states are also stored in bf16 (half the checkpoint
    traffic); measured errors do not move (at most 5.3e-3)."""
    rng = np.random.default_rng(0)
    H, V, B = 1, 2, 4
    R = L - P
    unit = lambda a: a / np.linalg.norm(a, axis=-1, keepdims=True)
    x = lambda *s: rng.standard_normal(s)
    ins = dict(q=bf16(unit(x(L, H, d))), k=bf16(unit(x(L, H, d))), v=bf16(x(L, H, d)), g=-0.1 * rng.random((L, H)),
               beta=1 / (1 + np.exp(-x(L, H))), qn=bf16(unit(x(V, R, H, d))), kn=bf16(unit(x(V, R, H, d))),
               vn=bf16(x(V, R, H, d)), gn=-0.1 * rng.random((V, R, H)), betan=1 / (1 + np.exp(-x(V, R, H))))
    order = ("q", "k", "v", "g", "beta", "qn", "kn", "vn", "gn", "betan")
    do, don, dsf = bf16(x(L, H, d)), bf16(x(V, R, H, d)), x(1, H, d, d)
    offs = np.array([0, L], np.int32)
    ref = ob.dual_backward(*(ins[n] for n in order), offs, [P], B, do, don, dsf)
    cbr.set_operand_rounding(bf16)
    try:
        got = cbr.dual_backward_chunked(*(ins[n] for n in order), offs, [P], B, do, don, dsf, C=64,
                                        checkpoint_round=bf16 if ckpt else None)
    finally:
        cbr.set_operand_rounding(None)
    errs = {n: float(np.abs(got[n] - ref[n]).max() / np.abs(ref[n]).max()) for n in ref}
    assert max(errs.values()) <= 2e-2, errs
    # the rounding really happened (not an exact run)
    assert max(errs.values()) > 1e-4, errs
