"""Decode-side kernels (include/gdn_decode.h) against the fp64 oracle, element by element.

Causal replay, verify forward with state cache, and the gather-scatter commit (the serving
paragraph of the FLARE notes), through the C ABI.  Tolerances: bf16 I/O max|gpu - ref| <=
2e-2 max|ref| per tensor (outputs), fp32 states <= 1e-4 max|ref|; fp32 I/O 1e-4 everywhere."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_dual_b200 import binding as b
from gated_deltanet_dual_b200 import synth

pytestmark = pytest.mark.gpu


def _close(gpu, ref, tol, what):
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(gpu - ref).max()
    assert err <= tol * scale, f"{what}: max err {err:.3e} > {tol} * {scale:.3e}"


def _tols(dtype):
    return (2e-2, 1e-4) if dtype == "bf16" else (1e-4, 1e-4)


def _problem(N, H, d, L, P, dtype, seed=0):
    return synth.make_decode_problem(N, H, d, L, P, dtype=dtype, seed=seed, device="cuda")


def _oracle_steps(pr, record=False):
    S0 = pr.state_pool[pr.slots.long()]
    return oracle.decode_steps(S0, pr.q, pr.k, pr.v, pr.g, pr.beta, record_states=record)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("L", [1, 4, 17])
def test_replay(dtype, d, L):
    pr = _problem(3, 4, d, L, 7, dtype, seed=d + L)
    before = pr.state_pool.clone()
    ref = _oracle_steps(pr)
    out = b.decode_replay(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta)
    torch.cuda.synchronize()
    to, ts = _tols(dtype)
    _close(out, ref["out"], to, "replay out")
    used = pr.slots.long()
    _close(pr.state_pool[used], ref["final_state"], ts, "replay pool rows")
    mask = torch.ones(pr.state_pool.shape[0], dtype=torch.bool, device="cuda")
    mask[used] = False
    assert torch.equal(pr.state_pool[mask], before[mask]), "replay touched rows of other sequences"


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("d", [64, 128])
def test_verify_caches_every_step(dtype, d):
    pr = _problem(4, 3, d, 5, 9, dtype, seed=11)
    before = pr.state_pool.clone()
    ref = _oracle_steps(pr, record=True)
    out, cache = b.decode_verify(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta)
    torch.cuda.synchronize()
    to, ts = _tols(dtype)
    _close(out, ref["out"], to, "verify out")
    _close(cache, ref["states"], ts, "verify state cache")
    assert torch.equal(pr.state_pool, before), "verify must not write the pool"


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_commit_accepts_prefix(dtype):
    """verify -> commit(r) leaves, in each sequence's pool row, the state of a run over only its
    first r candidates (r = 0 keeps the row); other rows are untouched, bit for bit."""
    N, H, d, L, P = 5, 2, 128, 4, 12
    pr = _problem(N, H, d, L, P, dtype, seed=5)
    before = pr.state_pool.clone()
    _, cache = b.decode_verify(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta)
    acc = torch.tensor([0, 1, 4, 2, 3], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.decode_commit(pr.state_pool, pr.slots, cache, acc, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == b.GDN_OK
    # the gather itself is exact: compare with the definition applied to the GPU cache
    expect = oracle.commit(before.cpu().numpy(), pr.slots.cpu().numpy(), cache.cpu().numpy(), acc.cpu().numpy())
    assert np.array_equal(pr.state_pool.cpu().numpy().astype(np.float64), expect)
    # and the committed state is the prefix run of the oracle
    _, ts = _tols(dtype)
    S0 = before[pr.slots.long()]
    for n, r in enumerate(acc.tolist()):
        row = int(pr.slots[n])
        if r == 0:
            assert torch.equal(pr.state_pool[row], before[row])
            continue
        pre = oracle.decode_steps(S0[n:n + 1], pr.q[n:n + 1, :r], pr.k[n:n + 1, :r], pr.v[n:n + 1, :r],
                                  pr.g[n:n + 1, :r], pr.beta[n:n + 1, :r])
        _close(pr.state_pool[row], pre["final_state"][0], ts, f"committed state of sequence {n}")


def test_verify_commit_then_replay_continues_the_run():
    """AR-Trust accepts r of K candidates, Diffusion-Trust then replays the next block: the pool
    ends where one oracle run over the r accepted tokens and the block ends."""
    N, H, d, K, P = 3, 4, 128, 4, 8
    pr = _problem(N, H, d, K, P, "fp32", seed=21)
    nxt = _problem(N, H, d, 4, P, "fp32", seed=22)
    S0 = pr.state_pool[pr.slots.long()].clone()
    _, cache = b.decode_verify(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta)
    acc = torch.tensor([2, 4, 1], dtype=torch.int32, device="cuda")
    b.decode_commit(pr.state_pool, pr.slots, cache, acc)
    out = b.decode_replay(pr.state_pool, pr.slots, nxt.q, nxt.k, nxt.v, nxt.g, nxt.beta)
    torch.cuda.synchronize()
    for n, r in enumerate(acc.tolist()):
        sl = slice(n, n + 1)
        cat = lambda a, c: torch.cat([a[sl, :r], c[sl]], dim=1)
        ref = oracle.decode_steps(S0[sl], cat(pr.q, nxt.q), cat(pr.k, nxt.k), cat(pr.v, nxt.v),
                                  cat(pr.g, nxt.g), cat(pr.beta, nxt.beta))
        _close(out[sl], ref["out"][:, r:], 1e-4, f"replayed outputs of sequence {n}")
        _close(pr.state_pool[int(pr.slots[n])], ref["final_state"][0], 1e-4, f"pool row of sequence {n}")


def test_bad_slot_and_bad_accepted_are_flagged_and_skipped():
    N, H, d, L, P = 3, 2, 64, 3, 5
    pr = _problem(N, H, d, L, P, "fp32", seed=31)
    pr.slots[1] = P + 2                       # out of range: that sequence is skipped
    before = pr.state_pool.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.decode_replay(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == b.GDN_ERR_INVALID_ARG
    good = [0, 2]
    S0 = before[pr.slots[good].long()]
    ref = oracle.decode_steps(S0, pr.q[good], pr.k[good], pr.v[good], pr.g[good], pr.beta[good])
    _close(pr.state_pool[pr.slots[good].long()], ref["final_state"], 1e-4, "valid sequences")
    untouched = [s for s in range(P) if s not in pr.slots[good].tolist()]
    assert torch.equal(pr.state_pool[untouched], before[untouched])
    # commit with an accepted count beyond L
    pr2 = _problem(N, H, d, L, P, "fp32", seed=32)
    _, cache = b.decode_verify(pr2.state_pool, pr2.slots, pr2.q, pr2.k, pr2.v, pr2.g, pr2.beta)
    before2 = pr2.state_pool.clone()
    acc = torch.tensor([L + 1, 0, 1], dtype=torch.int32, device="cuda")
    b.decode_commit(pr2.state_pool, pr2.slots, cache, acc, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == b.GDN_ERR_INVALID_ARG
    assert torch.equal(pr2.state_pool[int(pr2.slots[0])], before2[int(pr2.slots[0])])
    assert torch.equal(pr2.state_pool[int(pr2.slots[2])], cache[2, 0])


@pytest.mark.parametrize("name", sorted(synth.DECODE_WORKLOADS))
def test_decode_workloads_full_size(name):
    """The benchmarked decode shapes: replay and verify at full size against the oracle."""
    cfg = synth.DECODE_WORKLOADS[name]
    pr = synth.make_decode_problem(**cfg, dtype="bf16", seed=3, device="cuda")
    ref = _oracle_steps(pr, record=True)
    out, cache = b.decode_verify(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta)
    out2 = b.decode_replay(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta)
    torch.cuda.synchronize()
    _close(out, ref["out"], 2e-2, "verify out")
    _close(out2, ref["out"], 2e-2, "replay out")
    _close(cache, ref["states"], 1e-4, "state cache")
    _close(pr.state_pool[pr.slots.long()], ref["final_state"], 1e-4, "replayed pool rows")
