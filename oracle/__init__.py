"""fp64 CPU oracle for the dual-stream Gated DeltaNet forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package.  It shares no code with the CUDA
library (it is plain C compiled with gcc, called through ctypes).

The C source (gdn_oracle.c) states what it computes and which passage of
"FLARE: Diffusion for Hybrid Language Model" (papernotes.org notes, Method >
Key design 2 and Key design 3) each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O3, OpenMP, fp64; no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def open_library(path: str):
    """Load a compiled oracle (the default one, or a test-built variant) and set its
    ctypes signature."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int32)
    lib.gdn_oracle_forward.restype = ctypes.c_int
    lib.gdn_oracle_forward.argtypes = ([ctypes.c_int] * 7 + [ip, ip] + [dp] * 10 + [dp]
                                       + [dp, dp, dp, dp] + [ctypes.c_int])
    lib.gdn_oracle_max_threads.restype = ctypes.c_int
    lib.gdn_oracle_decode_steps.restype = ctypes.c_int
    lib.gdn_oracle_decode_steps.argtypes = [ctypes.c_int] * 5 + [dp] * 9 + [ctypes.c_int]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = open_library(_LIB)
    return _lib


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        x = x.double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().gdn_oracle_max_threads())


def forward(q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, block_size,
            conv_w=None, num_threads: int = 0, return_noisy_state: bool = False, _lib=None):
    """Run the oracle.  Shapes as in the CUDA library (see include/gdn_dual.h); inputs may be
    numpy arrays or torch tensors (any dtype, any device): they are widened to fp64 on the host.

    Returns dict(out=[T,H,dv], out_noisy=[V,T_R,H,dv], final_state=[N,H,dk,dv]
    [, noisy_state=[V, T_R/B, H, dk, dv]]) as fp64 numpy arrays."""
    lib = _lib if _lib is not None else _load()
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    qn, kn, vn, gn, betan = (_f64(x) for x in (qn, kn, vn, gn, betan))
    offs = np.ascontiguousarray(np.asarray(doc_offsets, dtype=np.int32))
    pl = np.ascontiguousarray(np.asarray(prompt_len, dtype=np.int32))
    T, H, dk = q.shape
    dv = v.shape[2]
    V = qn.shape[0]
    TR = qn.shape[1]
    N = offs.shape[0] - 1
    W = 0
    cw = None
    if conv_w is not None:
        cw = _f64(conv_w)
        W = int(cw.shape[-1])
    out = np.zeros((T, H, dv))
    out_noisy = np.zeros((V, TR, H, dv))
    final_state = np.zeros((N, H, dk, dv))
    ns = np.zeros((V, TR // block_size, H, dk, dv)) if return_noisy_state else None
    ip = ctypes.POINTER(ctypes.c_int32)
    rc = lib.gdn_oracle_forward(N, H, dk, dv, V, int(block_size), W,
                                offs.ctypes.data_as(ip), pl.ctypes.data_as(ip),
                                _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                _ptr(qn), _ptr(kn), _ptr(vn), _ptr(gn), _ptr(betan),
                                _ptr(cw), _ptr(out), _ptr(out_noisy), _ptr(final_state), _ptr(ns),
                                int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle rejected the inputs (code {rc})")
    res = dict(out=out, out_noisy=out_noisy, final_state=final_state)
    if return_noisy_state:
        res["noisy_state"] = ns
    return res


def forward_problem(prob, num_threads: int = 0, return_noisy_state: bool = False, _lib=None):
    """Convenience wrapper for objects with the synthetic-problem attributes."""
    return forward(prob.q, prob.k, prob.v, prob.g, prob.beta, prob.qn, prob.kn, prob.vn,
                   prob.gn, prob.betan, prob.doc_offsets, prob.prompt_len, prob.block_size,
                   conv_w=prob.conv_w, num_threads=num_threads,
                   return_noisy_state=return_noisy_state, _lib=_lib)


def decode_steps(S0, q, k, v, g, beta, record_states: bool = False, num_threads: int = 0, _lib=None):
    """Decode-side clean steps from given states (the serving paragraph of the FLARE notes:
    Diffusion-Trust causal replay of a committed block; AR-Trust verify forward with every
    step's state kept for the rollback).  S0 [Nseq,H,dk,dv]; q,k [Nseq,L,H,dk]; v [Nseq,L,H,dv];
    g, beta [Nseq,L,H].  Returns dict(out=[Nseq,L,H,dv], final_state=[Nseq,H,dk,dv]
    [, states=[Nseq,L,H,dk,dv]]) as fp64 arrays."""
    lib = _lib if _lib is not None else _load()
    S0, q, k, v, g, beta = (_f64(x) for x in (S0, q, k, v, g, beta))
    Nseq, L, H, dk = q.shape
    dv = v.shape[3]
    out = np.zeros((Nseq, L, H, dv))
    fin = np.zeros((Nseq, H, dk, dv))
    st = np.zeros((Nseq, L, H, dk, dv)) if record_states else None
    rc = lib.gdn_oracle_decode_steps(Nseq, H, L, dk, dv, _ptr(S0), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                     _ptr(beta), _ptr(out), _ptr(fin), _ptr(st), int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle rejected the inputs (code {rc})")
    res = dict(out=out, final_state=fin)
    if record_states:
        res["states"] = st
    return res


def commit(pool, slots, states, accepted):
    """AR-Trust rollback by gather-scatter (the serving paragraph of the FLARE notes): for every
    sequence i with accepted[i] = r >= 1, pool[slots[i]] := states[i, r - 1] (the state after the
    r accepted candidates); r = 0 leaves the pool row as it was.  Returns a new fp64 array."""
    pool = _f64(pool).copy()
    states = _f64(states)
    for i, (slot, r) in enumerate(zip(np.asarray(slots), np.asarray(accepted))):
        if r >= 1:
            pool[int(slot)] = states[i, int(r) - 1]
    return pool
