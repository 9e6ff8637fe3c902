"""Thin ctypes binding of libgdn_dual.so (the C ABI in include/gdn_dual.h).

Argument marshalling only: every step of the forward runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.  There is no fallback: if the
library is missing or cannot load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn_dual.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_ALIGNMENT, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, GDN_ERR_BOUNDS = range(7)
GDN_BF16, GDN_FP32 = 0, 1
ALGO_AUTO, ALGO_SEQUENTIAL, ALGO_CHUNKED, ALGO_ROUTE1, ALGO_PIPELINED = 0, 1, 2, 3, 4
EXPORTED = ("gdn_dual_forward", "gdn_dual_workspace_size", "gdn_dual_read_device_status",
            "gdn_status_string", "gdn_dual_version", "gdn_dual_select_algo",
            "gdn_decode_replay", "gdn_decode_verify", "gdn_decode_commit", "gdn_dual_workspace_size_route1",
            "gdn_attn_forward", "gdn_attn_workspace_size", "gdn_dual_backward",
            "gdn_dual_backward_workspace_size", "gdn_dual_forward_noalloc",
            "gdn_dual_noalloc_read_device_status", "gdn_dual_forward_test_wait_limit",
            "gdn_dual_read_device_status_where", "gdn_attn_forward_test_wait_limit",
            "gdn_dual_backward_conv", "gdn_dual_backward_conv_workspace_size",
            "gdn_dual_forward_host", "gdn_dual_host_staging_size", "gdn_dual_host_read_device_status")


class GdnError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


class Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("num_docs", "num_heads", "d_k", "d_v", "num_views",
                                               "block_size", "dtype", "conv_width", "algo", "reserved")]


class DecodeDesc(ctypes.Structure):
    """gdn_decode_desc of include/gdn_decode.h."""
    _fields_ = [(n, ctypes.c_int32) for n in ("num_seqs", "num_heads", "d_k", "d_v", "num_tokens",
                                               "pool_slots", "dtype", "reserved")]


class AttnDesc(ctypes.Structure):
    """gdn_attn_desc of include/gdn_attention.h."""
    _fields_ = [(n, ctypes.c_int32) for n in ("num_docs", "num_heads", "num_kv_heads", "head_dim", "num_views",
                                               "block_size", "dtype", "reserved")]


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library (raises OSError if it is missing; nothing falls back)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise OSError(f"{path} not found: build it with `python -m gated_deltanet_dual_b200.build`")
            lib = ctypes.CDLL(path)
            vp, fp, ip = ctypes.c_void_p, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32)
            lib.gdn_dual_forward.restype = ctypes.c_int
            lib.gdn_dual_forward.argtypes = [ctypes.POINTER(Desc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                             ip, ip, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
            lib.gdn_dual_workspace_size.restype = ctypes.c_size_t
            lib.gdn_dual_workspace_size.argtypes = [ctypes.POINTER(Desc), ip]
            lib.gdn_dual_workspace_size_route1.restype = ctypes.c_size_t
            lib.gdn_dual_workspace_size_route1.argtypes = [ctypes.POINTER(Desc), ip, ip]
            lib.gdn_dual_read_device_status.restype = ctypes.c_int
            lib.gdn_dual_read_device_status.argtypes = [vp, vp]
            lib.gdn_status_string.restype = ctypes.c_char_p
            lib.gdn_status_string.argtypes = [ctypes.c_int]
            lib.gdn_dual_version.restype = ctypes.c_int32
            lib.gdn_dual_select_algo.restype = ctypes.c_int32
            lib.gdn_dual_select_algo.argtypes = [ctypes.POINTER(Desc)]
            dd = ctypes.POINTER(DecodeDesc)
            for name in ("gdn_decode_replay", "gdn_decode_verify", "gdn_decode_commit"):
                getattr(lib, name).restype = ctypes.c_int
            lib.gdn_decode_replay.argtypes = [dd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            lib.gdn_decode_verify.argtypes = [dd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            lib.gdn_decode_commit.argtypes = [dd, vp, vp, vp, vp, vp, vp]
            lib.gdn_dual_backward_workspace_size.restype = ctypes.c_size_t
            lib.gdn_dual_backward_workspace_size.argtypes = [ctypes.POINTER(Desc), ip]
            lib.gdn_dual_backward.restype = ctypes.c_int
            lib.gdn_dual_backward.argtypes = ([ctypes.POINTER(Desc)] + [vp] * 10 + [ip, ip] + [vp] * 3 + [vp] * 10
                                              + [vp, ctypes.c_size_t, vp])
            ad = ctypes.POINTER(AttnDesc)
            lib.gdn_attn_workspace_size.restype = ctypes.c_size_t
            lib.gdn_attn_workspace_size.argtypes = [ad, ip, ip]
            lib.gdn_attn_forward.restype = ctypes.c_int
            lib.gdn_attn_forward.argtypes = [ad, vp, vp, vp, vp, vp, vp, ip, ip, vp, vp, vp, ctypes.c_size_t, vp]
            lib.gdn_dual_host_staging_size.restype = ctypes.c_size_t
            lib.gdn_dual_host_staging_size.argtypes = [ctypes.POINTER(Desc), ip, ip, ctypes.c_int32]
            lib.gdn_dual_forward_host.restype = ctypes.c_int
            lib.gdn_dual_forward_host.argtypes = ([ctypes.POINTER(Desc)] + [vp] * 10 + [ip, ip, vp, vp, vp, vp, vp,
                                                  ctypes.c_size_t, ctypes.c_int32, vp])
            lib.gdn_dual_host_read_device_status.restype = ctypes.c_int
            lib.gdn_dual_host_read_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32), vp]
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load_library().gdn_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_FP32
    raise TypeError(f"unsupported I/O dtype {t.dtype}")


def make_desc(num_docs, num_heads, d_k, d_v, num_views, block_size, dtype_code, conv_width=0, algo=ALGO_AUTO):
    return Desc(num_docs, num_heads, d_k, d_v, num_views, block_size, dtype_code, conv_width, algo, 0)


def _host_i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def workspace_size(desc: Desc, doc_offsets) -> int:
    offs = _host_i32(doc_offsets)
    return int(load_library().gdn_dual_workspace_size(ctypes.byref(desc),
                                                      offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))))


def workspace_size_route1(desc: Desc, doc_offsets, prompt_len) -> int:
    """Workspace bytes for ALGO_ROUTE1 (header plus the materialised block-boundary states)."""
    offs, pl = _host_i32(doc_offsets), _host_i32(prompt_len)
    ip = ctypes.POINTER(ctypes.c_int32)
    return int(load_library().gdn_dual_workspace_size_route1(ctypes.byref(desc), offs.ctypes.data_as(ip),
                                                             pl.ctypes.data_as(ip)))


def select_algo(desc: Desc) -> int:
    return int(load_library().gdn_dual_select_algo(ctypes.byref(desc)))


def forward_raw(desc: Desc, q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, conv_w,
                out, out_noisy, final_state, workspace, stream=None) -> int:
    """Direct C-ABI call with tensors (or None) for every pointer; returns the status code."""
    lib = load_library()
    offs = _host_i32(doc_offsets)
    pl = _host_i32(prompt_len)
    ip = ctypes.POINTER(ctypes.c_int32)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return int(lib.gdn_dual_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                    _ptr(qn), _ptr(kn), _ptr(vn), _ptr(gn), _ptr(betan),
                                    offs.ctypes.data_as(ip), pl.ctypes.data_as(ip), _ptr(conv_w),
                                    _ptr(out), _ptr(out_noisy), _ptr(final_state),
                                    _ptr(workspace), ctypes.c_size_t(ws_bytes), ctypes.c_void_p(stream)))


def forward_test_wait_limit_raw(desc: Desc, q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len,
                                conv_w, out, out_noisy, final_state, workspace, wait_iters: int, stream=None) -> int:
    """C-ABI call of gdn_dual_forward_test_wait_limit (tests of the bounded-wait error path only:
    every device-side wait is bounded by `wait_iters` try-waits).  Returns the status code."""
    lib = load_library()
    fn = lib.gdn_dual_forward_test_wait_limit
    vp, ip = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(Desc)] + [vp] * 10 + [ip, ip] + [vp] * 5 + [ctypes.c_size_t, ctypes.c_uint32, vp]
    offs = _host_i32(doc_offsets)
    pl = _host_i32(prompt_len)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    ws_bytes = workspace.numel() * workspace.element_size()
    return int(fn(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(qn), _ptr(kn), _ptr(vn),
                  _ptr(gn), _ptr(betan), offs.ctypes.data_as(ip), pl.ctypes.data_as(ip), _ptr(conv_w),
                  _ptr(out), _ptr(out_noisy), _ptr(final_state), _ptr(workspace), ctypes.c_size_t(ws_bytes),
                  ctypes.c_uint32(wait_iters), ctypes.c_void_p(stream)))


def read_device_status_where(workspace_tensor, stream=None):
    """(status, where): the device-side status word of a workspace and the diagnostic code of the
    wait that gave up (0 when none did).  Synchronises the stream."""
    lib = load_library()
    fn = lib.gdn_dual_read_device_status_where
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p]
    where = ctypes.c_int32(0)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    st = int(fn(_ptr(workspace_tensor), ctypes.byref(where), ctypes.c_void_p(stream)))
    return st, int(where.value)


class Workspace:
    """Caller-owned device scratch for gdn_dual_forward (allocated by torch, reused)."""

    def __init__(self, nbytes: int, device="cuda"):
        self.tensor = torch.zeros(max(256, (nbytes + 255) // 256 * 256), dtype=torch.uint8, device=device)


def _check(t: Optional[torch.Tensor], name: str, shape, dtype, device):
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype} != {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def forward(q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, block_size,
            conv_w=None, *, algo: int = ALGO_AUTO, out=None, out_noisy=None, final_state=None,
            workspace: Optional[Workspace] = None, stream=None):
    """Dual-stream Gated DeltaNet forward on the GPU.

    Shapes: q, k [T,H,d]; v [T,H,d]; g, beta [T,H] fp32; qn, kn, vn [V,T_R,H,d]; gn, betan
    [V,T_R,H] fp32; conv_w [3,H*d,4] fp32 or None; doc_offsets [N+1], prompt_len [N] host ints.
    Returns (out [T,H,d], out_noisy [V,T_R,H,d], final_state [N,H,d,d] fp32)."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    T, H, dk = q.shape
    dv = v.shape[2]
    V, TR = qn.shape[0], qn.shape[1]
    offs = _host_i32(doc_offsets)
    pl = _host_i32(prompt_len)
    N = offs.shape[0] - 1
    io = q.dtype
    f32 = torch.float32
    if offs.ndim != 1 or pl.shape != (N,):
        raise ValueError("doc_offsets must be [N+1] and prompt_len [N]")
    if N >= 1 and int(offs[-1]) != T:
        raise ValueError(f"doc_offsets[-1] = {int(offs[-1])} but q has {T} tokens")
    if N >= 1 and int((np.diff(offs.astype(np.int64)) - pl).sum()) != TR:
        raise ValueError(f"noisy tensors have {TR} rows but the documents have "
                         f"{int((np.diff(offs.astype(np.int64)) - pl).sum())} response tokens")
    for t, name, shape, dt in ((q, "q", (T, H, dk), io), (k, "k", (T, H, dk), io), (v, "v", (T, H, dv), io),
                               (g, "g", (T, H), f32), (beta, "beta", (T, H), f32),
                               (qn, "qn", (V, TR, H, dk), io), (kn, "kn", (V, TR, H, dk), io),
                               (vn, "vn", (V, TR, H, dv), io), (gn, "gn", (V, TR, H), f32),
                               (betan, "betan", (V, TR, H), f32)):
        _check(t, name, shape, dt, dev)
    conv_width = 0
    if conv_w is not None:
        conv_width = int(conv_w.shape[-1])
        _check(conv_w, "conv_w", (3, H * dk, conv_width), f32, dev)
    if out is None:
        out = torch.empty(T, H, dv, dtype=io, device=dev)
    if out_noisy is None:
        out_noisy = torch.empty(V, TR, H, dv, dtype=io, device=dev)
    if final_state is None:
        final_state = torch.empty(N, H, dk, dv, dtype=f32, device=dev)
    _check(out, "out", (T, H, dv), io, dev)
    _check(out_noisy, "out_noisy", (V, TR, H, dv), io, dev)
    _check(final_state, "final_state", (N, H, dk, dv), f32, dev)
    desc = make_desc(N, H, dk, dv, V, int(block_size), _dtype_code(q), conv_width, algo)
    ws_tensor = workspace.tensor if workspace is not None else None
    if workspace is None:
        nbytes = workspace_size_route1(desc, offs, pl) if algo == ALGO_ROUTE1 else workspace_size(desc, offs)
        # size 0: the descriptor or the layout is invalid; the library's own validation below
        # then returns the status (nothing launches)
        if nbytes:
            ws_tensor = Workspace(nbytes, device=dev).tensor
    st = forward_raw(desc, q, k, v, g, beta, qn, kn, vn, gn, betan, offs, pl, conv_w,
                     out, out_noisy, final_state, ws_tensor, stream=stream)
    if st != GDN_OK:
        raise GdnError(st, f"gdn_dual_forward failed: {status_string(st)}")
    return out, out_noisy, final_state


def read_device_status(workspace: Workspace, stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return int(load_library().gdn_dual_read_device_status(_ptr(workspace.tensor), ctypes.c_void_p(stream)))


def host_staging_size(desc: Desc, doc_offsets, prompt_len, groups: int) -> int:
    """Device staging bytes gdn_dual_forward_host needs (0: invalid descriptor or layout)."""
    offs, pl = _host_i32(doc_offsets), _host_i32(prompt_len)
    ip = ctypes.POINTER(ctypes.c_int32)
    return int(load_library().gdn_dual_host_staging_size(ctypes.byref(desc), offs.ctypes.data_as(ip),
                                                         pl.ctypes.data_as(ip), int(groups)))


def forward_host_raw(desc: Desc, q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, conv_w,
                     out, out_noisy, final_state, staging: torch.Tensor, groups: int, stream=None) -> int:
    """C-ABI call of gdn_dual_forward_host: every tensor argument is a (pinned) CPU tensor, `staging`
    a CUDA byte tensor of host_staging_size() bytes.  Returns the status code; the outputs are in
    host memory once `stream` is synchronised."""
    lib = load_library()
    offs, pl = _host_i32(doc_offsets), _host_i32(prompt_len)
    ip = ctypes.POINTER(ctypes.c_int32)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return int(lib.gdn_dual_forward_host(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                         _ptr(qn), _ptr(kn), _ptr(vn), _ptr(gn), _ptr(betan),
                                         offs.ctypes.data_as(ip), pl.ctypes.data_as(ip), _ptr(conv_w),
                                         _ptr(out), _ptr(out_noisy), _ptr(final_state), _ptr(staging),
                                         ctypes.c_size_t(staging.numel()), int(groups), ctypes.c_void_p(stream)))


def read_host_device_status(staging: torch.Tensor, stream=None):
    """(status, where) recorded by the groups of the last gdn_dual_forward_host on `staging`."""
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    where = ctypes.c_int32(0)
    st = int(load_library().gdn_dual_host_read_device_status(_ptr(staging), ctypes.byref(where),
                                                             ctypes.c_void_p(stream)))
    return st, int(where.value)


def forward_problem(prob, **kw):
    """Run the forward on a synthetic problem whose tensors live on the GPU."""
    return forward(prob.q, prob.k, prob.v, prob.g, prob.beta, prob.qn, prob.kn, prob.vn, prob.gn,
                   prob.betan, prob.doc_offsets, prob.prompt_len, prob.block_size, conv_w=prob.conv_w, **kw)


def forward_noalloc_raw(desc: Desc, q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, conv_w,
                        out, out_noisy, final_state, stream=None) -> int:
    """C-ABI call of gdn_dual_forward_noalloc (no workspace: the library's fixed device scratch
    is used, for callers that cannot allocate).  Returns the status code."""
    lib = load_library()
    fn = lib.gdn_dual_forward_noalloc
    vp, ip = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(Desc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ip, ip, vp, vp, vp, vp, vp]
    offs = _host_i32(doc_offsets)
    pl = _host_i32(prompt_len)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return int(fn(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(qn), _ptr(kn), _ptr(vn),
                  _ptr(gn), _ptr(betan), offs.ctypes.data_as(ip), pl.ctypes.data_as(ip), _ptr(conv_w),
                  _ptr(out), _ptr(out_noisy), _ptr(final_state), ctypes.c_void_p(stream)))


def noalloc_read_device_status(stream=None) -> int:
    """C-ABI call of gdn_dual_noalloc_read_device_status: the device-side status of the last
    gdn_dual_forward_noalloc on the current device (synchronises the stream)."""
    lib = load_library()
    fn = lib.gdn_dual_noalloc_read_device_status
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p]
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return int(fn(ctypes.c_void_p(stream)))


# ----------------------------------------------------------------------------- decode side
def make_decode_desc(num_seqs, num_heads, d_k, d_v, num_tokens, pool_slots, dtype_code) -> DecodeDesc:
    return DecodeDesc(num_seqs, num_heads, d_k, d_v, num_tokens, pool_slots, dtype_code, 0)


def _decode_args(state_pool, slots, q, k, v, g, beta):
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    N, L, H, dk = q.shape
    dv = v.shape[3]
    P = state_pool.shape[0]
    io, f32 = q.dtype, torch.float32
    for t, name, shape, dt in ((state_pool, "state_pool", (P, H, dk, dv), f32), (slots, "slots", (N,), torch.int32),
                               (q, "q", (N, L, H, dk), io), (k, "k", (N, L, H, dk), io), (v, "v", (N, L, H, dv), io),
                               (g, "g", (N, L, H), f32), (beta, "beta", (N, L, H), f32)):
        _check(t, name, shape, dt, dev)
    return make_decode_desc(N, H, dk, dv, L, P, _dtype_code(q)), dev, (N, L, H, dk, dv)


def _stream(stream):
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream if stream is None else stream)


def decode_replay(state_pool, slots, q, k, v, g, beta, *, out=None, device_status=None, stream=None):
    """Causal replay of a committed block (gdn_decode_replay): runs the L tokens of every sequence
    from its pooled state, writes the outputs and the final state back into state_pool[slots]."""
    desc, dev, (N, L, H, dk, dv) = _decode_args(state_pool, slots, q, k, v, g, beta)
    if out is None:
        out = torch.empty(N, L, H, dv, dtype=q.dtype, device=dev)
    _check(out, "out", (N, L, H, dv), q.dtype, dev)
    st = load_library().gdn_decode_replay(ctypes.byref(desc), _ptr(state_pool), _ptr(slots), _ptr(q), _ptr(k),
                                          _ptr(v), _ptr(g), _ptr(beta), _ptr(out), _ptr(device_status),
                                          _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, f"gdn_decode_replay failed: {status_string(st)}")
    return out


def decode_verify(state_pool, slots, q, k, v, g, beta, *, out=None, state_cache=None, device_status=None,
                  stream=None):
    """Verify forward with state cache (gdn_decode_verify): outputs of the L candidates and the
    state after each step in state_cache [N, L, H, d_k, d_v]; the pool is only read."""
    desc, dev, (N, L, H, dk, dv) = _decode_args(state_pool, slots, q, k, v, g, beta)
    if out is None:
        out = torch.empty(N, L, H, dv, dtype=q.dtype, device=dev)
    if state_cache is None:
        state_cache = torch.empty(N, L, H, dk, dv, dtype=torch.float32, device=dev)
    _check(out, "out", (N, L, H, dv), q.dtype, dev)
    _check(state_cache, "state_cache", (N, L, H, dk, dv), torch.float32, dev)
    st = load_library().gdn_decode_verify(ctypes.byref(desc), _ptr(state_pool), _ptr(slots), _ptr(q), _ptr(k),
                                          _ptr(v), _ptr(g), _ptr(beta), _ptr(out), _ptr(state_cache),
                                          _ptr(device_status), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, f"gdn_decode_verify failed: {status_string(st)}")
    return out, state_cache


def decode_commit(state_pool, slots, state_cache, accepted, *, device_status=None, stream=None):
    """Commit the accepted prefix (gdn_decode_commit): state_pool[slots[n]] := state_cache[n, r-1]
    for r = accepted[n] >= 1."""
    dev = state_pool.device
    N, L, H, dk, dv = state_cache.shape
    P = state_pool.shape[0]
    for t, name, shape, dt in ((state_pool, "state_pool", (P, H, dk, dv), torch.float32),
                               (slots, "slots", (N,), torch.int32), (accepted, "accepted", (N,), torch.int32),
                               (state_cache, "state_cache", (N, L, H, dk, dv), torch.float32)):
        _check(t, name, shape, dt, dev)
    desc = make_decode_desc(N, H, dk, dv, L, P, GDN_FP32)
    st = load_library().gdn_decode_commit(ctypes.byref(desc), _ptr(state_pool), _ptr(slots), _ptr(state_cache),
                                          _ptr(accepted), _ptr(device_status), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, f"gdn_decode_commit failed: {status_string(st)}")
    return state_pool


# ----------------------------------------------------------------------------- softmax attention
def make_attn_desc(num_docs, num_heads, num_kv_heads, head_dim, num_views, block_size, dtype_code) -> AttnDesc:
    return AttnDesc(num_docs, num_heads, num_kv_heads, head_dim, num_views, block_size, dtype_code, 0)


def attn_workspace_size(desc: AttnDesc, doc_offsets, prompt_len) -> int:
    offs = np.ascontiguousarray(doc_offsets, dtype=np.int32)
    pl = np.ascontiguousarray(prompt_len, dtype=np.int32)
    ip = ctypes.POINTER(ctypes.c_int32)
    return int(load_library().gdn_attn_workspace_size(ctypes.byref(desc), offs.ctypes.data_as(ip),
                                                      pl.ctypes.data_as(ip)))


def attention_forward(q, k, v, qn, kn, vn, doc_offsets, prompt_len, block_size, *, out=None, out_noisy=None,
                      workspace=None, stream=None):
    """Dual-stream softmax attention with the document-blocked causal / block-bidirectional mask
    (gdn_attn_forward).  q [T, H, d], k and v [T, H_kv, d]; qn [V, T_R, H, d], kn and vn
    [V, T_R, H_kv, d]; doc_offsets [N+1] and prompt_len [N] on the host.  Returns (out, out_noisy)."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    T, H, d = q.shape
    Hkv = k.shape[1]
    V, TR = qn.shape[0], qn.shape[1]
    offs = np.ascontiguousarray(doc_offsets, dtype=np.int32)
    pl = np.ascontiguousarray(prompt_len, dtype=np.int32)
    N = len(pl)
    if offs.ndim != 1 or offs.shape[0] != N + 1:
        raise ValueError("doc_offsets must be [N+1] and prompt_len [N]")
    if N >= 1 and int(offs[-1]) != T:
        raise ValueError(f"doc_offsets[-1] = {int(offs[-1])} but q has {T} tokens")
    if N >= 1 and int((np.diff(offs.astype(np.int64)) - pl).sum()) != TR:
        raise ValueError(f"noisy tensors have {TR} rows but the documents have "
                         f"{int((np.diff(offs.astype(np.int64)) - pl).sum())} response tokens")
    io = q.dtype
    for t, name, shape in ((q, "q", (T, H, d)), (k, "k", (T, Hkv, d)), (v, "v", (T, Hkv, d)),
                           (qn, "qn", (V, TR, H, d)), (kn, "kn", (V, TR, Hkv, d)), (vn, "vn", (V, TR, Hkv, d))):
        _check(t, name, shape, io, dev)
    if out is None:
        out = torch.empty(T, H, d, dtype=io, device=dev)
    if out_noisy is None:
        out_noisy = torch.empty(V, TR, H, d, dtype=io, device=dev)
    _check(out, "out", (T, H, d), io, dev)
    _check(out_noisy, "out_noisy", (V, TR, H, d), io, dev)
    desc = make_attn_desc(N, H, Hkv, d, V, int(block_size), _dtype_code(q))
    ws = workspace
    if ws is None:
        nbytes = attn_workspace_size(desc, offs, pl)
        if nbytes:
            ws = Workspace(nbytes, device=dev).tensor
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    ip = ctypes.POINTER(ctypes.c_int32)
    noisy = V > 0 and TR > 0
    st = load_library().gdn_attn_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(qn) if noisy else None, _ptr(kn) if noisy else None,
                                         _ptr(vn) if noisy else None, offs.ctypes.data_as(ip), pl.ctypes.data_as(ip),
                                         _ptr(out), _ptr(out_noisy) if noisy else None, _ptr(ws),
                                         ctypes.c_size_t(ws_bytes), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, f"gdn_attn_forward failed: {status_string(st)}")
    return out, out_noisy


def attention_forward_test_wait_limit_raw(desc, q, k, v, qn, kn, vn, doc_offsets, prompt_len, out, out_noisy,
                                          workspace, wait_iters: int, stream=None) -> int:
    """C-ABI call of gdn_attn_forward_test_wait_limit (tests of the bounded-wait error path only).
    Returns the status code."""
    lib = load_library()
    fn = lib.gdn_attn_forward_test_wait_limit
    vp, ip = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(AttnDesc)] + [vp] * 6 + [ip, ip] + [vp] * 3 + [ctypes.c_size_t, ctypes.c_uint32, vp]
    offs = np.ascontiguousarray(doc_offsets, dtype=np.int32)
    pl = np.ascontiguousarray(prompt_len, dtype=np.int32)
    ws_bytes = workspace.numel() * workspace.element_size()
    return int(fn(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(qn), _ptr(kn), _ptr(vn),
                  offs.ctypes.data_as(ip), pl.ctypes.data_as(ip), _ptr(out), _ptr(out_noisy), _ptr(workspace),
                  ctypes.c_size_t(ws_bytes), ctypes.c_uint32(wait_iters), _stream(stream)))


# ----------------------------------------------------------------------------- backward
def backward_workspace_size(desc: Desc, doc_offsets) -> int:
    offs = np.ascontiguousarray(doc_offsets, dtype=np.int32)
    return int(load_library().gdn_dual_backward_workspace_size(ctypes.byref(desc),
                                                                offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))))


def backward(q, k, v, g, beta, qn, kn, vn, gn, betan, doc_offsets, prompt_len, block_size, d_out, d_out_noisy,
             d_final_state=None, *, conv_w=None, workspace=None, stream=None):
    """Gradients of <d_out, out> + <d_out_noisy, out_noisy> + <d_final_state, final_state> with
    respect to every input of the dual-stream forward, fp32 (gdn_dual_backward; with conv_w, the
    width-4 ShortConv prologue: gdn_dual_backward_conv, gradients of the raw inputs plus dconv_w).
    Returns a dict dq, dk, dv, dg, dbeta, dqn, dkn, dvn, dgn, dbetan (and dconv_w)."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    T, H, dk_ = q.shape
    dv_ = v.shape[2]
    V, TR = qn.shape[0], qn.shape[1]
    offs = np.ascontiguousarray(doc_offsets, dtype=np.int32)
    pl = np.ascontiguousarray(prompt_len, dtype=np.int32)
    N = len(pl)
    if offs.shape != (N + 1,) or (N >= 1 and int(offs[-1]) != T):
        raise ValueError("doc_offsets must be [N+1] and end at T")
    if N >= 1 and int((np.diff(offs.astype(np.int64)) - pl).sum()) != TR:
        raise ValueError("noisy tensors do not match the documents' response tokens")
    io, f32 = q.dtype, torch.float32
    for t, name, shape, dt in ((q, "q", (T, H, dk_), io), (k, "k", (T, H, dk_), io), (v, "v", (T, H, dv_), io),
                               (g, "g", (T, H), f32), (beta, "beta", (T, H), f32),
                               (qn, "qn", (V, TR, H, dk_), io), (kn, "kn", (V, TR, H, dk_), io),
                               (vn, "vn", (V, TR, H, dv_), io), (gn, "gn", (V, TR, H), f32),
                               (betan, "betan", (V, TR, H), f32), (d_out, "d_out", (T, H, dv_), io),
                               (d_out_noisy, "d_out_noisy", (V, TR, H, dv_), io),
                               (d_final_state, "d_final_state", (N, H, dk_, dv_), f32)):
        _check(t, name, shape, dt, dev)
    conv_width = 0
    if conv_w is not None:
        conv_width = int(conv_w.shape[-1])
        _check(conv_w, "conv_w", (3, H * dk_, conv_width), f32, dev)
    out = {n: torch.empty(x.shape, dtype=f32, device=dev) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g),
                                                                         ("dbeta", beta), ("dqn", qn), ("dkn", kn),
                                                                         ("dvn", vn), ("dgn", gn), ("dbetan", betan))}
    desc = make_desc(N, H, dk_, dv_, V, int(block_size), _dtype_code(q), conv_width)
    lib = load_library()
    ws = workspace
    if ws is None:
        nbytes = backward_workspace_size(desc, offs) if conv_w is None else backward_conv_workspace_size(desc, offs)
        if nbytes:
            ws = Workspace(nbytes, device=dev).tensor
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    noisy = V > 0 and TR > 0
    nz = lambda t: _ptr(t) if noisy else None
    ip = ctypes.POINTER(ctypes.c_int32)
    head = [ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), nz(qn), nz(kn), nz(vn), nz(gn),
            nz(betan), offs.ctypes.data_as(ip), pl.ctypes.data_as(ip)]
    grads = [_ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
             nz(out["dqn"]), nz(out["dkn"]), nz(out["dvn"]), nz(out["dgn"]), nz(out["dbetan"])]
    ups = [_ptr(d_out), nz(d_out_noisy), _ptr(d_final_state)]
    if conv_w is None:
        st = lib.gdn_dual_backward(*head, *ups, *grads, _ptr(ws), ctypes.c_size_t(ws_bytes), _stream(stream))
        name = "gdn_dual_backward"
    else:
        out["dconv_w"] = torch.empty_like(conv_w)
        fn = lib.gdn_dual_backward_conv
        fn.restype = ctypes.c_int
        vp = ctypes.c_void_p
        fn.argtypes = [ctypes.POINTER(Desc)] + [vp] * 10 + [ip, ip] + [vp] * 4 + [vp] * 10 + [vp, vp, ctypes.c_size_t, vp]
        st = fn(*head, _ptr(conv_w), *ups, *grads, _ptr(out["dconv_w"]), _ptr(ws), ctypes.c_size_t(ws_bytes),
                _stream(stream))
        name = "gdn_dual_backward_conv"
    if st != GDN_OK:
        raise GdnError(st, f"{name} failed: {status_string(st)}")
    return out


def backward_conv_workspace_size(desc: Desc, doc_offsets) -> int:
    offs = np.ascontiguousarray(doc_offsets, dtype=np.int32)
    fn = load_library().gdn_dual_backward_conv_workspace_size
    fn.restype = ctypes.c_size_t
    fn.argtypes = [ctypes.POINTER(Desc), ctypes.POINTER(ctypes.c_int32)]
    return int(fn(ctypes.byref(desc), offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))))
