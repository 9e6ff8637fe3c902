"""C-ABI library: loads, exports every declared symbol, validates on the host (CPU only).

The error-path cases here pass placeholder addresses that the host validation must reject
before anything is enqueued; they never run where a GPU is visible."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from gated_deltanet_dual_b200 import binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]

no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers: host-only check")


def declared_functions():
    src = "\n".join(open(h).read() for h in HEADERS)
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(gdn_[a-z0-9_]+)\s*\(",
                                 src, flags=re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    assert "gdn_dual_forward" in names and "gdn_dual_workspace_size" in names
    assert {"gdn_decode_replay", "gdn_decode_verify", "gdn_decode_commit"} <= set(names)
    assert set(b.EXPORTED) <= set(names)


def test_library_exports_every_declared_symbol():
    lib = b.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_range_checking_build_exports_every_declared_symbol():
    """libgdn_dual_debug.so (GDN_DEBUG_BOUNDS) is a drop-in replacement: same C ABI."""
    import ctypes
    from gated_deltanet_dual_b200 import build as gbuild
    lib = ctypes.CDLL(gbuild.build_debug())
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported by the range-checking build"


def test_version_and_status_strings():
    lib = b.load_library()
    assert lib.gdn_dual_version() >= 100
    for code, name in enumerate(["GDN_OK", "GDN_ERR_INVALID_ARG", "GDN_ERR_ALIGNMENT", "GDN_ERR_UNSUPPORTED",
                                 "GDN_ERR_CUDA", "GDN_ERR_TIMEOUT", "GDN_ERR_BOUNDS"]):
        assert b.status_string(code) == name
    assert b.status_string(99) == "GDN_ERR_UNKNOWN"


def test_workspace_size_and_algo_selection():
    d = b.make_desc(2, 4, 128, 128, 2, 4, b.GDN_BF16)
    assert b.workspace_size(d, [0, 64, 128]) >= 256
    assert b.workspace_size(d, [0, 64, 32]) == 0          # non-monotone
    assert b.workspace_size(d, [1, 64, 128]) == 0         # must start at 0
    assert b.select_algo(b.make_desc(1, 2, 32, 32, 2, 4, b.GDN_FP32)) == b.ALGO_SEQUENTIAL
    assert b.select_algo(b.make_desc(1, 2, 32, 32, 2, 4, b.GDN_FP32, algo=7)) == -1


class _Fake:
    """Stands in for a tensor: a placeholder device address (never dereferenced)."""
    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def _call(desc, offs, pl, **over):
    base = 0x7f0000000000
    names = ["q", "k", "v", "g", "beta", "qn", "kn", "vn", "gn", "betan", "conv_w",
             "out", "out_noisy", "final_state", "workspace"]
    ptr = {n: _Fake(base + 0x10000000 * i) for i, n in enumerate(names)}
    ptr["conv_w"] = None
    ptr.update(over)
    lib = b.load_library()
    ip = ctypes.POINTER(ctypes.c_int32)
    offs = np.ascontiguousarray(offs, dtype=np.int32)
    pl = np.ascontiguousarray(pl, dtype=np.int32)
    p = lambda n: None if ptr[n] is None else ctypes.c_void_p(ptr[n].data_ptr())
    ws_bytes = over.get("_ws_bytes", 256)
    return lib.gdn_dual_forward(ctypes.byref(desc), p("q"), p("k"), p("v"), p("g"), p("beta"),
                                p("qn"), p("kn"), p("vn"), p("gn"), p("betan"),
                                offs.ctypes.data_as(ip), pl.ctypes.data_as(ip), p("conv_w"),
                                p("out"), p("out_noisy"), p("final_state"), p("workspace"),
                                ctypes.c_size_t(ws_bytes), None)


@no_gpu
@pytest.mark.parametrize("case,expect", [
    ("offsets_not_from_zero", b.GDN_ERR_INVALID_ARG),
    ("offsets_decreasing", b.GDN_ERR_INVALID_ARG),
    ("prompt_longer_than_doc", b.GDN_ERR_INVALID_ARG),
    ("negative_prompt", b.GDN_ERR_INVALID_ARG),
    ("response_not_multiple_of_B", b.GDN_ERR_INVALID_ARG),
    ("null_q", b.GDN_ERR_INVALID_ARG),
    ("null_noisy", b.GDN_ERR_INVALID_ARG),
    ("null_final_state", b.GDN_ERR_INVALID_ARG),
    ("conv_without_weights", b.GDN_ERR_INVALID_ARG),
    ("workspace_too_small", b.GDN_ERR_INVALID_ARG),
    ("null_workspace", b.GDN_ERR_INVALID_ARG),
    ("misaligned_k", b.GDN_ERR_ALIGNMENT),
    ("misaligned_out", b.GDN_ERR_ALIGNMENT),
    ("unsupported_d", b.GDN_ERR_UNSUPPORTED),
    ("unequal_dk_dv", b.GDN_ERR_UNSUPPORTED),
    ("unsupported_conv_width", b.GDN_ERR_UNSUPPORTED),
    ("bad_dtype", b.GDN_ERR_INVALID_ARG),
    ("zero_docs", b.GDN_ERR_INVALID_ARG),
    ("zero_block", b.GDN_ERR_INVALID_ARG),
    ("reserved_nonzero", b.GDN_ERR_INVALID_ARG),
    ("too_many_docs", b.GDN_ERR_UNSUPPORTED),
])
def test_host_validation_rejects(case, expect):
    d = b.make_desc(2, 2, 32, 32, 2, 4, b.GDN_FP32)
    offs, pl = [0, 16, 40], [8, 4]
    kw = {}
    if case == "offsets_not_from_zero":
        offs = [4, 16, 40]
    elif case == "offsets_decreasing":
        offs = [0, 16, 12]
    elif case == "prompt_longer_than_doc":
        pl = [20, 4]
    elif case == "negative_prompt":
        pl = [-4, 4]
    elif case == "response_not_multiple_of_B":
        pl = [7, 4]
    elif case == "null_q":
        kw["q"] = None
    elif case == "null_noisy":
        kw["vn"] = None
    elif case == "null_final_state":
        kw["final_state"] = None
    elif case == "conv_without_weights":
        d = b.make_desc(2, 2, 32, 32, 2, 4, b.GDN_FP32, conv_width=4)
    elif case == "workspace_too_small":
        kw["_ws_bytes"] = 64
    elif case == "null_workspace":
        kw["workspace"] = None
    elif case == "misaligned_k":
        kw["k"] = _Fake(0x7f0000000008)
    elif case == "misaligned_out":
        kw["out"] = _Fake(0x7f0000000004)
    elif case == "unsupported_d":
        d = b.make_desc(2, 2, 48, 48, 2, 4, b.GDN_FP32)
    elif case == "unequal_dk_dv":
        d = b.make_desc(2, 2, 64, 32, 2, 4, b.GDN_FP32)
    elif case == "unsupported_conv_width":
        d = b.make_desc(2, 2, 32, 32, 2, 4, b.GDN_FP32, conv_width=3)
        kw["conv_w"] = _Fake(0x7f0000000000)
    elif case == "bad_dtype":
        d = b.make_desc(2, 2, 32, 32, 2, 4, 5)
    elif case == "zero_docs":
        d = b.make_desc(0, 2, 32, 32, 2, 4, b.GDN_FP32)
        offs, pl = [0], []
    elif case == "zero_block":
        d = b.make_desc(2, 2, 32, 32, 2, 0, b.GDN_FP32)
    elif case == "reserved_nonzero":
        d = b.make_desc(2, 2, 32, 32, 2, 4, b.GDN_FP32)
        d.reserved = 1
    elif case == "too_many_docs":
        n = 1025
        d = b.make_desc(n, 1, 32, 32, 0, 4, b.GDN_FP32)
        offs, pl = list(range(0, 4 * (n + 1), 4)), [0] * n
    assert _call(d, offs, pl, **kw) == expect


@no_gpu
def test_valid_arguments_without_device_report_cuda_error():
    """All arguments valid, no GPU visible: the first CUDA call fails and maps to GDN_ERR_CUDA
    (no crash, no abort)."""
    d = b.make_desc(2, 2, 32, 32, 2, 4, b.GDN_FP32)
    assert _call(d, [0, 16, 40], [8, 4]) == b.GDN_ERR_CUDA


def test_auto_selects_tensor_core_kernel_where_supported():
    assert b.select_algo(b.make_desc(2, 16, 128, 128, 2, 4, b.GDN_BF16)) == b.ALGO_CHUNKED
    assert b.select_algo(b.make_desc(2, 16, 128, 128, 2, 32, b.GDN_BF16)) == b.ALGO_CHUNKED
    assert b.select_algo(b.make_desc(2, 16, 128, 128, 2, 4, b.GDN_BF16, conv_width=4)) == b.ALGO_CHUNKED
    assert b.select_algo(b.make_desc(2, 16, 128, 128, 2, 64, b.GDN_BF16)) == b.ALGO_SEQUENTIAL
    assert b.select_algo(b.make_desc(2, 16, 64, 64, 2, 4, b.GDN_BF16)) == b.ALGO_SEQUENTIAL
    assert b.select_algo(b.make_desc(2, 16, 128, 128, 2, 4, b.GDN_FP32)) == b.ALGO_SEQUENTIAL


def _decode_call(fn, desc, **over):
    base = 0x7f0000000000
    names = ["pool", "slots", "q", "k", "v", "g", "beta", "out", "cache", "accepted", "status"]
    ptr = {n: base + 0x10000000 * i for i, n in enumerate(names)}
    ptr["status"] = None
    ptr.update(over)
    lib = b.load_library()
    p = lambda n: None if ptr[n] is None else ctypes.c_void_p(ptr[n])
    d = ctypes.byref(desc)
    if fn == "replay":
        return lib.gdn_decode_replay(d, p("pool"), p("slots"), p("q"), p("k"), p("v"), p("g"), p("beta"),
                                     p("out"), p("status"), None)
    if fn == "verify":
        return lib.gdn_decode_verify(d, p("pool"), p("slots"), p("q"), p("k"), p("v"), p("g"), p("beta"),
                                     p("out"), p("cache"), p("status"), None)
    return lib.gdn_decode_commit(d, p("pool"), p("slots"), p("cache"), p("accepted"), p("status"), None)


@no_gpu
@pytest.mark.parametrize("fn", ["replay", "verify", "commit"])
@pytest.mark.parametrize("case,expect", [
    ("zero_seqs", b.GDN_ERR_INVALID_ARG), ("zero_tokens", b.GDN_ERR_INVALID_ARG),
    ("zero_pool", b.GDN_ERR_INVALID_ARG), ("reserved", b.GDN_ERR_INVALID_ARG),
    ("bad_dtype", b.GDN_ERR_INVALID_ARG), ("d48", b.GDN_ERR_UNSUPPORTED), ("dk_ne_dv", b.GDN_ERR_UNSUPPORTED),
    ("L65", b.GDN_ERR_UNSUPPORTED), ("null_pool", b.GDN_ERR_INVALID_ARG), ("null_slots", b.GDN_ERR_INVALID_ARG),
    ("misaligned_pool", b.GDN_ERR_ALIGNMENT), ("misaligned_slots", b.GDN_ERR_ALIGNMENT),
    ("valid_no_device", b.GDN_ERR_CUDA),
])
def test_decode_host_validation(fn, case, expect):
    d = b.make_decode_desc(2, 4, 64, 64, 4, 8, b.GDN_BF16)
    over = {}
    if case == "zero_seqs":
        d.num_seqs = 0
    elif case == "zero_tokens":
        d.num_tokens = 0
    elif case == "zero_pool":
        d.pool_slots = 0
    elif case == "reserved":
        d.reserved = 3
    elif case == "bad_dtype":
        d.dtype = 7
    elif case == "d48":
        d.d_k = d.d_v = 48
    elif case == "dk_ne_dv":
        d.d_v = 32
    elif case == "L65":
        d.num_tokens = 65
    elif case == "null_pool":
        over["pool"] = None
    elif case == "null_slots":
        over["slots"] = None
    elif case == "misaligned_pool":
        over["pool"] = 0x7f0000000008
    elif case == "misaligned_slots":
        over["slots"] = 0x7f0000000002
    assert _decode_call(fn, d, **over) == expect


def test_route1_workspace_and_validation():
    d = b.make_desc(2, 4, 64, 64, 2, 16, b.GDN_BF16, algo=b.ALGO_ROUTE1)
    offs, pl = [0, 96, 160], [32, 32]                 # responses 64 and 32 tokens: 6 blocks of 16
    assert b.workspace_size(d, offs) == 0             # needs the prompt lengths
    assert b.workspace_size_route1(d, offs, pl) == 256 + 6 * 4 * 64 * 64 * 4
    assert b.workspace_size_route1(d, offs, [30, 32]) == 0          # response not a multiple of B
    assert b.select_algo(b.make_desc(2, 4, 64, 64, 2, 16, b.GDN_BF16)) != b.ALGO_ROUTE1
    # the tensor-core form with ShortConv (bf16, d = 128, B = 16) adds the conv pass's convolved
    # copies, 3 (T + V T_R) H d bf16 elements; any other ShortConv case adds nothing (unsupported)
    dt = b.make_desc(2, 4, 128, 128, 2, 16, b.GDN_BF16, conv_width=4, algo=b.ALGO_ROUTE1)
    assert b.workspace_size_route1(dt, offs, pl) == 256 + 6 * 4 * 128 * 128 * 4 + 3 * (160 + 2 * 96) * 4 * 128 * 2
    dc = b.make_desc(2, 4, 64, 64, 2, 16, b.GDN_BF16, conv_width=4, algo=b.ALGO_ROUTE1)
    assert b.workspace_size_route1(dc, offs, pl) == 256 + 6 * 4 * 64 * 64 * 4


@no_gpu
def test_route1_host_validation():
    d = b.make_desc(2, 2, 32, 32, 2, 4, b.GDN_FP32, algo=b.ALGO_ROUTE1)
    need = b.workspace_size_route1(d, [0, 16, 40], [8, 4])
    assert _call(d, [0, 16, 40], [8, 4], _ws_bytes=need - 16) == b.GDN_ERR_INVALID_ARG   # states do not fit
    dc = b.make_desc(2, 2, 32, 32, 2, 4, b.GDN_FP32, conv_width=4, algo=b.ALGO_ROUTE1)
    assert _call(dc, [0, 16, 40], [8, 4], conv_w=_Fake(0x7f0000000000), _ws_bytes=need) == b.GDN_ERR_UNSUPPORTED
    assert _call(d, [0, 16, 40], [8, 4], _ws_bytes=need) == b.GDN_ERR_CUDA              # valid; no device here
    # the tensor-core form takes ShortConv; its workspace must hold the convolved copies too
    dt = b.make_desc(2, 2, 128, 128, 2, 16, b.GDN_BF16, conv_width=4, algo=b.ALGO_ROUTE1)
    offs, pl = [0, 48, 96], [16, 16]
    need_t = b.workspace_size_route1(dt, offs, pl)
    assert _call(dt, offs, pl, conv_w=_Fake(0x7f0000000000), _ws_bytes=need_t - 256) == b.GDN_ERR_INVALID_ARG
    assert _call(dt, offs, pl, conv_w=_Fake(0x7f0000000000), _ws_bytes=need_t) == b.GDN_ERR_CUDA


@no_gpu
def test_host_forward_validation():
    """gdn_dual_forward_host rejects bad arguments on the host before anything is enqueued; a
    valid call reaches the CUDA runtime (which fails here: no device)."""
    d = b.make_desc(3, 2, 64, 64, 2, 4, b.GDN_BF16)
    offs, pl = [0, 40, 40, 104], [8, 0, 32]
    need = b.host_staging_size(d, offs, pl, 2)
    assert need > 0 and need % 256 == 0
    assert b.host_staging_size(d, offs, pl, 0) == 0                     # groups < 1
    assert b.host_staging_size(d, [0, 40, 40, 103], pl, 2) == 0         # response not a multiple of B
    assert b.host_staging_size(d, offs, pl, 64) >= b.host_staging_size(d, offs, pl, 1) // 4
    lib = b.load_library()
    ip = ctypes.POINTER(ctypes.c_int32)

    def call(desc, offs, pl, groups, staging, nbytes, **over):
        base = 0x7f0000000000
        names = ["q", "k", "v", "g", "beta", "qn", "kn", "vn", "gn", "betan", "conv_w", "out", "out_noisy",
                 "final_state"]
        ptr = {n: ctypes.c_void_p(base + 0x10000000 * i) for i, n in enumerate(names)}
        ptr["conv_w"] = None
        ptr.update(over)
        o = np.ascontiguousarray(offs, dtype=np.int32)
        p = np.ascontiguousarray(pl, dtype=np.int32)
        return lib.gdn_dual_forward_host(ctypes.byref(desc), *[ptr[n] for n in names[:10]], o.ctypes.data_as(ip),
                                         p.ctypes.data_as(ip), ptr["conv_w"], ptr["out"], ptr["out_noisy"],
                                         ptr["final_state"], ctypes.c_void_p(staging), ctypes.c_size_t(nbytes),
                                         groups, None)

    stg = 0x7e0000000000
    assert call(d, offs, pl, 0, stg, need) == b.GDN_ERR_INVALID_ARG               # groups < 1
    assert call(d, offs, pl, 2, stg, need - 256) == b.GDN_ERR_INVALID_ARG         # staging too small
    assert call(d, offs, pl, 2, stg + 16, need) == b.GDN_ERR_INVALID_ARG          # staging not 256-aligned
    assert call(d, offs, pl, 2, 0, need) == b.GDN_ERR_INVALID_ARG                 # no staging
    assert call(d, offs, pl, 2, stg, need, q=None) == b.GDN_ERR_INVALID_ARG       # missing input
    bad = b.make_desc(3, 2, 48, 48, 2, 4, b.GDN_BF16)                              # d = 48: unsupported
    assert call(bad, offs, pl, 2, stg, b.host_staging_size(bad, offs, pl, 2)) == b.GDN_ERR_UNSUPPORTED
    assert call(d, offs, pl, 2, stg, need) == b.GDN_ERR_CUDA                      # valid; no device here


def _attn_call(desc, offs, pl, ws_bytes=None, **over):
    base = 0x7f0000000000
    names = ["q", "k", "v", "qn", "kn", "vn", "out", "out_noisy", "ws"]
    ptr = {n: base + 0x10000000 * i for i, n in enumerate(names)}
    ptr.update(over)
    lib = b.load_library()
    p = lambda n: None if ptr[n] is None else ctypes.c_void_p(ptr[n])
    o = np.ascontiguousarray(offs, dtype=np.int32)
    l = np.ascontiguousarray(pl, dtype=np.int32)
    ip = ctypes.POINTER(ctypes.c_int32)
    if ws_bytes is None:
        ws_bytes = b.attn_workspace_size(desc, o, l)
    return lib.gdn_attn_forward(ctypes.byref(desc) if desc is not None else None, p("q"), p("k"), p("v"), p("qn"),
                                p("kn"), p("vn"), o.ctypes.data_as(ip), l.ctypes.data_as(ip), p("out"),
                                p("out_noisy"), p("ws"), ctypes.c_size_t(ws_bytes), None)


def test_attention_workspace_size():
    d = b.make_attn_desc(2, 4, 2, 128, 2, 4, b.GDN_BF16)
    assert b.attn_workspace_size(d, [0, 300, 400], [100, 4]) == 256     # the device status word
    assert b.attn_workspace_size(d, [0, 300, 400], [101, 4]) == 0       # response 199 % 4
    assert b.attn_workspace_size(d, [0, 300, 200], [100, 4]) == 0       # offsets decrease
    assert b.attn_workspace_size(d, [1, 300, 400], [100, 4]) == 0       # must start at 0
    bad = b.make_attn_desc(2, 4, 2, 128, 2, 4, b.GDN_BF16)
    bad.reserved = 1
    assert b.attn_workspace_size(bad, [0, 300, 400], [100, 4]) == 0


@no_gpu
@pytest.mark.parametrize("case,expect", [
    ("null_desc", b.GDN_ERR_INVALID_ARG), ("reserved", b.GDN_ERR_INVALID_ARG), ("zero_heads", b.GDN_ERR_INVALID_ARG),
    ("bad_layout", b.GDN_ERR_INVALID_ARG), ("null_q", b.GDN_ERR_INVALID_ARG), ("null_noisy", b.GDN_ERR_INVALID_ARG),
    ("small_workspace", b.GDN_ERR_INVALID_ARG), ("misaligned_k", b.GDN_ERR_ALIGNMENT),
    ("d64", b.GDN_ERR_UNSUPPORTED), ("fp32", b.GDN_ERR_UNSUPPORTED), ("kv_heads_3", b.GDN_ERR_UNSUPPORTED),
    ("views_3", b.GDN_ERR_UNSUPPORTED), ("block_3", b.GDN_ERR_UNSUPPORTED),
    ("valid_no_device", b.GDN_ERR_CUDA),
])
def test_attention_host_validation(case, expect):
    d = b.make_attn_desc(2, 4, 2, 128, 2, 4, b.GDN_BF16)
    offs, pl, over, ws = [0, 300, 400], [100, 4], {}, None
    if case == "null_desc":
        d = None
        ws = 4096
    elif case == "reserved":
        d.reserved = 2
        ws = 4096
    elif case == "zero_heads":
        d.num_heads = 0
        ws = 4096
    elif case == "bad_layout":
        pl = [101, 4]
        ws = 4096
    elif case == "null_q":
        over["q"] = None
    elif case == "null_noisy":
        over["vn"] = None
    elif case == "small_workspace":
        ws = 128
    elif case == "misaligned_k":
        over["k"] = 0x7f0000000004
    elif case == "d64":
        d.head_dim = 64
    elif case == "fp32":
        d.dtype = b.GDN_FP32
    elif case == "kv_heads_3":
        d.num_kv_heads = 3
    elif case == "views_3":
        d.num_views = 3
    elif case == "block_3":
        d.block_size = 3
        pl = [102, 4]     # responses 198 and 96: multiples of 3
    assert _attn_call(d, offs, pl, ws_bytes=ws, **over) == expect


@no_gpu
def test_backward_host_validation():
    base = 0x7f0000000000
    lib = b.load_library()
    offs = np.array([0, 40, 73], np.int32)
    pl = np.array([8, 1], np.int32)
    ip = ctypes.POINTER(ctypes.c_int32)

    def call(desc, ws_bytes=None, over=None):
        ptr = [ctypes.c_void_p(base + 0x10000000 * i) for i in range(24)]   # 10 inputs, 3 upstream, 10 grads, ws
        for i, v in (over or {}).items():
            ptr[i] = None if v is None else ctypes.c_void_p(v)
        nb = b.backward_workspace_size(desc, offs) if ws_bytes is None else ws_bytes
        return lib.gdn_dual_backward(ctypes.byref(desc), *ptr[:10], offs.ctypes.data_as(ip), pl.ctypes.data_as(ip),
                                     *ptr[10:23], ptr[23], ctypes.c_size_t(nb), None)

    d = b.make_desc(2, 2, 64, 64, 2, 4, b.GDN_FP32)
    # 73 tokens in 16-token checkpoints: 3 + 3 per head, 64 x 64 fp32 each, plus 256 bytes; then the
    # column-summed gradients' partials, per 32-column slice (2 here): [dq | dk] (T H d each) and
    # [dg | dbeta] (T H each), and the same for the noisy stream over V x T rows
    th = 73 * 2
    partial = 2 * (2 * th * 64 + 2 * th) * (1 + 2)
    assert b.backward_workspace_size(d, offs) == 256 + 6 * 2 * 64 * 64 * 4 + partial * 4
    assert call(d, ws_bytes=1024) == b.GDN_ERR_INVALID_ARG
    assert call(d, over={0: None}) == b.GDN_ERR_INVALID_ARG                  # q
    assert call(d, over={3: base + 4}) == b.GDN_ERR_ALIGNMENT                # g
    dc = b.make_desc(2, 2, 64, 64, 2, 4, b.GDN_FP32, conv_width=4)
    assert call(dc) == b.GDN_ERR_UNSUPPORTED
    d48 = b.make_desc(2, 2, 48, 48, 2, 4, b.GDN_FP32)
    assert call(d48) == b.GDN_ERR_UNSUPPORTED
    assert call(d) == b.GDN_ERR_CUDA                                         # valid; no device here


@no_gpu
def test_backward_more_documents_than_supported():
    lib = b.load_library()
    N = 1025
    offs = np.arange(N + 1, dtype=np.int32) * 4
    pl = np.zeros(N, np.int32)
    d = b.make_desc(N, 1, 32, 32, 1, 4, b.GDN_FP32)
    ip = ctypes.POINTER(ctypes.c_int32)
    ptr = [ctypes.c_void_p(0x7f0000000000 + 0x10000000 * i) for i in range(24)]
    nb = b.backward_workspace_size(d, offs)
    assert nb > 0
    st = lib.gdn_dual_backward(ctypes.byref(d), *ptr[:10], offs.ctypes.data_as(ip), pl.ctypes.data_as(ip),
                               *ptr[10:23], ptr[23], ctypes.c_size_t(nb), None)
    assert st == b.GDN_ERR_UNSUPPORTED


def test_noalloc_rejects_route1_and_invalid_descriptors():
    """The no-allocation entry point refuses on the host, before any device work: Route I (its
    block-boundary states need far more than the fixed scratch array) is GDN_ERR_UNSUPPORTED, a
    NULL or invalid descriptor GDN_ERR_INVALID_ARG."""
    lib = b.load_library()
    offs = np.array([0, 64], np.int32)
    pl = np.array([32], np.int32)
    ip = ctypes.POINTER(ctypes.c_int32)
    fn = lib.gdn_dual_forward_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(b.Desc)] + [ctypes.c_void_p] * 10 + [ip, ip] + [ctypes.c_void_p] * 5

    def call(desc):
        ref = None if desc is None else ctypes.byref(desc)
        return fn(ref, *([None] * 10), offs.ctypes.data_as(ip), pl.ctypes.data_as(ip), *([None] * 5))

    assert call(b.make_desc(1, 2, 128, 128, 2, 4, b.GDN_BF16, algo=b.ALGO_ROUTE1)) == b.GDN_ERR_UNSUPPORTED
    assert call(None) == b.GDN_ERR_INVALID_ARG
    assert call(b.make_desc(1, 2, 128, 128, 9, 4, b.GDN_BF16)) == b.GDN_ERR_INVALID_ARG    # views > 8
    assert call(b.make_desc(0, 2, 128, 128, 2, 4, b.GDN_BF16)) == b.GDN_ERR_INVALID_ARG    # no documents


@no_gpu
def test_backward_conv_host_validation():
    """gdn_dual_backward_conv refuses on the host: conv width other than 4, NULL weights or weight
    gradient, a workspace smaller than gdn_dual_backward_conv_workspace_size."""
    base = 0x7f0000000000
    lib = b.load_library()
    offs = np.array([0, 40, 73], np.int32)
    pl = np.array([8, 1], np.int32)
    ip = ctypes.POINTER(ctypes.c_int32)
    fn = lib.gdn_dual_backward_conv
    fn.restype = ctypes.c_int
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(b.Desc)] + [vp] * 10 + [ip, ip] + [vp] * 4 + [vp] * 10 + [vp, vp, ctypes.c_size_t, vp]

    def call(desc, ws_bytes=None, over=None):
        ptr = [ctypes.c_void_p(base + 0x10000000 * i) for i in range(26)]   # 10 in, conv_w, 3 up, 10 grads, dw, ws
        for i, v in (over or {}).items():
            ptr[i] = None if v is None else ctypes.c_void_p(v)
        nb = b.backward_conv_workspace_size(desc, offs) if ws_bytes is None else ws_bytes
        return fn(ctypes.byref(desc), *ptr[:10], offs.ctypes.data_as(ip), pl.ctypes.data_as(ip), *ptr[10:25],
                  ptr[25], ctypes.c_size_t(nb), None)

    d = b.make_desc(2, 2, 64, 64, 2, 4, b.GDN_FP32, conv_width=4)
    need = b.backward_conv_workspace_size(d, offs)
    assert need > b.backward_workspace_size(b.make_desc(2, 2, 64, 64, 2, 4, b.GDN_FP32), offs)
    assert call(d, ws_bytes=need - 16) == b.GDN_ERR_INVALID_ARG
    assert call(d, over={10: None}) == b.GDN_ERR_INVALID_ARG                 # conv_w
    assert call(d, over={24: None}) == b.GDN_ERR_INVALID_ARG                 # dconv_w
    assert call(b.make_desc(2, 2, 64, 64, 2, 4, b.GDN_FP32, conv_width=3)) == b.GDN_ERR_UNSUPPORTED
    assert call(b.make_desc(2, 2, 64, 64, 2, 4, b.GDN_FP32)) == b.GDN_ERR_UNSUPPORTED   # no conv: gdn_dual_backward


def test_workspace_size_covers_the_conv_pass():
    """With ShortConv, AUTO on the chunked path asks for room for the convolved bf16 inputs
    (3 T H d clean + 3 V T H d noisy elements, T_R bounded by T); an explicit algorithm needs the
    256-byte header only."""
    offs = [0, 64, 192]
    T, H, d, V = 192, 2, 128, 2
    auto = b.make_desc(2, H, d, d, V, 4, b.GDN_BF16, conv_width=4)
    conv_bytes = 3 * (T * H * d + V * T * H * d) * 2
    assert b.workspace_size(auto, offs) == 256 + (conv_bytes + 255) // 256 * 256
    assert b.workspace_size(b.make_desc(2, H, d, d, V, 4, b.GDN_BF16, conv_width=4, algo=b.ALGO_CHUNKED), offs) == 256
    assert b.workspace_size(b.make_desc(2, H, d, d, V, 4, b.GDN_BF16), offs) == 256
