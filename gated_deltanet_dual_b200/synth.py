"""Seeded synthetic inputs for the dual-stream Gated DeltaNet forward.

This module only draws random tensors and lays them out; it holds none of the
method's arithmetic.  The same generator feeds the CPU oracle (tests), the CUDA
path (tests, bench) and the CPU baseline leg of the bench.

Workloads are named by what they are.  The shapes follow the dual-stream
training setting of "FLARE: Diffusion for Hybrid Language Model"
(papernotes.org notes, Method > Overall framework: prompt kept causal, response
cut into blocks of B, two complementary noisy views per block) and its
document-packing rule (Key design 3: document boundaries aligned to B).

Layout (row-major, contiguous):
  q, k          [T, H, d_k]      I/O dtype (fp32 or bf16)
  v             [T, H, d_v]      I/O dtype
  g, beta       [T, H]           fp32   (g = log alpha)
  qn, kn        [V, T_R, H, d_k] I/O dtype, packed over response tokens only
  vn            [V, T_R, H, d_v]
  gn, betan     [V, T_R, H]      fp32
  conv_w        [3, H*d, W]      fp32 (q, k, v channel weights; tap W-1 = current token)
  doc_offsets   [N+1] int32 (host), prompt_len [N] int32 (host)

Draw order (one torch.Generator on the target device, seeded once):
  q, k, v, g, beta, then for each view: qn, kn, vn, gn, betan, then conv_w.
The document split of the packed workload is drawn first, on the host, from
numpy's PCG64 seeded with the same seed, so it does not depend on the device.
q, k ~ N(0,1) normalised to unit L2 norm per (token, head) in fp32 before the
cast; v ~ N(0,1); g ~ U(g_lo, 0); beta = sigmoid(N(0, beta_std)).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_heads: int
    d: int
    block_size: int
    num_views: int = 2
    dtype: str = "bf16"            # "bf16" or "fp32"
    # plain batch: num_docs equal documents of doc_len tokens, prompt_len each
    num_docs: int = 0
    doc_len: int = 0
    prompt: int = 0
    # packed row: one row of packed_total tokens split into documents
    packed_total: int = 0
    packed_min: int = 256
    packed_max: int = 4096
    g_lo: float = -0.1
    beta_std: float = 1.0
    conv_width: int = 0
    conv_std: float = 0.5

    def with_block(self, b: int) -> "Workload":
        return dataclasses.replace(self, block_size=b, name=f"{self.name.split('_B')[0]}_B{b}")


def _wl(**kw) -> Workload:
    return Workload(**kw)


# The five workloads of the benchmark plan (names give their sizes).
WORKLOADS = {
    "tiny_fp32_1x64_h2_d32": _wl(name="tiny_fp32_1x64_h2_d32", num_heads=2, d=32, block_size=4,
                                 dtype="fp32", num_docs=1, doc_len=64, prompt=32),
    "train_8x4096_h16_d128": _wl(name="train_8x4096_h16_d128", num_heads=16, d=128, block_size=4,
                                 num_docs=8, doc_len=4096, prompt=1024),
    "packed_32768_h16_d128": _wl(name="packed_32768_h16_d128", num_heads=16, d=128, block_size=4,
                                 packed_total=32768),
    "conv_4x8192_h16_d128_B4": _wl(name="conv_4x8192_h16_d128_B4", num_heads=16, d=128, block_size=4,
                                   num_docs=4, doc_len=8192, prompt=2048, conv_width=4),
    "large_32x8192_h32_d128": _wl(name="large_32x8192_h32_d128", num_heads=32, d=128, block_size=4,
                                  num_docs=32, doc_len=8192, prompt=2048, g_lo=-0.5, beta_std=2.0),
}
BLOCK_SWEEP = (2, 4, 8, 16, 32)


def get_workload(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    if name.startswith("conv_4x8192_h16_d128_B"):
        return WORKLOADS["conv_4x8192_h16_d128_B4"].with_block(int(name.rsplit("B", 1)[1]))
    if name.startswith("train_8x4096_h16_d128_B"):       # the training shape at other block sizes
        return WORKLOADS["train_8x4096_h16_d128"].with_block(int(name.rsplit("B", 1)[1]))
    raise KeyError(name)


@dataclasses.dataclass
class Problem:
    """One batch of inputs plus its host-side metadata."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    qn: torch.Tensor
    kn: torch.Tensor
    vn: torch.Tensor
    gn: torch.Tensor
    betan: torch.Tensor
    conv_w: Optional[torch.Tensor]
    doc_offsets: np.ndarray   # int32 [N+1]
    prompt_len: np.ndarray    # int32 [N]
    block_size: int
    num_views: int
    conv_width: int

    @property
    def num_docs(self) -> int:
        return int(self.doc_offsets.shape[0] - 1)

    @property
    def T(self) -> int:
        return int(self.q.shape[0])

    @property
    def T_R(self) -> int:
        return int(self.qn.shape[1])

    @property
    def num_heads(self) -> int:
        return int(self.q.shape[1])

    @property
    def d_k(self) -> int:
        return int(self.q.shape[2])

    @property
    def d_v(self) -> int:
        return int(self.v.shape[2])

    def tokens(self) -> int:
        """Clean plus noisy tokens (the throughput unit)."""
        return self.T + self.num_views * self.T_R

    def response_offsets(self) -> np.ndarray:
        """Start row of each document's response inside the packed noisy tensors."""
        lens = np.diff(self.doc_offsets.astype(np.int64)) - self.prompt_len.astype(np.int64)
        out = np.zeros(self.num_docs + 1, dtype=np.int64)
        out[1:] = np.cumsum(lens)
        return out


def packed_split(total: int, lo: int, hi: int, block: int, seed: int):
    """Document lengths for one packed row: lengths 4*floor(U[lo,hi]/4) drawn until the
    sum reaches `total`, the last one clipped; prompt = 4*floor(len/16) (a quarter)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = []
    acc = 0
    while acc < total:
        ln = int(4 * (int(rng.uniform(lo, hi)) // 4))
        ln = max(ln, 4)
        ln = min(ln, total - acc)
        lens.append(ln)
        acc += ln
    lens = np.array(lens, dtype=np.int64)
    prompts = 4 * (lens // 16)
    # response must be a multiple of the block size (boundaries aligned to B)
    resp = lens - prompts
    prompts = prompts + (resp % block)
    return lens, prompts


def doc_layout(wl: Workload, seed: int = 0):
    if wl.packed_total:
        lens, prompts = packed_split(wl.packed_total, wl.packed_min, wl.packed_max, wl.block_size, seed)
    else:
        lens = np.full(wl.num_docs, wl.doc_len, dtype=np.int64)
        prompts = np.full(wl.num_docs, wl.prompt, dtype=np.int64)
    offs = np.zeros(len(lens) + 1, dtype=np.int64)
    offs[1:] = np.cumsum(lens)
    return offs.astype(np.int32), prompts.astype(np.int32)


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_problem_from_layout(doc_offsets, prompt_len, *, num_heads: int, d_k: int, d_v: int,
                             block_size: int, num_views: int = 2, dtype: str = "bf16",
                             g_lo: float = -0.1, beta_std: float = 1.0, conv_width: int = 0,
                             conv_std: float = 0.5, seed: int = 0, device="cpu") -> Problem:
    doc_offsets = np.asarray(doc_offsets, dtype=np.int32)
    prompt_len = np.asarray(prompt_len, dtype=np.int32)
    T = int(doc_offsets[-1])
    T_R = int((np.diff(doc_offsets.astype(np.int64)) - prompt_len).sum())
    H, V = num_heads, num_views
    tdt = {"bf16": torch.bfloat16, "fp32": torch.float32}[dtype]
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    def normal(*shape):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)

    def uniform(*shape):
        return torch.rand(*shape, generator=gen, device=device, dtype=torch.float32)

    def stream(rows):
        q = _unit_rows(normal(rows, H, d_k)).to(tdt)
        k = _unit_rows(normal(rows, H, d_k)).to(tdt)
        v = normal(rows, H, d_v).to(tdt)
        g = (uniform(rows, H) * g_lo).contiguous()
        b = torch.sigmoid(normal(rows, H) * beta_std).contiguous()
        return q, k, v, g, b

    q, k, v, g, beta = stream(T)
    views = [stream(T_R) for _ in range(V)]
    if V > 0:
        qn, kn, vn, gn, betan = (torch.stack([vw[i] for vw in views]).contiguous() for i in range(5))
    else:
        qn = torch.empty(0, T_R, H, d_k, dtype=tdt, device=device)
        kn = torch.empty(0, T_R, H, d_k, dtype=tdt, device=device)
        vn = torch.empty(0, T_R, H, d_v, dtype=tdt, device=device)
        gn = torch.empty(0, T_R, H, device=device)
        betan = torch.empty(0, T_R, H, device=device)
    conv_w = None
    if conv_width:
        if d_k != d_v:
            raise ValueError("ShortConv weights assume d_k == d_v")
        conv_w = (normal(3, H * d_k, conv_width) * conv_std).contiguous()
    return Problem(q=q, k=k, v=v, g=g, beta=beta, qn=qn, kn=kn, vn=vn, gn=gn, betan=betan,
                   conv_w=conv_w, doc_offsets=doc_offsets, prompt_len=prompt_len,
                   block_size=block_size, num_views=V, conv_width=conv_width)


def make_problem(wl: Workload | str, seed: int = 0, device="cpu") -> Problem:
    if isinstance(wl, str):
        wl = get_workload(wl)
    offs, prompts = doc_layout(wl, seed)
    return make_problem_from_layout(offs, prompts, num_heads=wl.num_heads, d_k=wl.d, d_v=wl.d,
                                    block_size=wl.block_size, num_views=wl.num_views,
                                    dtype=wl.dtype, g_lo=wl.g_lo, beta_std=wl.beta_std,
                                    conv_width=wl.conv_width, conv_std=wl.conv_std,
                                    seed=seed, device=device)


# ----------------------------------------------------------------------------- decode side
@dataclasses.dataclass
class DecodeProblem:
    """One decode call's inputs: a state pool, the pool row of each sequence, and L tokens per
    sequence (layouts of include/gdn_decode.h)."""
    state_pool: torch.Tensor   # [P, H, d, d] fp32
    slots: torch.Tensor        # [N] int32
    q: torch.Tensor            # [N, L, H, d]
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor            # [N, L, H] fp32
    beta: torch.Tensor


DECODE_WORKLOADS = {
    # the pages' serving shape: 8 concurrent sequences; one block of B = 4 tokens per replay and
    # K = 4 drafted candidates per verify
    "decode_8seq_h32_d128_L4": dict(num_seqs=8, num_heads=32, d=128, num_tokens=4, pool_slots=64),
    "decode_64seq_h32_d128_L4": dict(num_seqs=64, num_heads=32, d=128, num_tokens=4, pool_slots=128),
}


def make_decode_problem(num_seqs: int, num_heads: int, d: int, num_tokens: int, pool_slots: int,
                        dtype: str = "bf16", g_lo: float = -0.1, beta_std: float = 1.0,
                        state_std: float = 0.3, seed: int = 0, device="cpu") -> DecodeProblem:
    """Seeded decode inputs: pool rows ~ N(0, state_std^2), slots a seeded permutation prefix of
    the pool rows, tokens drawn like the forward workloads (unit q, k; v ~ N(0,1);
    g ~ U(g_lo, 0); beta = sigmoid(N(0, beta_std^2)))."""
    tdt = {"bf16": torch.bfloat16, "fp32": torch.float32}[dtype]
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    N, H, L = num_seqs, num_heads, num_tokens
    normal = lambda *s: torch.randn(*s, generator=gen, device=device, dtype=torch.float32)
    pool = (normal(pool_slots, H, d, d) * state_std).contiguous()
    slots = torch.randperm(pool_slots, generator=gen, device=device)[:N].to(torch.int32).contiguous()
    q = _unit_rows(normal(N, L, H, d)).to(tdt)
    k = _unit_rows(normal(N, L, H, d)).to(tdt)
    v = normal(N, L, H, d).to(tdt)
    g = (torch.rand(N, L, H, generator=gen, device=device) * g_lo).contiguous()
    beta = torch.sigmoid(normal(N, L, H) * beta_std).contiguous()
    return DecodeProblem(state_pool=pool, slots=slots, q=q, k=k, v=v, g=g, beta=beta)


# ----------------------------------------------------------------------------- softmax attention
@dataclasses.dataclass
class AttnProblem:
    """Inputs of one dual-stream attention call (layouts of include/gdn_attention.h)."""
    q: torch.Tensor            # [T, H, d]
    k: torch.Tensor            # [T, H_kv, d]
    v: torch.Tensor
    qn: torch.Tensor           # [V, T_R, H, d]
    kn: torch.Tensor           # [V, T_R, H_kv, d]
    vn: torch.Tensor
    doc_offsets: np.ndarray    # int32 [N+1]
    prompt_len: np.ndarray     # int32 [N]
    block_size: int


# The attention layers of the same hybrid model on the same token layouts as the GDN workloads
# (same document split and blocks); H query heads, H_kv key/value heads.
ATTN_WORKLOADS = {
    "attn_train_8x4096_h16_d128": dict(layout="train_8x4096_h16_d128", num_heads=16, num_kv_heads=16),
    "attn_packed_32768_h16_d128": dict(layout="packed_32768_h16_d128", num_heads=16, num_kv_heads=16),
    "attn_train_8x4096_h32kv8_d128": dict(layout="train_8x4096_h16_d128", num_heads=32, num_kv_heads=8),
}


def make_attn_problem_from_layout(doc_offsets, prompt_len, *, num_heads: int, num_kv_heads: int, d: int,
                                  block_size: int, num_views: int = 2, seed: int = 0,
                                  device="cpu") -> AttnProblem:
    """q, k, v ~ N(0, 1) in fp32, cast to bf16 (scores q.k / sqrt(d) ~ N(0, 1)).  Draw order:
    q, k, v, then per view qn, kn, vn."""
    doc_offsets = np.asarray(doc_offsets, dtype=np.int32)
    prompt_len = np.asarray(prompt_len, dtype=np.int32)
    T = int(doc_offsets[-1])
    T_R = int((np.diff(doc_offsets.astype(np.int64)) - prompt_len).sum())
    H, Hkv, V = num_heads, num_kv_heads, num_views
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    normal = lambda *s: torch.randn(*s, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    q, k, v = normal(T, H, d), normal(T, Hkv, d), normal(T, Hkv, d)
    views = [(normal(T_R, H, d), normal(T_R, Hkv, d), normal(T_R, Hkv, d)) for _ in range(V)]
    if V > 0:
        qn, kn, vn = (torch.stack([vw[i] for vw in views]).contiguous() for i in range(3))
    else:
        qn = torch.empty(0, T_R, H, d, dtype=torch.bfloat16, device=device)
        kn = torch.empty(0, T_R, Hkv, d, dtype=torch.bfloat16, device=device)
        vn = torch.empty(0, T_R, Hkv, d, dtype=torch.bfloat16, device=device)
    return AttnProblem(q=q, k=k, v=v, qn=qn, kn=kn, vn=vn, doc_offsets=doc_offsets, prompt_len=prompt_len,
                       block_size=block_size)


def make_attn_problem(name: str, seed: int = 0, device="cpu") -> AttnProblem:
    cfg = ATTN_WORKLOADS[name]
    wl = get_workload(cfg["layout"])
    offs, prompts = doc_layout(wl, seed)
    return make_attn_problem_from_layout(offs, prompts, num_heads=cfg["num_heads"], num_kv_heads=cfg["num_kv_heads"],
                                         d=wl.d, block_size=wl.block_size, num_views=wl.num_views, seed=seed,
                                         device=device)
