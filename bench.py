#!/usr/bin/env python
"""Benchmark: dual-stream Gated DeltaNet forward on B200, tokens/s (clean + noisy tokens).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Each rank runs its own replica of the workload
(documents are independent units, so ranks share nothing on the data path: weak scaling).
Rank 0 prints ONE JSON line.  A step is one gdn_dual_forward call (both streams, all
documents and heads) on inputs already resident in HBM; `e2e` repeats the measurement
through the public Python API with pinned-host inputs copied in and outputs copied back
inside the timed region.  `--impl reference` times the fp64 CPU oracle on the host cores
(a bounded sample of the same workload per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_dual_b200 import binding as gb  # noqa: E402
from gated_deltanet_dual_b200 import replicas  # noqa: E402
from gated_deltanet_dual_b200 import synth  # noqa: E402

DEFAULT_WORKLOAD = "large_32x8192_h32_d128"   # the largest single-GPU workload
METRIC = "dual-stream GDN fwd tokens/s on 1 B200 and % of roofline (HBM/tensor)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = {
    gb.ALGO_SEQUENTIAL: ["gated_deltanet_dual_b200/csrc/gdn_sequential.cu"],
    gb.ALGO_CHUNKED: ["gated_deltanet_dual_b200/csrc/gdn_chunked.cu", "gated_deltanet_dual_b200/csrc/gdn_chunk_common.cuh",
                      "gated_deltanet_dual_b200/csrc/gdn_conv.cu"],
    gb.ALGO_PIPELINED: ["gated_deltanet_dual_b200/csrc/gdn_pipe.cu", "gated_deltanet_dual_b200/csrc/gdn_chunk_common.cuh"],
    gb.ALGO_ROUTE1: ["gated_deltanet_dual_b200/csrc/gdn_decode.cu"],
    "route1_tc": ["gated_deltanet_dual_b200/csrc/gdn_route1_tc.cu", "gated_deltanet_dual_b200/csrc/gdn_chunked.cu",
                  "gated_deltanet_dual_b200/csrc/gdn_chunk_common.cuh", "gated_deltanet_dual_b200/csrc/gdn_conv.cu"],
    "attention": ["gated_deltanet_dual_b200/csrc/gdn_attention.cu"],
}
KERNEL_NAMES = {gb.ALGO_SEQUENTIAL: "gdn_sequential_kernel", gb.ALGO_CHUNKED: "gdn_chunked_kernel",
                gb.ALGO_PIPELINED: "gdn_pipe_kernel",
                gb.ALGO_ROUTE1: "gdn_route1_chain_kernel + gdn_decode_kernel (block end)",
                "route1_tc": "gdn_chunked_kernel (state export) + gdn_route1_refine_kernel",
                "attention": "gdn_attention_kernel"}


# ----------------------------------------------------------------------------- work model
def algorithmic_work(prob) -> dict:
    """Algorithmic bytes and FLOPs of one forward (what must move / be computed at minimum):
    per (stream-token, head) read q, k, v and g, beta, write o; plus the fp32 final state per
    (doc, head) and the conv weights.  FLOPs: k^T S, the rank-1 update and S^T q = 6 d_k d_v
    per (stream-token, head), plus 2 W FLOPs per conv'd channel."""
    s = prob.q.element_size()
    H, dk, dv = prob.num_heads, prob.d_k, prob.d_v
    toks = prob.tokens()
    per_tok_head = (2 * dk + dv) * s + 8 + dv * s
    nbytes = toks * H * per_tok_head + prob.num_docs * H * dk * dv * 4
    flops = toks * H * 6 * dk * dv
    if prob.conv_width:
        nbytes += 3 * H * dk * prob.conv_width * 4
        flops += toks * H * (2 * dk + dv) * 2 * prob.conv_width
    return {"bytes": int(nbytes), "flops": int(flops), "bytes_per_token_head": per_tok_head}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_hash(algo) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES.get(algo, []) + ["gated_deltanet_dual_b200/csrc/gdn_internal.cuh",
                                               "gated_deltanet_dual_b200/csrc/sm100.cuh"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(algo, workload, alg_bytes=None):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current
    kernel source (same hash) for this workload; else None.  A record may instead name a
    smaller captured workload of the same kernel (`scaled_from`, for a workload too large to
    capture): its traffic is then scaled by the ratio of the two workloads' algorithmic bytes."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        recs = json.load(open(path))
    except Exception:
        return None
    rec = recs.get(f"{KERNEL_NAMES[algo]}:{workload}")
    if rec and rec.get("scaled_from") and alg_bytes:
        src = recs.get(f"{KERNEL_NAMES[algo]}:{rec['scaled_from']}")
        if not src or src.get("kernel_hash") != kernel_hash(algo) or not src.get("algorithmic_bytes"):
            return None
        return int(src["dram_bytes_per_launch"] * alg_bytes / src["algorithmic_bytes"])
    if not rec or rec.get("kernel_hash") != kernel_hash(algo):
        return None
    return rec.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle-reason samples taken DURING the timed region.

    NVML is polled from a thread about every millisecond between mark_start() and mark_stop(),
    so even a timed region of a few milliseconds gets samples; without NVML, nvidia-smi is run
    in the background (100 ms period) and its lines are kept."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.samples = []          # (sm_mhz, max_mhz, {reason names})
        self.source = None
        self._on = threading.Event()
        self._quit = threading.Event()
        self._thread = None
        self._proc = None
        self._lines = []

    # -- NVML
    def _nvml_handle(self, nv):
        try:
            props = torch.cuda.get_device_properties(self.device)
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.device)

    def _nvml_loop(self, nv, h):
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._quit.is_set():
            if self._on.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h) if hasattr(
                        nv, "nvmlDeviceGetCurrentClocksEventReasons") else nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                    self.samples.append((float(sm), float(mx), {n for n, m in self.REASONS.items() if bits & m}))
                except Exception:
                    pass
            time.sleep(0.001)

    # -- nvidia-smi fallback
    def _smi_read(self):
        for line in self._proc.stdout:
            if self._on.is_set():
                self._lines.append(line.strip())

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._nvml_handle(nv)
            self._nv, self._h = nv, h
            self._mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self._thread.start()
            self.source = "nvml"
        except Exception:
            try:
                self._proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                               "-lms", "100", "-i", str(self.device)],
                                              stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self._thread = threading.Thread(target=self._smi_read, daemon=True)
                self._thread.start()
                self.source = "nvidia-smi"
            except (FileNotFoundError, OSError):
                self.source = None
        return self

    def mark_start(self):
        self._on.set()

    def poll_until(self, event):
        """Sample from the calling thread until `event` (a CUDA event recorded after the timed
        work) has completed, so a short timed region still gets samples under load."""
        nv, h = getattr(self, "_nv", None), getattr(self, "_h", None)
        while not event.query():
            if nv is not None:
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h) if hasattr(
                        nv, "nvmlDeviceGetCurrentClocksEventReasons") else nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                    self.samples.append((float(sm), float(self._mx), {n for n, m in self.REASONS.items() if bits & m}))
                except Exception:
                    pass
            time.sleep(0.0005)

    def mark_stop(self):
        self._on.clear()

    def __exit__(self, *exc):
        self._quit.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        samples = list(self.samples)
        for ln in self._lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rs = {n for n, v in zip(["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"],
                                        parts[5:9]) if v.lower().startswith("active")}
                samples.append((float(parts[1]), float(parts[2]), rs))
            except ValueError:
                continue
        if not samples:
            return None
        reasons = set().union(*[r for _, _, r in samples])
        return {"sm_mhz": statistics.median(s for s, _, _ in samples), "sm_max_mhz": max(m for _, m, _ in samples),
                "reasons": sorted(reasons), "samples": len(samples), "source": self.source}


# ----------------------------------------------------------------------------- reference arm
def oracle_sample_problem(wl, max_units: int, seed: int = 0):
    """A bounded sample of the workload for the CPU oracle: its first documents (all heads),
    generated on the host with the same distributions."""
    offs, prompts = synth.doc_layout(wl, seed)
    H = wl.num_heads
    ndocs = max(1, min(len(prompts), max_units // H))
    sub_offs = offs[:ndocs + 1] - offs[0]
    prob = synth.make_problem_from_layout(sub_offs, prompts[:ndocs], num_heads=H, d_k=wl.d, d_v=wl.d,
                                          block_size=wl.block_size, num_views=wl.num_views, dtype=wl.dtype,
                                          g_lo=wl.g_lo, beta_std=wl.beta_std, conv_width=wl.conv_width,
                                          conv_std=wl.conv_std, seed=seed, device="cpu")
    return prob, ndocs


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def time_oracle(wl, steps: int, warmup: int, max_units: int):
    import oracle  # test infrastructure: the CPU baseline / reference arm only
    prob, ndocs = oracle_sample_problem(wl, max_units)
    threads = min(host_cores(), prob.num_docs * prob.num_heads)
    for _ in range(warmup):
        oracle.forward_problem(prob, num_threads=threads)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle.forward_problem(prob, num_threads=threads)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    return {"value": prob.tokens() * steps / tot, "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{ndocs} of the workload's documents x all {wl.num_heads} heads "
                      f"({prob.tokens()} clean+noisy tokens), fp64, host-generated with the same distributions",
            "seconds_per_step": tot / steps}


def units_for_seconds(wl, target_s: float) -> int:
    """Units (doc, head) the oracle finishes in about target_s on this host (one probe unit)."""
    import oracle
    probe = synth.make_problem_from_layout([0, 512], [128], num_heads=1, d_k=wl.d, d_v=wl.d,
                                           block_size=wl.block_size, num_views=wl.num_views, dtype=wl.dtype,
                                           conv_width=wl.conv_width, device="cpu")
    t0 = time.perf_counter()
    oracle.forward_problem(probe, num_threads=1)
    per_token = (time.perf_counter() - t0) / probe.tokens()
    offs, prompts = synth.doc_layout(wl, 0)
    lens = np.diff(offs)
    unit_tokens = float(np.mean(lens + wl.num_views * (lens - prompts)))
    per_unit = per_token * unit_tokens
    return max(wl.num_heads, int(target_s * host_cores() / max(per_unit, 1e-9)))


def run_reference(args, wl, rank):
    if rank != 0:
        return
    max_units = units_for_seconds(wl, target_s=min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    cb = time_oracle(wl, args.steps, args.warmup, max_units)
    line = {"metric": METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": cb["seconds_per_step"] * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "parallelism": "replicas", "l2": "not applicable (host)"},
            "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- decode side
DECODE_METRIC = "decode-side GDN state cycle (verify K + commit + replay) tokens/s on 1 B200 and % of HBM roofline"


def decode_bytes(N, H, d, L, n_accepted, io_bytes=2):
    """Algorithmic HBM bytes of the three decode kernels (fp32 states, bf16 tokens)."""
    st = d * d * 4
    tok = 3 * d * io_bytes + 8 + d * io_bytes            # q, k, v, g, beta in; o out
    return {"verify": N * H * (st + L * st + L * tok), "commit": n_accepted * H * 2 * st,
            "replay": N * H * (2 * st + L * tok)}


def time_decode_oracle(cfg, seed=0, min_seconds=1.0):
    import oracle  # test infrastructure: the CPU baseline / reference arm only
    pr = synth.make_decode_problem(**cfg, dtype="bf16", seed=seed, device="cpu")
    acc = np.random.Generator(np.random.PCG64(seed)).integers(0, cfg["num_tokens"] + 1, cfg["num_seqs"])
    pool = pr.state_pool.double().numpy()
    slots = pr.slots.numpy()
    threads = min(host_cores(), cfg["num_seqs"] * cfg["num_heads"])
    n, t0 = 0, time.perf_counter()
    while True:
        S0 = pool[slots]
        rec = oracle.decode_steps(S0, pr.q, pr.k, pr.v, pr.g, pr.beta, record_states=True, num_threads=threads)
        pool = oracle.commit(pool, slots, rec["states"], acc)
        rep = oracle.decode_steps(pool[slots], pr.q, pr.k, pr.v, pr.g, pr.beta, num_threads=threads)
        pool[slots] = rep["final_state"]
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    toks = cfg["num_seqs"] * cfg["num_tokens"]
    return {"value": toks * n / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"the whole workload ({cfg['num_seqs']} sequences x {cfg['num_heads']} heads x "
                      f"{cfg['num_tokens']} tokens), {n} verify+commit+replay cycles, fp64",
            "seconds_per_step": el / n}


def run_decode(args, name, rank, world, local):
    cfg = synth.DECODE_WORKLOADS[name]
    N, H, d, L, P = cfg["num_seqs"], cfg["num_heads"], cfg["d"], cfg["num_tokens"], cfg["pool_slots"]
    if args.impl == "reference":
        if rank != 0:
            return
        cb = time_decode_oracle(cfg, min_seconds=2.0)
        line = {"metric": DECODE_METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": cb["seconds_per_step"] * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": name, "parallelism": "replicas", "l2": "not applicable (host)"},
                "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    replicas.init(world, backend="nccl", device=dev)
    seed = replicas.replica_seed(0, rank)
    pr = synth.make_decode_problem(**cfg, dtype="bf16", seed=seed, device=dev)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed + 1)
    accepted = torch.randint(0, L + 1, (N,), generator=gen, dtype=torch.int32).to(dev)
    n_acc = int((accepted > 0).sum())
    out_v = torch.empty(N, L, H, d, dtype=pr.q.dtype, device=dev)
    out_r = torch.empty_like(out_v)
    cache = torch.empty(N, L, H, d, d, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)    # > L2, rewritten between steps
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        gb.decode_verify(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta, out=out_v, state_cache=cache)
        if ev:
            ev[1].record(stream)
        gb.decode_commit(pr.state_pool, pr.slots, cache, accepted)
        if ev:
            ev[2].record(stream)
        gb.decode_replay(pr.state_pool, pr.slots, pr.q, pr.k, pr.v, pr.g, pr.beta, out=out_r)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
        flush.zero_()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        replicas.barrier(world)
        torch.cuda.synchronize()
        clocks.mark_start()
        for i in range(args.steps):
            flush.zero_()                   # L2 flushed before every timed step (outside its events)
            step(evs[i])
        clocks.poll_until(evs[-1][3])
        torch.cuda.synchronize()
        clocks.mark_stop()
        replicas.barrier(world)
    per = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3]),
                     e[0].elapsed_time(e[3])] for e in evs])
    step_ms = replicas.max_over_ranks(float(per[:, 3].mean()), world, device=dev)
    kms = {k: replicas.max_over_ranks(float(per[:, i].mean()), world, device=dev)
           for i, k in enumerate(("verify", "commit", "replay"))}
    by = decode_bytes(N, H, d, L, n_acc)
    peaks = measured_peaks()
    kernels = {k: {"ms": kms[k], "algorithmic_bytes": by[k], "GBps": by[k] / (kms[k] / 1e3) / 1e9,
                   "frac": by[k] / (kms[k] / 1e3) / 1e9 / peaks["hbm_gbs"]} for k in kms}
    roofline = {"bound": "hbm", "achieved": kernels["verify"]["GBps"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": kernels["verify"]["frac"], "traffic": None, "peak_source": peaks["source"],
                "kernel": "gdn_decode_kernel (verify)", "kernels": kernels,
                "step_frac": sum(by.values()) / (step_ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
    toks = N * L * world
    value = toks / (step_ms / 1e3)

    e2e = None
    if not args.no_e2e:
        names = ["q", "k", "v", "g", "beta"]
        host = {n: getattr(pr, n).cpu().pin_memory() for n in names}
        h_acc = accepted.cpu().pin_memory()
        h_ov, h_or = (torch.empty(out_v.shape, dtype=out_v.dtype, pin_memory=True) for _ in range(2))
        dbuf = {n: torch.empty_like(getattr(pr, n)) for n in names}
        d_acc = torch.empty_like(accepted)

        def e2e_step():
            for n in names:
                dbuf[n].copy_(host[n], non_blocking=True)
            d_acc.copy_(h_acc, non_blocking=True)
            gb.decode_verify(pr.state_pool, pr.slots, dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["beta"],
                             out=out_v, state_cache=cache)
            gb.decode_commit(pr.state_pool, pr.slots, cache, d_acc)
            gb.decode_replay(pr.state_pool, pr.slots, dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["beta"],
                             out=out_r)
            h_ov.copy_(out_v, non_blocking=True)
            h_or.copy_(out_r, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ns = max(3, args.steps)
        a.record(stream)
        for _ in range(ns):
            e2e_step()
        z.record(stream)
        torch.cuda.synchronize()
        e2e_ms = replicas.max_over_ranks(a.elapsed_time(z) / ns, world, device=dev)
        h2d = sum(t.numel() * t.element_size() for t in host.values()) + h_acc.numel() * 4
        e2e = {"value": toks / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(2 * h_ov.numel() * h_ov.element_size()), "ms_per_step": e2e_ms,
               "steps": ns}

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = time_decode_oracle(cfg, min_seconds=2.0)
        cpu_baseline = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    replicas.shutdown(world)
    if rank != 0:
        return
    line = {"metric": DECODE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": name, "sequences": N, "heads": H, "d": d, "tokens_per_call": L,
                       "pool_slots": P, "accepted": accepted.tolist(), "parallelism": f"replicas x{world}",
                       "l2": "flushed before every timed step (256 MB write, outside the step's events)"},
            "roofline": roofline, "cpu_baseline": cpu_baseline, "e2e": e2e,
            "gpu_launches": 3 * args.steps, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- softmax attention
ATTN_METRIC = "dual-stream softmax attention fwd tokens/s on 1 B200 and % of tensor roofline"


def attn_pairs(offs, pl, B, V):
    """Visible (query, key) pairs per head under the document-blocked mask."""
    offs = np.asarray(offs, dtype=np.int64)
    pairs = 0
    for n in range(len(pl)):
        L, P = int(offs[n + 1] - offs[n]), int(pl[n])
        pairs += L * (L + 1) // 2
        nb = (L - P) // B
        pairs += V * B * (nb * (P + B) + B * nb * (nb - 1) // 2)   # sum over blocks of P + b0 + B keys
    return pairs


def blas_threads() -> int:
    """Threads of the BLAS behind numpy (the numpy oracles' matrix products), else 1."""
    try:
        from threadpoolctl import threadpool_info
        n = [int(i.get("num_threads", 1)) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_attn_oracle(name, min_seconds=2.0, seed=0):
    """The fp64 oracle on a bounded sample: whole documents of one head (host cores, numpy)."""
    from oracle import attention as oa  # test infrastructure: the CPU baseline / reference arm only
    pr = synth.make_attn_problem(name, seed=seed, device="cpu")
    offs, pl, B = pr.doc_offsets.astype(np.int64), pr.prompt_len, pr.block_size
    V = pr.qn.shape[0]
    Hkv = pr.k.shape[1]
    roffs = np.concatenate([[0], np.cumsum(np.diff(offs) - pl)])
    toks, n, t0 = 0, 0, time.perf_counter()
    while True:
        d_ = n % len(pl)
        s, e, r0, r1 = int(offs[d_]), int(offs[d_ + 1]), int(roffs[d_]), int(roffs[d_ + 1])
        o1 = np.array([0, e - s], dtype=np.int32)
        oa.dual_attention(pr.q[s:e, :1], pr.k[s:e, :1], pr.v[s:e, :1], pr.qn[:, r0:r1, :1], pr.kn[:, r0:r1, :1],
                          pr.vn[:, r0:r1, :1], o1, pl[d_:d_ + 1], B)
        toks += (e - s) + V * (r1 - r0)
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    H = pr.q.shape[1]
    return {"value": toks / el / H, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} whole documents of one head (of {H}; {Hkv} key/value heads) through the fp64 "
                      f"numpy oracle; tokens/s scaled to all heads", "seconds": el}


def run_attention(args, name, rank, world, local):
    cfg = synth.ATTN_WORKLOADS[name]
    if args.impl == "reference":
        if rank != 0:
            return
        cb = time_attn_oracle(name)
        pr = synth.make_attn_problem(name, seed=0, device="cpu")
        toks = pr.q.shape[0] + pr.qn.shape[0] * pr.qn.shape[1]
        line = {"metric": ATTN_METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": toks / cb["value"] * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": name, "parallelism": "replicas", "l2": "not applicable (host)"},
                "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    replicas.init(world, backend="nccl", device=dev)
    pr = synth.make_attn_problem(name, seed=replicas.replica_seed(0, rank), device=dev)
    T, H, d = pr.q.shape
    V, TR = pr.qn.shape[0], pr.qn.shape[1]
    desc = gb.make_attn_desc(len(pr.prompt_len), H, pr.k.shape[1], d, V, pr.block_size, gb.GDN_BF16)
    ws = gb.Workspace(gb.attn_workspace_size(desc, pr.doc_offsets, pr.prompt_len), device=dev).tensor
    out = torch.empty_like(pr.q)
    out_n = torch.empty_like(pr.qn)
    stream = torch.cuda.current_stream(dev)

    def step():
        gb.attention_forward(pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn, pr.doc_offsets, pr.prompt_len, pr.block_size,
                             out=out, out_noisy=out_n, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        replicas.barrier(world)
        torch.cuda.synchronize()
        clocks.mark_start()
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        clocks.poll_until(evs[-1][1])
        torch.cuda.synchronize()
        clocks.mark_stop()
        replicas.barrier(world)
    ms = replicas.max_over_ranks(float(np.mean([a.elapsed_time(z) for a, z in evs])), world, device=dev)
    pairs = attn_pairs(pr.doc_offsets, pr.prompt_len, pr.block_size, V) * H
    flops = 4 * d * pairs
    peaks = measured_peaks()
    achieved = flops / (ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": profiled_traffic("attention", name),
                "peak_source": peaks["source"] + " (burst)",
                "kernel": "gdn_attention_kernel", "algorithmic_flops": flops, "visible_pairs": pairs}
    toks = (T + V * TR) * world
    value = toks / (ms / 1e3)
    e2e = None
    if not args.no_e2e:
        names = ["q", "k", "v", "qn", "kn", "vn"]
        host = {n: getattr(pr, n).cpu().pin_memory() for n in names}
        dbuf = {n: torch.empty_like(getattr(pr, n)) for n in names}
        h_o = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h_on = torch.empty(out_n.shape, dtype=out_n.dtype, pin_memory=True)

        def e2e_step():
            for n in names:
                dbuf[n].copy_(host[n], non_blocking=True)
            gb.attention_forward(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["qn"], dbuf["kn"], dbuf["vn"], pr.doc_offsets,
                                 pr.prompt_len, pr.block_size, out=out, out_noisy=out_n, workspace=ws)
            h_o.copy_(out, non_blocking=True)
            h_on.copy_(out_n, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ns = max(3, args.steps)
        a.record(stream)
        for _ in range(ns):
            e2e_step()
        z.record(stream)
        torch.cuda.synchronize()
        e2e_ms = replicas.max_over_ranks(a.elapsed_time(z) / ns, world, device=dev)
        e2e = {"value": toks / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in host.values())),
               "d2h_bytes_per_step": int(h_o.numel() * 2 + h_on.numel() * 2), "ms_per_step": e2e_ms, "steps": ns}
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = time_attn_oracle(name)
        cpu_baseline = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    replicas.shutdown(world)
    if rank != 0:
        return
    line = {"metric": ATTN_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": name, "layout": cfg["layout"], "heads": H, "kv_heads": int(pr.k.shape[1]), "d": d,
                       "block": pr.block_size, "views": V, "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2 ({sum(t.numel() * t.element_size() for t in (pr.q, pr.k, pr.v, pr.qn, pr.kn, pr.vn)) / 1e9:.2f} GB; K/V reuse inside a call goes through L2)"},
            "roofline": roofline, "cpu_baseline": cpu_baseline, "e2e": e2e,
            "gpu_launches": args.steps, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- backward
BWD_METRIC = "dual-stream GDN backward tokens/s on 1 B200 and % of HBM roofline"
BWD_WORKLOADS = {"bwd_train_8x4096_h16_d128": "train_8x4096_h16_d128",
                 "bwd_conv_4x8192_h16_d128_B4": "conv_4x8192_h16_d128_B4"}


def backward_bytes(prob) -> int:
    """Algorithmic HBM bytes of one backward call: read q, k, v, g, beta (both streams) and the
    upstream output gradients (I/O dtype) and final-state gradient (fp32); write the fp32
    gradients of every input."""
    s = prob.q.element_size()
    d = prob.d_k
    toks = (prob.T + prob.num_views * prob.T_R) * prob.num_heads
    conv = 3 * prob.num_heads * d * 4 * 4 * 2 if prob.conv_width else 0       # weights in, dconv_w out
    return int(toks * (4 * d * s + 8 + 3 * d * 4 + 8) + prob.num_docs * prob.num_heads * d * d * 4 + conv)


def time_backward_oracle(prob, min_seconds=2.0):
    """The fp64 backward oracle on a bounded sample: whole documents of one head."""
    from oracle import backward as ob  # test infrastructure: the CPU baseline / reference arm only
    offs = prob.doc_offsets.astype(np.int64)
    roffs = prob.response_offsets()
    toks, n, t0 = 0, 0, time.perf_counter()
    while True:
        d_ = n % prob.num_docs
        s, e, r0, r1 = int(offs[d_]), int(offs[d_ + 1]), int(roffs[d_]), int(roffs[d_ + 1])
        sl = lambda t: t[s:e, :1]
        sn = lambda t: t[:, r0:r1, :1]
        do = np.ones((e - s, 1, prob.d_v))
        don = np.ones((prob.num_views, r1 - r0, 1, prob.d_v))
        args_ = (sl(prob.q), sl(prob.k), sl(prob.v), sl(prob.g), sl(prob.beta), sn(prob.qn), sn(prob.kn),
                 sn(prob.vn), sn(prob.gn), sn(prob.betan), [0, e - s], prob.prompt_len[d_:d_ + 1], prob.block_size)
        if prob.conv_width:     # head 0's weights: conv_w is [3, H d, W]
            ob.dual_backward_conv(*args_, prob.conv_w[:, :prob.d_k, :], do, don, None)
        else:
            ob.dual_backward(*args_, do, don, None)
        toks += (e - s) + prob.num_views * (r1 - r0)
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return {"value": toks / el / prob.num_heads, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} whole documents of one head (of {prob.num_heads}) through the fp64 numpy backward "
                      f"oracle; tokens/s scaled to all heads", "seconds": el}


def run_backward(args, name, rank, world, local):
    wl = synth.get_workload(BWD_WORKLOADS[name])
    if args.impl == "reference":
        if rank != 0:
            return
        prob = synth.make_problem(wl, seed=0, device="cpu")
        cb = time_backward_oracle(prob)
        line = {"metric": BWD_METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": prob.tokens() / cb["value"] * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": name, "parallelism": "replicas", "l2": "not applicable (host)"},
                "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    replicas.init(world, backend="nccl", device=dev)
    prob = synth.make_problem(wl, seed=replicas.replica_seed(0, rank), device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7 + rank)
    do = torch.randn(prob.T, prob.num_heads, prob.d_v, generator=gen, device=dev).to(prob.q.dtype)
    don = torch.randn(prob.num_views, prob.T_R, prob.num_heads, prob.d_v, generator=gen, device=dev).to(prob.q.dtype)
    desc = gb.make_desc(prob.num_docs, prob.num_heads, prob.d_k, prob.d_v, prob.num_views, prob.block_size,
                        gb._dtype_code(prob.q), prob.conv_width)
    wsize = (gb.backward_conv_workspace_size(desc, prob.doc_offsets) if prob.conv_width
             else gb.backward_workspace_size(desc, prob.doc_offsets))
    ws = gb.Workspace(wsize, device=dev).tensor
    names = ("q", "k", "v", "g", "beta", "qn", "kn", "vn", "gn", "betan")
    ins = [getattr(prob, n) for n in names]
    stream = torch.cuda.current_stream(dev)

    def step(inputs=None, d_o=None, d_on=None):
        return gb.backward(*(inputs or ins), prob.doc_offsets, prob.prompt_len, prob.block_size,
                           do if d_o is None else d_o, don if d_on is None else d_on, None,
                           conv_w=prob.conv_w, workspace=ws)

    steps = max(1, args.steps)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with ClockSampler(local) as clocks:
        replicas.barrier(world)
        torch.cuda.synchronize()
        clocks.mark_start()
        for i in range(steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        clocks.poll_until(evs[-1][1])
        torch.cuda.synchronize()
        clocks.mark_stop()
        replicas.barrier(world)
    ms = replicas.max_over_ranks(float(np.mean([a.elapsed_time(z) for a, z in evs])), world, device=dev)
    nbytes = backward_bytes(prob)
    peaks = measured_peaks()
    gbps = nbytes / (ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": gbps, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbps / peaks["hbm_gbs"], "traffic": None, "peak_source": peaks["source"],
                "kernel": "gdn_backward_kernel" + (" (+ ShortConv forward, backward and weight-gradient kernels)"
                                                   if prob.conv_width else ""), "algorithmic_bytes": nbytes}
    toks = prob.tokens() * world
    value = toks / (ms / 1e3)
    e2e = None
    if not args.no_e2e:
        host = {n: getattr(prob, n).cpu().pin_memory() for n in names}
        h_do, h_don = do.cpu().pin_memory(), don.cpu().pin_memory()
        dbuf = {n: torch.empty_like(getattr(prob, n)) for n in names}
        d_do, d_don = torch.empty_like(do), torch.empty_like(don)
        outs_h = None

        def e2e_step():
            nonlocal outs_h
            for n in names:
                dbuf[n].copy_(host[n], non_blocking=True)
            d_do.copy_(h_do, non_blocking=True)
            d_don.copy_(h_don, non_blocking=True)
            gr = step([dbuf[n] for n in names], d_do, d_don)
            if outs_h is None:
                outs_h = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in gr.items()}
            for k, v in gr.items():
                outs_h[k].copy_(v, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ns = 3
        a.record(stream)
        for _ in range(ns):
            e2e_step()
        z.record(stream)
        torch.cuda.synchronize()
        e2e_ms = replicas.max_over_ranks(a.elapsed_time(z) / ns, world, device=dev)
        e2e = {"value": toks / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in host.values())
                                         + h_do.numel() * h_do.element_size() + h_don.numel() * h_don.element_size()),
               "d2h_bytes_per_step": int(sum(t.numel() * t.element_size() for t in outs_h.values())),
               "ms_per_step": e2e_ms, "steps": ns}
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = time_backward_oracle(synth.make_problem(wl, seed=0, device="cpu"))
        cpu_baseline = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    replicas.shutdown(world)
    if rank != 0:
        return
    # kernels of one backward call: the backward kernel and four slice reductions per stream (dq,
    # dk, dg, dbeta); with ShortConv also the conv forward, the bf16 upstream-gradient casts (one
    # per stream), the conv backward and the weight gradient
    noisy_bwd = prob.num_views > 0 and prob.T_R > 0
    bwd_launches = 1 + 4 + (4 if noisy_bwd else 0)
    if prob.conv_width:
        bwd_launches += 1 + ((1 + (1 if noisy_bwd else 0)) if prob.q.dtype == torch.bfloat16 else 0) + 2
    line = {"metric": BWD_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 I/O, fp32 arithmetic and gradients", "data": "synthetic",
            "config": {"workload": name, "layout": BWD_WORKLOADS[name], "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2"},
            "roofline": roofline, "cpu_baseline": cpu_baseline, "e2e": e2e,
            "gpu_launches": bwd_launches * steps, "launches_per_step": bwd_launches, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "sequential", "chunked", "route1", "pipelined"])
    ap.add_argument("--e2e-groups", type=int, default=8,
                    help="document groups of the host-buffer call (its copies in and out overlap across groups)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local = replicas.env_rank()
    if args.workload in synth.DECODE_WORKLOADS:
        run_decode(args, args.workload, rank, world, local)
        return
    if args.workload in synth.ATTN_WORKLOADS:
        run_attention(args, args.workload, rank, world, local)
        return
    if args.workload in BWD_WORKLOADS:
        run_backward(args, args.workload, rank, world, local)
        return
    wl = synth.get_workload(args.workload)

    if args.impl == "reference":
        run_reference(args, wl, rank)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    replicas.init(world, backend="nccl", device=dev)
    algo = {"auto": gb.ALGO_AUTO, "sequential": gb.ALGO_SEQUENTIAL, "chunked": gb.ALGO_CHUNKED,
            "route1": gb.ALGO_ROUTE1, "pipelined": gb.ALGO_PIPELINED}[args.algo]

    prob = synth.make_problem(wl, seed=replicas.replica_seed(0, rank), device=dev)
    T, TR, V, H, d = prob.T, prob.T_R, prob.num_views, prob.num_heads, prob.d_k
    desc = gb.make_desc(prob.num_docs, H, d, d, V, prob.block_size, gb._dtype_code(prob.q), prob.conv_width, algo)
    used_algo = gb.select_algo(desc)
    ws = gb.Workspace(gb.workspace_size_route1(desc, prob.doc_offsets, prob.prompt_len) if algo == gb.ALGO_ROUTE1
                      else gb.workspace_size(desc, prob.doc_offsets), device=dev)
    out = torch.empty(T, H, d, dtype=prob.q.dtype, device=dev)
    out_n = torch.empty(V, TR, H, d, dtype=prob.q.dtype, device=dev)
    fs = torch.empty(prob.num_docs, H, d, d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        gb.forward_problem(prob, algo=algo, out=out, out_noisy=out_n, final_state=fs, workspace=ws)

    def barrier():
        replicas.barrier(world)

    def max_over_ranks(x: float) -> float:
        return replicas.max_over_ranks(x, world, device=dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dstatus = gb.read_device_status(ws)

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        clocks.mark_start()
        start.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        stop.record(stream)
        clocks.poll_until(stop)
        torch.cuda.synchronize()
        clocks.mark_stop()
        barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(stop))
    launch_ms = [a.elapsed_time(b) for a, b in evs]
    kernel_ms = max_over_ranks(sum(launch_ms) / len(launch_ms))

    work = algorithmic_work(prob)
    toks_all = prob.tokens() * world
    value = replicas.throughput(prob.tokens(), world, args.steps, elapsed_ms)
    peaks = measured_peaks()
    achieved_gbs = work["bytes"] / (kernel_ms / 1e3) / 1e9
    traffic = profiled_traffic(used_algo, wl.name, work["bytes"])
    # ShortConv under AUTO with a full-size workspace: the call is the conv pass, then the chunked
    # kernel on the convolved copies; the events time both, against the forward's algorithmic bytes
    conv_pass = (algo == gb.ALGO_AUTO and used_algo == gb.ALGO_CHUNKED and prob.conv_width == 4
                 and gb.workspace_size(desc, prob.doc_offsets) > 256)
    # Route I on tensor cores (bf16, d = 128, B in {16, 32}; ShortConv as a pass of its own first)
    r1_tc = (used_algo == gb.ALGO_ROUTE1 and prob.q.dtype == torch.bfloat16 and d == 128
             and prob.block_size in (16, 32))
    if r1_tc:
        traffic = profiled_traffic("route1_tc", wl.name, work["bytes"])
    # kernels one forward call launches: the chunked kernel once per pair of views (each launch
    # recomputes the clean stream), plus the ShortConv pass; Route I two stages (plus the conv pass)
    v_eff = V if TR > 0 else 0
    if used_algo in (gb.ALGO_CHUNKED, gb.ALGO_PIPELINED):
        launches = max(1, (v_eff + 1) // 2) + (1 if conv_pass else 0)
    elif used_algo == gb.ALGO_ROUTE1:
        launches = 1 + (1 if v_eff > 0 else 0) + (1 if r1_tc and prob.conv_width == 4 else 0)
    else:
        launches = 1
    kname = ("conv_pass_kernel + " + KERNEL_NAMES[used_algo] + " (one forward call)") if conv_pass \
        else ("conv_pass_kernel + " if prob.conv_width == 4 else "") + KERNEL_NAMES["route1_tc"] if r1_tc \
        else KERNEL_NAMES.get(used_algo)
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": peaks["source"], "kernel": kname,
                "algorithmic_bytes_per_launch": work["bytes"], "algorithmic_flops_per_launch": work["flops"],
                "tensor_frac_at_algorithmic_flops": work["flops"] / (kernel_ms / 1e3) / 1e12 / peaks["bf16_tflops"]}

    # ---- end to end through the public API: pinned host inputs in, outputs back to pinned host
    #      memory, by gdn_dual_forward_host (document groups pipelined across the host link) ----
    e2e = None
    if not args.no_e2e:
        names = ["q", "k", "v", "g", "beta", "qn", "kn", "vn", "gn", "betan"] + (["conv_w"] if prob.conv_w is not None else [])
        host = {n: getattr(prob, n).cpu().pin_memory() for n in names}
        h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h_outn = torch.empty(out_n.shape, dtype=out_n.dtype, pin_memory=True)
        h_fs = torch.empty(fs.shape, dtype=fs.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in (h_out, h_outn, h_fs))
        staging = torch.empty(gb.host_staging_size(desc, prob.doc_offsets, prob.prompt_len, args.e2e_groups),
                              dtype=torch.uint8, device=dev)

        def e2e_step():
            st = gb.forward_host_raw(desc, host["q"], host["k"], host["v"], host["g"], host["beta"], host["qn"],
                                     host["kn"], host["vn"], host["gn"], host["betan"], prob.doc_offsets,
                                     prob.prompt_len, host.get("conv_w"), h_out, h_outn, h_fs, staging,
                                     args.e2e_groups, stream=stream.cuda_stream)
            if st != gb.GDN_OK:
                raise gb.GdnError(st, f"gdn_dual_forward_host failed: {gb.status_string(st)}")

        e2e_steps = max(3, min(args.steps, 10))
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        z.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(z)) / e2e_steps
        e2e = {"value": toks_all / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms, "steps": e2e_steps,
               "api": "gdn_dual_forward_host", "groups": args.e2e_groups,
               "host_status": gb.status_string(gb.read_host_device_status(staging, stream.cuda_stream)[0])}
        del host, staging

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        max_units = units_for_seconds(wl, target_s=8.0)
        cb = time_oracle(wl, steps=1, warmup=1, max_units=max_units)
        cpu_baseline = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}

    replicas.shutdown(world)
    if rank != 0:
        return
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if prob.q.dtype == torch.bfloat16 else "fp32",
            "data": "synthetic",
            "config": {"workload": wl.name, "docs": prob.num_docs, "tokens_clean": T, "tokens_noisy": V * TR,
                       "heads": H, "d": d, "block_size": prob.block_size, "views": V, "conv_width": prob.conv_width,
                       "algo": {1: "sequential", 2: "chunked", 3: "route1", 4: "pipelined"}.get(used_algo, str(used_algo)),
                       "parallelism": f"replicas x{world}", "l2": "inputs larger than L2 (no flush)"},
            "roofline": roofline, "cpu_baseline": cpu_baseline, "e2e": e2e,
            "gpu_launches": launches * args.steps, "launches_per_step": launches, "clocks": clocks.summary(),
            "device_status": gb.status_string(dstatus), "kernel_ms_mean": kernel_ms}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
