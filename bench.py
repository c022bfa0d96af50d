#!/usr/bin/env python
"""Benchmark: dynamic short convolution forward + backward tokens/s on B200.

One step = one forward and one backward pass of every layer of the workload
(the hot path: filter generation, causal conv + residual, du, dz/dwh, dA/dB or
dW, dh) over one batch of seeded synthetic inputs already resident in HBM.
The default workload is the 2B-scale all-linear block (B=4, T=4096, K=3,
low-rank r=64, bf16; one dynamic conv after each of the QKV (d 2048, C 3072),
O (2048, 2048), gate+up (2048, 11264) and down (5632, 2048) linears).

Prints ONE JSON line (rank 0).  Under torchrun each rank runs its own replica
on its own seeded shard (weak scaling, no data-path collective); the timing
is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dyn-conv fwd+bwd tokens/s at 1 B200; achieved HBM GB/s vs ~8 TB/s roofline"
DEFAULT_CONFIG = "c4_all_linear_2b_block"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def cores_used() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    if n and n.isdigit():
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- algorithmic traffic
def layer_bytes(w, layer):
    """Algorithmic HBM bytes of one forward+backward of one layer call: every tensor
    the op must read or write, once (bf16 storage s bytes, fp32 parameter grads):
    fwd reads u, h, writes y, z; bwd reads g, u, h, z, writes du, dh; parameters
    A, B (or W) read in both passes; dA, dB (or dW) written once.  The [N,C,K]
    filter is never materialised, so it counts zero."""
    s = 2 if w.dtype == "bf16" else 4
    N, d, C, K = w.tokens, layer.d_model, layer.channels, w.ksize
    per_tok = s * (2 * C + d) + s * (3 * C + d) + s * d   # fwd u,y,h ; bwd g,u,du,h ; dh
    if w.kind == "lowrank":
        r = w.rank
        per_tok += 2 * s * r                               # z written in fwd, read in bwd
        params = 2 * s * (d * r + r * C * K) + 4 * (d * r + r * C * K)
    else:
        H = C // w.head_dim
        params = 2 * s * d * H * K + 4 * d * H * K
    return N * per_tok + params


def layer_flops(w, layer):
    """Tensor-core FLOPs of one forward+backward: low-rank 2rCK per token for each of
    w (fwd), w (bwd recompute), dz and dB, plus 2dr for z, dA and dh; head-wise
    2dHK for the filters, dW and dh."""
    N, d, C, K = w.tokens, layer.d_model, layer.channels, w.ksize
    if w.kind == "lowrank":
        return N * (8 * w.rank * C * K + 6 * d * w.rank)
    H = C // w.head_dim
    return N * 6 * d * H * K


# DRAM bytes (read + write) per launch of a workload's dominant kernel, averaged over the launches
# of one step, from an ncu capture of dram__bytes_read.sum + dram__bytes_write.sum, keyed by
# (kernel, workload) and stored with the SHA-256 of the kernel's source files at capture time: a
# figure is reported only while those files are unchanged (else traffic is null).
NCU_TRAFFIC = {
    ("tc_lowrank_bwd", "c4_all_linear_2b_block"): (550760853, "d9ad7f0ee6101c83"),
    ("tc_lowrank_bwd", "c2_qkv_150m_lowrank"): (192719232, "d9ad7f0ee6101c83"),
    ("tc_headwise_bwd", "c3_qkv_2b_headwise_gqa"): (302353258, "c06e68dc5e1a32cf"),
    ("tc_lowrank_bwd", "c5_varlen_packed"): (2170718763, "d9ad7f0ee6101c83"),
}
KERNEL_SOURCES = {
    "tc_lowrank_bwd": ("tc_bwd.cu", "tc_common.cuh", "common.cuh"),
    "tc_lowrank_fwd": ("tc.cu", "tc_common.cuh", "common.cuh"),
    "tc_headwise_bwd": ("tc_headwise.cu", "tc_common.cuh", "common.cuh"),
    "tc_headwise_fwd": ("tc_headwise.cu", "tc_common.cuh", "common.cuh"),
}


def kernel_source_sha(name):
    """SHA-256 (first 16 hex digits) over the source files of a kernel family, or None."""
    import hashlib

    files = KERNEL_SOURCES.get(name)
    if not files:
        return None
    hsh = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "dynamic_short_convolutions_b200", "csrc", f), "rb") as fh:
            hsh.update(fh.read())
    return hsh.hexdigest()[:16]


def ncu_traffic(name, workload):
    rec = NCU_TRAFFIC.get((name, workload))
    if rec is None:
        return None
    nbytes, sha = rec
    return nbytes if sha == kernel_source_sha(name) else None


def kernel_flops(name, w, layer):
    """Tensor-core FLOPs of ONE launch of a library kernel on one layer call (0 for CUDA-core kernels)."""
    N, d, C, K = w.tokens, layer.d_model, layer.channels, w.ksize
    if w.kind == "lowrank":
        R = w.rank
        conv = {"tc_lowrank_fwd": 2 * N * R * C * K, "tc_lowrank_bwd": 6 * N * R * C * K}
    else:
        R = (C // w.head_dim) * K
        conv = {}
    table = {"tc_gen": 2 * N * d * R, "tc_gen_bwd": 4 * N * d * R, **conv}
    return table.get(name, 0)


def kernel_bytes(name, w, layer):
    """Algorithmic bytes of ONE launch of a library kernel on one layer call
    (inputs read once, outputs written once, at the kernel's interface)."""
    s = 2 if w.dtype == "bf16" else 4
    N, d, C, K = w.tokens, layer.d_model, layer.channels, w.ksize
    if w.kind == "lowrank":
        R, P = w.rank, d * w.rank
        BW = w.rank * C * K
    else:
        R = (C // w.head_dim) * K
        P = d * R
        BW = 0
    table = {
        "simt_gen": N * d * s + P * s + N * R * (4 + (s if w.kind == "lowrank" else 0)),
        "simt_widen": N * R * (s + 4),
        "simt_conv_fwd": N * C * 2 * s + N * R * 4 + BW * s,
        "simt_conv_bwd": N * C * 3 * s + N * R * 8 + BW * s,
        "simt_dB": N * R * 4 + N * C * 2 * s + BW * 4,
        "simt_hTX": N * d * s + N * R * 4 + P * 4,
        "simt_dh": N * R * 4 + P * s + N * d * s,
        "tc_gen": N * d * s + P * s + N * R * s,
        "tc_lowrank_fwd": N * C * 2 * s + N * R * s + BW * s,
        "tc_lowrank_bwd": N * C * 3 * s + N * R * s + BW * s,
        "tc_gen_bwd": N * d * 2 * s + N * R * s + P * (s + 4),
        "tc_headwise_fwd": N * C * 2 * s + N * R * s,
        "tc_headwise_bwd": N * C * 3 * s + N * R * 4,
    }
    return table.get(name)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML every 20 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml as N

            N.nvmlInit()
            import torch

            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = N.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
            self.N = N
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _run(self):
        N = self.N
        while not self._stop.is_set():
            try:
                sm = N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM)
                rs = N.nvmlDeviceGetCurrentClocksEventReasons(self.h) \
                    if hasattr(N, "nvmlDeviceGetCurrentClocksEventReasons") \
                    else N.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                util = N.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((sm, rs, util))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": getattr(self, "err", "no NVML")}
        busy = [s for s in self.samples if s[2] > 0] or self.samples
        reasons = set()
        for _, rs, _ in busy:
            for bit, nm in self.REASONS.items():
                if rs & bit and nm != "gpu_idle":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median([s[0] for s in busy]) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(busy)}


# ----------------------------------------------------------------------------- CPU oracle leg
class OracleSample:
    """The fp64 oracle (as it stands) on a bounded sample of the workload: forward,
    per-token backward and parameter gradients of every layer on the first
    `seqs` sequences of the batch, truncated to T tokens each.  Inputs are drawn
    once, outside the timing."""

    def __init__(self, w, seqs, T):
        from dynamic_short_convolutions_b200 import workloads as W
        from oracle import oracle as O

        O.build()
        self.O = O
        self.tokens = seqs * T
        ws = W.scaled(w, seqs, T, name="oracle_sample")
        if ws.varlen:   # a prefix of the packed stream, with its own document boundaries
            import dataclasses
            ws = dataclasses.replace(ws, varlen=False)
        cu = [i * T for i in range(seqs + 1)]
        self.calls = []
        for li, layer in enumerate(ws.layers):
            x = W.make_inputs(ws, layer, li)
            p = O.Problem(O.LOWRANK if ws.kind == W.LOWRANK else O.HEADWISE, seqs * T, layer.d_model,
                          layer.channels, ws.ksize, cu, rank=ws.rank, head_dim=ws.head_dim)
            self.calls.append((p, x, x.get("A"), x["B"] if ws.kind == W.LOWRANK else x["W"]))

    def run(self) -> float:
        O = self.O
        t0 = time.perf_counter()
        for p, x, A, BW in self.calls:
            O.forward(p, x["u"], x["h"], A, BW)
            O.backward_rows(p, x["g"], x["u"], x["h"], A, BW)
            O.param_grads(p, x["g"], x["u"], x["h"], A, BW)
        return time.perf_counter() - t0


def oracle_sample_shape(w, budget_s: float):
    """(sequences, tokens per sequence) of a sample whose oracle run takes about
    budget_s seconds: whole sequences while they fit, else a prefix of one."""
    n_cal = min(256, w.seqlen)
    cal = OracleSample(w, 1, n_cal)
    per_tok = max(cal.run() / n_cal, 1e-7)
    want = max(16, int(budget_s / per_tok))
    if want <= w.seqlen:
        return 1, want
    return max(1, min(w.batch, want // w.seqlen)), w.seqlen


def oracle_sample_rate(w, budget_s: float):
    """(tokens/s, description, seconds) of one oracle run sized to about budget_s seconds."""
    seqs, T = oracle_sample_shape(w, budget_s)
    smp = OracleSample(w, seqs, T)
    secs = smp.run()
    return smp.tokens / secs, f"{seqs} sequence(s) x {T} tokens", secs


# ----------------------------------------------------------------------------- decode mode
DECODE_METRIC = "dyn-conv decode-step tokens/s at 1 B200 (one new token per sequence, rolling K-1 state)"


def decode_bytes(w, layer, batch):
    """Algorithmic HBM bytes of one decode step of one layer call: u, h read, y written,
    the state read and rewritten, the generator parameters read once."""
    s = 2 if w.dtype == "bf16" else 4
    d, C, K = layer.d_model, layer.channels, w.ksize
    per_seq = s * (2 * C + d + 2 * (K - 1) * C)
    if w.kind == "lowrank":
        params = s * (d * w.rank + w.rank * C * K)
    else:
        params = s * d * (C // w.head_dim) * K
    return batch * per_seq + params


def run_decode(args, rank, world, local_rank):
    """Decode steps of every layer of the workload for a batch of sequences: one call of
    dynconv_decode_step per layer per step, L2 flushed between timed steps."""
    import numpy as np
    import torch

    from dynamic_short_convolutions_b200 import _lib as L, workloads as W

    L.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = W.CONFIGS[args.config]
    Bd = args.decode_batch
    dt = W.storage_dtype(w)
    kind = L.LOWRANK if w.kind == W.LOWRANK else L.HEADWISE
    seed = shard_seed(w.seed, rank)
    calls = []
    for li, layer in enumerate(w.layers):
        d, C, K = layer.d_model, layer.channels, w.ksize
        rnd = lambda tag, n, std=1.0: W.normal_torch(seed, f"dec{li}{tag}", n, std, device=dev).to(dt)
        if kind == L.LOWRANK:
            A = rnd("A", d * w.rank, 1 / np.sqrt(d)).view(d, w.rank)
            BW = rnd("B", w.rank * C * K, 1 / np.sqrt(w.rank)).view(w.rank, C * K)
        else:
            A = None
            BW = rnd("W", d * (C // w.head_dim) * K, 1 / np.sqrt(d)).view(d, (C // w.head_dim) * K)
        u, h = rnd("u", Bd * C).view(Bd, C), rnd("h", Bd * d).view(Bd, d)
        desc = L.make_desc(kind, L.BF16 if dt == torch.bfloat16 else L.F32, Bd, 1, d, C, K, w.rank, w.head_dim)
        ws = torch.zeros(L.dynconv_workspace_bytes(desc), dtype=torch.uint8, device=dev)
        state = torch.zeros((Bd, K - 1, C), dtype=dt, device=dev) if K > 1 else None
        y = torch.empty((Bd, C), dtype=dt, device=dev)
        calls.append((layer, desc, u, h, A, BW, state, y, ws))
    stream = torch.cuda.current_stream(dev)

    def step():
        for layer, desc, u, h, A, BW, state, y, ws in calls:
            L.dynconv_decode_step(desc, u, h, A, BW, state, y, ws)

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for *_, ws in calls:
        assert L.dynconv_device_status(ws) == 0, L.dynconv_last_error()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(float(sum(a.elapsed_time(b) for a, b in ev)), world, dev)
    L.dynconv_profile_read(reset=True)
    L.dynconv_profile_enable(True)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()
    L.dynconv_profile_enable(False)
    prof = L.dynconv_profile_read(reset=True)
    # end to end: the step's inputs copied in from pinned host memory, outputs copied back
    host = [(u.cpu().pin_memory(), h.cpu().pin_memory(), torch.empty_like(y, device="cpu").pin_memory())
            for _, _, u, h, _, _, _, y, _ in calls]
    h2d = sum(a.numel() * a.element_size() + b.numel() * b.element_size() for a, b, _ in host)
    d2h = sum(c.numel() * c.element_size() for _, _, c in host)

    def e2e_step():
        for (layer, desc, u, h, A, BW, state, y, ws), (hu, hh, hy) in zip(calls, host):
            u.copy_(hu, non_blocking=True)
            h.copy_(hh, non_blocking=True)
            L.dynconv_decode_step(desc, u, h, A, BW, state, y, ws)
            hy.copy_(y, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    pk, pk_src = peaks()
    ms_step = total_ms / args.steps
    step_bytes = sum(decode_bytes(w, c[0], Bd) for c in calls)
    achieved = step_bytes / (ms_step / 1e3) / 1e9
    kernels = {n: {"launches": nl, "ms_total": round(ms, 4), "us_per_launch": round(1e3 * ms / nl, 2)}
               for n, (nl, ms) in prof.items()}
    line = {"metric": DECODE_METRIC, "mode": "decode", "value": round(job_throughput(Bd, world, args.steps, total_ms), 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "decode_batch": Bd, "ksize": w.ksize, "rank": w.rank,
                       "head_dim": w.head_dim, "layers": [[l.name, l.d_model, l.channels] for l in w.layers],
                       "l2": "flushed between timed steps (256 MiB write, outside the step events)"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": None, "peak_source": pk_src,
                         "algorithmic_bytes_per_step": int(step_bytes)},
            "kernels": kernels,
            "e2e": {"value": round(job_throughput(Bd, world, args.steps, e2e_ms), 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
            "gpu_launches": int(sum(v[0] for v in prof.values())), "clocks": clk.summary()}
    return line


def oracle_decode_rate(w, batch, budget_s):
    """tokens/s of the fp64 oracle's decode step on the workload's layers (batch sequences)."""
    import numpy as np

    from dynamic_short_convolutions_b200 import workloads as W
    from oracle import oracle as O

    O.build()
    calls = []
    for li, layer in enumerate(w.layers):
        d, C, K = layer.d_model, layer.channels, w.ksize
        rnd = lambda tag, n, std=1.0: W.round_to_storage(W.normal(w.seed, f"odec{li}{tag}", n, std), w.dtype)
        if w.kind == W.LOWRANK:
            A, BW = rnd("A", d * w.rank).reshape(d, w.rank), rnd("B", w.rank * C * K).reshape(w.rank, C * K)
        else:
            A, BW = None, rnd("W", d * (C // w.head_dim) * K).reshape(d, (C // w.head_dim) * K)
        p = O.Problem(O.LOWRANK if w.kind == W.LOWRANK else O.HEADWISE, batch, d, C, K, [0, batch], rank=w.rank,
                      head_dim=w.head_dim)
        calls.append((p, rnd("u", batch * C).reshape(batch, C), rnd("h", batch * d).reshape(batch, d), A, BW,
                      np.zeros((batch, K - 1, C))))
    steps, t0 = 0, time.perf_counter()
    while True:
        for i, (p, u, h, A, BW, st) in enumerate(calls):
            _, st = O.decode_step(p, u, h, A, BW, st)
            calls[i] = (p, u, h, A, BW, st)
        steps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    secs = time.perf_counter() - t0
    return batch * steps / secs, f"{steps} decode step(s) of {batch} sequences, every layer", secs


# ----------------------------------------------------------------------------- ranks
def shard_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s shard of a workload: each rank draws its own tokens (weak
    scaling, replicas with no exchange in the hot path)."""
    return seed + 7919 * rank


def max_over_ranks(value: float, world: int, device="cpu") -> float:
    """The maximum of `value` over the ranks (device time of the slowest rank); the value
    itself with one rank."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: the tokens every rank processed over the slowest rank's time."""
    return tokens_per_rank * world * steps / (max_ms / 1e3)


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from dynamic_short_convolutions_b200 import _lib as L, ops, workloads as W

    L.load()  # fails loudly if the CUDA library is missing
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = W.CONFIGS[args.config]
    if rank:
        import dataclasses
        w = dataclasses.replace(w, seed=shard_seed(w.seed, rank))   # each rank: its own shard
    kind = L.LOWRANK if w.kind == W.LOWRANK else L.HEADWISE
    dt = W.storage_dtype(w)
    layers = []
    for li, layer in enumerate(w.layers):
        t = W.make_inputs(w, layer, li, device=dev)
        batch, seqlen = (1, w.tokens) if w.varlen else (w.batch, w.seqlen)
        cf = args.layout == "channel_first"
        rope = W.ROPE_QKV.get(w.name) if args.rope and layer.name == "qkv" else None
        table = ops.rope_table(max(seqlen, 1), rope[1], device=dev) if rope else None
        plan = ops.DynConvPlan(kind, dt, batch, seqlen, layer.d_model, layer.channels, w.ksize, w.rank,
                               w.head_dim, algo=args.algo, device=dev, deterministic=args.deterministic,
                               layout=L.CHANNEL_FIRST if cf else L.TOKEN_MAJOR,
                               rope_channels=rope[0] if rope else 0, rope_head_dim=rope[1] if rope else 0,
                               rope_table=table)
        A = t.get("A")
        BW = t["B"] if kind == L.LOWRANK else t["W"]
        N = w.tokens
        conv_shape = (batch, layer.channels, seqlen) if cf else (N, layer.channels)
        if cf:      # u and g stored [batch, C, seqlen] (converted once, outside the timed region)
            for k in ("u", "g"):
                t[k] = t[k].reshape(batch, seqlen, layer.channels).transpose(1, 2).contiguous()
        bufs = dict(y=torch.empty(conv_shape, dtype=dt, device=dev),
                    z=torch.empty((N, w.rank if kind == L.LOWRANK else (layer.channels // w.head_dim) * w.ksize),
                                  dtype=dt, device=dev),
                    out={"du": torch.empty(conv_shape, dtype=dt, device=dev),
                         "dh": torch.empty((N, layer.d_model), dtype=dt, device=dev),
                         "dA": torch.empty(tuple(A.shape), dtype=torch.float32, device=dev) if A is not None else None,
                         "dBW": torch.empty(tuple(BW.shape), dtype=torch.float32, device=dev)})
        cu = t["cu_seqlens"] if w.varlen else None
        layers.append((layer, t, plan, A, BW, cu, bufs))
    fam = L.dynconv_query_family(layers[0][2].desc)
    stream = torch.cuda.current_stream(dev)

    def step():
        for layer, t, plan, A, BW, cu, b in layers:
            plan.forward(t["u"], t["h"], A, BW, cu, y=b["y"], z_save=b["z"])
            plan.backward(t["g"], t["u"], t["h"], A, BW, cu, z_saved=b["z"], out=b["out"])

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for _, _, plan, *_ in layers:
        assert L.dynconv_device_status(plan.ws) == 0, L.dynconv_last_error()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    # Per-kernel device times: the same steps again with the library's launch tracer on
    # (events on the launch stream around every launch; these serialise the launches, so
    # the step time above is measured with the tracer off).
    L.dynconv_profile_read(reset=True)
    L.dynconv_profile_enable(True)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()
    L.dynconv_profile_enable(False)
    prof = L.dynconv_profile_read(reset=True)
    total_ms = max_over_ranks(float(sum(step_ms)), world, dev)
    value = job_throughput(w.tokens, world, args.steps, total_ms)

    # ---- e2e through the public API with host buffers (pinned), copies inside the timed region
    host = []
    h2d = d2h = 0
    for layer, t, plan, A, BW, cu, b in layers:
        hin = {k: v.to("cpu").pin_memory() for k, v in t.items() if k in ("u", "h", "g", "A", "B", "W")}
        hout = {"y": torch.empty_like(b["y"], device="cpu").pin_memory(),
                "du": torch.empty_like(b["out"]["du"], device="cpu").pin_memory(),
                "dh": torch.empty_like(b["out"]["dh"], device="cpu").pin_memory(),
                "dBW": torch.empty_like(b["out"]["dBW"], device="cpu").pin_memory()}
        if b["out"]["dA"] is not None:
            hout["dA"] = torch.empty_like(b["out"]["dA"], device="cpu").pin_memory()
        h2d += sum(v.numel() * v.element_size() for v in hin.values())
        d2h += sum(v.numel() * v.element_size() for v in hout.values())
        host.append((hin, hout))

    # Copies run on their own streams (host -> device on one, device -> host on the other, PCIe being
    # full duplex) and overlap the compute of other layers, as a caller's input pipeline would; events
    # order each layer's copies against its compute in both directions (a layer's inputs are not
    # overwritten before its compute has read them, its outputs not before they have been copied out).
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = [{k: torch.cuda.Event() for k in ("in_ready", "done", "out_free")} for _ in layers]

    def e2e_step():
        for (layer, t, plan, A, BW, cu, b), (hin, hout), e in zip(layers, host, ev):
            with torch.cuda.stream(s_in):
                s_in.wait_event(e["done"])                   # the previous step's compute read these inputs
                for k, v in hin.items():
                    t[k].copy_(v, non_blocking=True)
                e["in_ready"].record(s_in)
            stream.wait_event(e["in_ready"])
            stream.wait_event(e["out_free"])                 # the previous step's outputs are copied out
            plan.forward(t["u"], t["h"], t.get("A"), t["B"] if "B" in t else t["W"], cu, y=b["y"], z_save=b["z"])
            plan.backward(t["g"], t["u"], t["h"], t.get("A"), t["B"] if "B" in t else t["W"], cu,
                          z_saved=b["z"], out=b["out"])
            e["done"].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e["done"])
                hout["y"].copy_(b["y"], non_blocking=True)
                for k in ("du", "dh", "dBW", "dA"):
                    if k in hout:
                        hout[k].copy_(b["out"][k], non_blocking=True)
                e["out_free"].record(s_out)

    for _ in range(max(1, min(args.warmup, 3))):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 20))
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for _ in range(e2e_steps):
        e2e_step()
    done_in, done_out = torch.cuda.Event(), torch.cuda.Event()
    done_in.record(s_in)
    done_out.record(s_out)
    stream.wait_event(done_in)
    stream.wait_event(done_out)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_throughput(w.tokens, world, e2e_steps, e2e_ms)

    # ---- roofline of the dominant kernel (live CUDA-event timing from the library's tracer)
    pk, pk_src = peaks()
    launches = sum(v[0] for v in prof.values())   # our kernels in the timed steps (same launches per step)
    dom = max(prof.items(), key=lambda kv: kv[1][1]) if prof else None
    roof = None
    kernels = {}
    prof_total = sum(ms for _, ms in prof.values())
    for name, (n_l, ms) in sorted(prof.items(), key=lambda kv: -kv[1][1]):
        k = {"launches": n_l, "ms_total": round(ms, 4), "us_per_launch": round(1e3 * ms / n_l, 2),
             "share": round(ms / max(prof_total, 1e-9), 4)}
        kb = [kernel_bytes(name, w, layer) for layer in w.layers]
        per_call = len(w.layers) * args.steps / n_l     # launches of this kernel per layer call
        if all(b is not None for b in kb) and per_call == 1:
            gbs = sum(kb) * args.steps / (ms / 1e3) / 1e9
            k["hbm_gbs"] = round(gbs, 1)
            k["hbm_frac"] = round(gbs / pk["hbm_gbs"], 4)
        kf = sum(kernel_flops(name, w, layer) for layer in w.layers)
        if kf and per_call == 1:
            tf = kf * args.steps / (ms / 1e3) / 1e12
            k["tensor_tflops"] = round(tf, 1)
            k["tensor_frac"] = round(tf / pk["bf16_tflops_sustained"], 4)
        kernels[name] = k
    if dom is not None:
        name, (n_l, ms) = dom
        per_launch_bytes = sum(kernel_bytes(name, w, layer) or 0 for layer in w.layers) / len(w.layers)
        avg_s = ms / n_l / 1e3
        achieved = per_launch_bytes / avg_s / 1e9
        roof = {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                "traffic": ncu_traffic(name, w.name) if args.layout == "token_major" else None,
                "kernel_source_sha": kernel_source_sha(name),
                "peak_source": pk_src, "avg_launch_us": round(avg_s * 1e6, 2),
                "timing": "CUDA events on the launch stream around each launch (this tracer serialises "
                          "launches, so kernel times sum above the step time, which is taken with it off)",
                "algorithmic_bytes_per_launch": int(per_launch_bytes)}
    step_bytes = sum(layer_bytes(w, layer) for layer in w.layers)
    step_flops = sum(layer_flops(w, layer) for layer in w.layers)
    ms_per_step = total_ms / args.steps
    t_hbm = step_bytes / (pk["hbm_gbs"] * 1e9)
    t_tc = step_flops / (pk["bf16_tflops_sustained"] * 1e12)
    step_roof = {"algorithmic_bytes": int(step_bytes), "tensor_flops": int(step_flops),
                 "achieved_gbs": round(step_bytes / (ms_per_step / 1e3) / 1e9, 1),
                 "roofline_us": round(max(t_hbm, t_tc) * 1e6, 2),
                 "frac_of_roofline": round(max(t_hbm, t_tc) / (ms_per_step / 1e3), 4),
                 "vs_8TBps_frac": round(step_bytes / 8e12 / (ms_per_step / 1e3), 4), "peak_source": pk_src}

    line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "kind": w.kind, "batch": w.batch, "seq_len": w.seqlen,
                       "tokens_per_gpu": w.tokens, "ksize": w.ksize, "rank": w.rank, "head_dim": w.head_dim,
                       "layers": [[l.name, l.d_model, l.channels] for l in w.layers],
                       "varlen": w.varlen, "parallelism": f"replicas{world}",
                       "l2": "flushed between timed steps (256 MiB write, outside the step events)",
                       "algo": {0: "auto", 1: "simt", 2: "tc"}[args.algo], "layout": args.layout,
                       "deterministic": bool(args.deterministic),
                       "rope": ({"channels": W.ROPE_QKV[w.name][0], "head_dim": W.ROPE_QKV[w.name][1],
                                 "layers": ["qkv"]} if args.rope and w.name in W.ROPE_QKV else None),
                       "kernel_family": {"fwd": fam[0], "bwd": fam[1], "note": fam[2]}},
            "roofline": roof, "step_roofline": step_roof, "kernels": kernels,
            "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "steps": e2e_steps},
            "gpu_launches": int(launches), "clocks": clk.summary()}
    return line


def build_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--algo", type=int, default=0, help="0 auto, 1 CUDA-core kernels, 2 tensor-core kernels")
    ap.add_argument("--deterministic", action="store_true",
                    help="bitwise-repeatable backward (no float atomics; the low-rank one runs the CUDA-core kernels)")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="train", choices=["train", "decode"],
                    help="train: forward + backward step (default); decode: one decode step per layer")
    ap.add_argument("--decode-batch", type=int, default=64, help="sequences per decode step")
    ap.add_argument("--rope", action="store_true",
                    help="fuse RoPE (base 10000, interleaved pairs) after the conv of the QKV layer (Q and K)")
    ap.add_argument("--layout", default="token_major", choices=["token_major", "channel_first"],
                    help="memory layout of u, y, g, du: [N, C] or [batch, C, seqlen]")
    return ap


def main():
    args = build_parser().parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from dynamic_short_convolutions_b200 import workloads as W

    w = W.CONFIGS[args.config]
    if args.impl == "reference" and args.mode == "decode":
        if rank != 0:
            return 0
        # the reference arm of the decode mode: the oracle's decode step as it stands
        rates = [oracle_decode_rate(w, args.decode_batch, 1.0) for _ in range(args.warmup + args.steps)]
        rates = rates[args.warmup:]
        value = sum(r for r, _, _ in rates) / len(rates)
        line = {"metric": DECODE_METRIC, "mode": "decode", "value": round(value, 2), "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * args.decode_batch / value, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": w.name, "decode_batch": args.decode_batch},
                "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores_used(), "kind": "oracle",
                                 "sample": rates[0][1]},
                "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    if args.impl == "reference":
        if rank != 0:
            return 0
        # The reference arm is the fp64 oracle as it stands, on this host's cores:
        # each step is a bounded sample of the workload (first T tokens, every layer).
        per_step_budget = min(2.0, 150.0 / max(1, args.steps + args.warmup))
        seqs, T = oracle_sample_shape(w, per_step_budget)
        sample = OracleSample(w, seqs, T)
        for _ in range(args.warmup):
            sample.run()
        secs = [sample.run() for _ in range(args.steps)]
        value = sample.tokens * args.steps / sum(secs)
        line = {"metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * sum(secs) / len(secs), 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": w.name, "sample_tokens_per_step": sample.tokens},
                "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores_used(),
                                 "kind": "oracle",
                                 "sample": f"fp64 oracle fwd+bwd on {seqs} sequence(s) x {T} tokens of "
                                           f"{w.name}, every layer, per step"},
                "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist

    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = (run_decode if args.mode == "decode" else run_ours)(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank == 0 and args.mode == "decode":
        if world == 1 and not args.no_cpu_baseline:
            rate, desc, secs = oracle_decode_rate(w, args.decode_batch, min(args.cpu_budget, 5.0))
            line["cpu_baseline"] = {"value": round(rate, 2), "unit": "tokens/s", "cores": cores_used(),
                                    "kind": "oracle", "sample": f"fp64 oracle: {desc} ({secs:.1f} s)"}
        print(json.dumps(line), flush=True)
        return 0
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            rate, desc, secs = oracle_sample_rate(w, args.cpu_budget)
            line["cpu_baseline"] = {"value": round(rate, 2), "unit": "tokens/s", "cores": cores_used(),
                                    "kind": "oracle",
                                    "sample": f"fp64 oracle fwd+bwd on {desc} of {w.name}, every layer "
                                              f"({secs:.1f} s)"}
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
