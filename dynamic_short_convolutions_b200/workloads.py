"""Seeded synthetic workloads for the dynamic short convolution hot path.

This module only draws numbers and describes shapes; it holds none of the
method's arithmetic.  It is the single source of inputs shared by the fp64
oracle, the CUDA path, the tests and the benchmark.

Generator definition (one counter-based stream per tensor):

* ``splitmix64`` (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014) applied to the counter ``key + (i + 1) * GOLDEN``
  gives 64 random bits for draw ``i``.  ``key`` is derived from the workload
  seed and a per-tensor tag.
* Two uniforms ``u1 = (a >> 11 + 1) / 2**53`` (in (0, 1]) and
  ``u2 = (b >> 11) / 2**53`` feed the Box-Muller transform
  ``sqrt(-2 ln u1) * cos(2 pi u2)``, giving N(0, 1) in fp64.
* The draw is scaled by the tensor's standard deviation, then rounded once to
  the storage dtype: fp64 -> fp32 (round to nearest even) -> bf16 (round to
  nearest even) for bf16 workloads, fp64 -> fp32 for fp32 workloads.  The
  oracle receives exactly these rounded values, widened back to fp64.

Workload shapes follow the five configurations of the dynamic short
convolution benchmark (dynamic filters on Q/K/V at 150M scale, head-wise on
2B-scale GQA, after every linear of a 2B block, packed variable-length
documents), see "Dynamic Short Convolutions Improve Transformers", gist.science
technical summary, sections "Placement" and "Language Modeling".
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

LOWRANK = "lowrank"
HEADWISE = "headwise"


def _mix(x: np.ndarray) -> np.ndarray:
    """splitmix64 output function on a uint64 array (wrapping arithmetic)."""
    with np.errstate(over="ignore"):
        z = x.copy()
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _key(seed: int, tag: str) -> np.uint64:
    """Stream key for one tensor: splitmix64 of the seed folded with the tag bytes."""
    k = np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    for ch in tag.encode():
        with np.errstate(over="ignore"):
            k = _mix(k ^ np.uint64(ch)) + GOLDEN
    return k[0]


def raw_bits(seed: int, tag: str, count: int, offset: int = 0) -> np.ndarray:
    """``count`` 64-bit draws of the stream (seed, tag), starting at draw ``offset``."""
    i = np.arange(offset, offset + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        ctr = _key(seed, tag) + (i + np.uint64(1)) * GOLDEN
    return _mix(ctr)


def uniform(seed: int, tag: str, count: int) -> np.ndarray:
    """Uniform fp64 draws in (0, 1]."""
    b = raw_bits(seed, tag, count)
    return ((b >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def normal(seed: int, tag: str, count: int, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) fp64 draws by Box-Muller on two interleaved uniform streams."""
    b = raw_bits(seed, tag, 2 * count)
    u1 = ((b[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (b[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return std * np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage dtype and return them widened to fp64."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.float32)
    if dtype == "bf16":
        t = t.to(torch.bfloat16).to(torch.float32)
    elif dtype != "f32":
        raise ValueError(f"unknown storage dtype {dtype!r}")
    return t.to(torch.float64).numpy()


def geometric_doc_lengths(seed: int, total: int, mean: float, lo: int, hi: int) -> List[int]:
    """Packed-document lengths: Geometric(p = 1/mean) on {1, 2, ...} by inverse CDF,
    clipped to [lo, hi], appended while the running sum is below ``total``; the
    last document takes the remainder, and a remainder below ``lo`` is merged
    into the previous document."""
    p = 1.0 / mean
    lengths: List[int] = []
    s = 0
    us = uniform(seed, "doclen", total // max(lo, 1) + 2)
    draw = 0
    while s < total:
        u = us[draw]
        draw += 1
        L = int(math.ceil(math.log(u) / math.log1p(-p))) if u < 1.0 else 1
        L = max(lo, min(hi, max(L, 1)))
        if s + L >= total:
            rem = total - s
            if rem < lo and lengths:
                lengths[-1] += rem
            else:
                lengths.append(rem)
            s = total
        else:
            lengths.append(L)
            s += L
    return lengths


@dataclasses.dataclass(frozen=True)
class Layer:
    """One dynamic short convolution call: C channels filtered from a d-wide hidden state."""

    name: str
    d_model: int
    channels: int


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                    # LOWRANK or HEADWISE
    dtype: str                   # "f32" or "bf16" (storage; accumulation is fp32)
    batch: int
    seqlen: int
    ksize: int
    rank: int                    # low-rank r (0 for head-wise)
    head_dim: int                # head-wise channels per head (0 for low-rank)
    layers: tuple                # tuple[Layer, ...]
    seed: int
    a_std: Optional[float] = None  # None: 1/sqrt(d)
    b_std: Optional[float] = None  # None: 1/sqrt(r)
    varlen: bool = False
    doc_mean: float = 2048.0
    doc_lo: int = 16
    doc_hi: int = 16384

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


def _cfg() -> Dict[str, Workload]:
    return {
        "c1_fp32_lowrank": Workload(
            "c1_fp32_lowrank", LOWRANK, "f32", 2, 128, 3, 4, 0,
            (Layer("conv", 64, 64),), seed=0, a_std=1.0 / 8.0, b_std=0.5),
        "c2_qkv_150m_lowrank": Workload(
            "c2_qkv_150m_lowrank", LOWRANK, "bf16", 8, 2048, 3, 32, 0,
            (Layer("qkv", 768, 2304),), seed=1),
        "c3_qkv_2b_headwise_gqa": Workload(
            "c3_qkv_2b_headwise_gqa", HEADWISE, "bf16", 4, 4096, 4, 0, 128,
            (Layer("qkv", 2048, 3072),), seed=2),
        "c4_all_linear_2b_block": Workload(
            "c4_all_linear_2b_block", LOWRANK, "bf16", 4, 4096, 3, 64, 0,
            (Layer("qkv", 2048, 3072), Layer("o", 2048, 2048),
             Layer("gate_up", 2048, 11264), Layer("down", 5632, 2048)), seed=3),
        "c5_varlen_packed": Workload(
            "c5_varlen_packed", LOWRANK, "bf16", 1, 65536, 4, 64, 0,
            (Layer("conv", 4096, 4096),), seed=4, varlen=True),
    }


CONFIGS: Dict[str, Workload] = _cfg()

# RoPE fused after the conv of the QKV placement: (rotated channels = Q and K, rotary head dim).
# 150M: 12 heads of 64 for each of Q, K, V; 2B GQA: Q 16 heads, K 4 and V 4 heads of 128.
ROPE_QKV = {"c2_qkv_150m_lowrank": (1536, 64), "c3_qkv_2b_headwise_gqa": (2560, 128),
            "c4_all_linear_2b_block": (2560, 128)}
CONFIG_ORDER = list(CONFIGS)


def scaled(w: Workload, batch: int, seqlen: int, layers=None, name=None) -> Workload:
    """The same workload recipe at a smaller token count (and optionally other layers)."""
    return dataclasses.replace(w, batch=batch, seqlen=seqlen,
                               layers=tuple(layers) if layers is not None else w.layers,
                               name=name or f"{w.name}_B{batch}T{seqlen}")


def cu_seqlens_for(w: Workload) -> np.ndarray:
    """int32 document offsets [n_docs + 1]: uniform sequences for dense batches,
    Geometric document lengths for packed workloads."""
    if w.varlen:
        lens = geometric_doc_lengths(w.seed, w.tokens, w.doc_mean, w.doc_lo, w.doc_hi)
    else:
        lens = [w.seqlen] * w.batch
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def _mix_t(x):
    """splitmix64 output function on an int64 torch tensor (two's-complement
    wrapping; logical right shifts by masking), bit-identical to ``_mix``."""
    M1 = int(_M1) - (1 << 64)
    M2 = int(_M2) - (1 << 64)
    x = x ^ ((x >> 30) & ((1 << 34) - 1))
    x = x * M1
    x = x ^ ((x >> 27) & ((1 << 37) - 1))
    x = x * M2
    return x ^ ((x >> 31) & ((1 << 33) - 1))


def normal_torch(seed: int, tag: str, count: int, std: float = 1.0, device="cpu", chunk: int = 1 << 24):
    """The same recipe as ``normal`` evaluated with torch ops on ``device`` (fp64).
    The bits are identical to ``normal``; the fp64 log/cos may differ from
    numpy's in the last ulp, which the storage rounding almost always absorbs.
    Each test or benchmark uses one realisation for both sides of a comparison."""
    import torch

    key = int(_key(seed, tag))
    key = key - (1 << 64) if key >= (1 << 63) else key
    G = int(GOLDEN) - (1 << 64)
    out = torch.empty(count, dtype=torch.float64, device=device)
    for a in range(0, count, chunk):
        b = min(count, a + chunk)
        i = torch.arange(2 * a, 2 * b, dtype=torch.int64, device=device)
        bits = _mix_t(key + (i + 1) * G)
        m53 = (1 << 53) - 1
        u1 = (((bits[0::2] >> 11) & m53).to(torch.float64) + 1.0) * (2.0 ** -53)
        u2 = ((bits[1::2] >> 11) & m53).to(torch.float64) * (2.0 ** -53)
        out[a:b] = std * torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)
    return out


def storage_dtype(w: "Workload"):
    import torch

    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def make_inputs(w: Workload, layer: Layer, layer_index: int = 0, device=None) -> Dict[str, object]:
    """Seeded inputs for one layer call.

    device None: fp64 numpy arrays holding values already rounded to the
    storage dtype (small problems, CPU-only tests).  device given: torch
    tensors in the storage dtype on that device (same recipe, drawn there).

    Keys: u [N,C], h [N,d], g [N,C] (upstream gradient), and A [d,r] + B [r,C*K]
    (low-rank) or W [d,(C/head_dim)*K] (head-wise), cu_seqlens int32 [docs+1].
    """
    N, d, C, K = w.tokens, layer.d_model, layer.channels, w.ksize
    s = w.seed * 1000 + layer_index
    shapes = {"u": ((N, C), 1.0), "h": ((N, d), 1.0), "g": ((N, C), 1.0)}
    if w.kind == LOWRANK:
        r = w.rank
        a_std = w.a_std if w.a_std is not None else 1.0 / math.sqrt(d)
        b_std = w.b_std if w.b_std is not None else 1.0 / math.sqrt(r)
        shapes["A"] = ((d, r), a_std)
        shapes["B"] = ((r, C * K), b_std)
    else:
        H = C // w.head_dim
        shapes["W"] = ((d, H * K), 1.0 / math.sqrt(d))
    out: Dict[str, object] = {}
    for name, (shape, std) in shapes.items():
        cnt = int(np.prod(shape))
        if device is None:
            out[name] = round_to_storage(normal(s, name, cnt, std).reshape(shape), w.dtype)
        else:
            out[name] = normal_torch(s, name, cnt, std, device=device).to(
                __import__("torch").float32).to(storage_dtype(w)).reshape(shape)
    cu = cu_seqlens_for(w)
    if device is None:
        out["cu_seqlens"] = cu
    else:
        import torch
        out["cu_seqlens"] = torch.from_numpy(cu).to(device)
    return out


def to_f64(x) -> np.ndarray:
    """Host fp64 copy of a torch tensor or numpy array (for the oracle)."""
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float64)
    import torch

    return x.detach().to("cpu", torch.float64).contiguous().numpy()
