"""ctypes wrapper over the fp64 C oracle (``dynconv_oracle.c``).

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the bench).

All arrays are fp64, dense row-major; see the C file's header for the
definitions each function follows ("Dynamic Short Convolutions Improve
Transformers", gist.science technical summary, "Dynamic Short Convolutions":
the Mechanism formula, the Parameterization list and the residual Placement).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

LOWRANK = "lowrank"
HEADWISE = "headwise"

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dynconv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdynconv_oracle.so")
# A prebuilt oracle library to load instead of this directory's build: the mutation
# tests point it at copies of the C file with one planted mistake each.
_LIB_OVERRIDE = os.environ.get("DYNCONV_ORACLE_LIB")
_lock = threading.Lock()
_lib = None


def compile_library(src: str, out: str) -> None:
    """gcc with the oracle's flags: fp64 as written (no fast-math, no FMA contraction), OpenMP."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
                           "-ffp-contract=off", "-fno-fast-math", src, "-o", tmp, "-lm"])
    os.replace(tmp, out)


def build(force: bool = False) -> str:
    """Compile the oracle (when its library is missing or older than the C file)."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_library(_SRC, _LIB_PATH)
    return _LIB_PATH


class _Problem(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int64), ("n_tokens", ctypes.c_int64), ("d_model", ctypes.c_int64),
                ("channels", ctypes.c_int64), ("ksize", ctypes.c_int64), ("rank", ctypes.c_int64),
                ("head_dim", ctypes.c_int64), ("n_segs", ctypes.c_int64),
                ("cu_seqlens", ctypes.POINTER(ctypes.c_int64))]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER(_Problem)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int64)
            lib.orc_forward.argtypes = [P, dp, dp, dp, dp, ctypes.c_int64, ip, dp, dp, dp]
            lib.orc_backward_rows.argtypes = [P, dp, dp, dp, dp, dp, ctypes.c_int64, ip, dp, dp, dp]
            lib.orc_param_grads.argtypes = [P, dp, dp, dp, dp, dp, dp, dp]
            lib.orc_param_grad_entries.argtypes = [P, dp, dp, dp, dp, dp, ctypes.c_int64, ctypes.c_int64,
                                                   ip, ip, dp]
            lib.orc_decode_step.argtypes = [P, dp, dp, dp, dp, dp, dp]
            lib.orc_rope.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_double, ctypes.c_int64,
                                     ctypes.c_int64, ip, dp]
            for f in (lib.orc_forward, lib.orc_backward_rows, lib.orc_param_grads, lib.orc_param_grad_entries,
                      lib.orc_decode_step, lib.orc_rope):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


@dataclasses.dataclass
class Problem:
    """Shapes of one call.  cu_seqlens: document/sequence offsets [S+1] (0 ... N)."""

    kind: str
    n_tokens: int
    d_model: int
    channels: int
    ksize: int
    cu_seqlens: Sequence[int]
    rank: int = 0
    head_dim: int = 0

    def _c(self):
        cu = np.ascontiguousarray(np.asarray(self.cu_seqlens, dtype=np.int64))
        s = _Problem(0 if self.kind == LOWRANK else 1, self.n_tokens, self.d_model, self.channels,
                     self.ksize, self.rank, self.head_dim, len(cu) - 1,
                     cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
        return s, cu

    @property
    def gen_dim(self) -> int:
        return self.rank if self.kind == LOWRANK else (self.channels // self.head_dim) * self.ksize


def _d(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _rows(rows):
    if rows is None:
        return None, None
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def forward(p: Problem, u, h, A, BW, rows=None, want_w: bool = False):
    """Returns (y, z, w) for the listed tokens (all when rows is None).
    z is None for head-wise; w [rows, C*K] only when want_w."""
    lib = _load()
    u, h, A, BW = _f64(u), _f64(h), _f64(A), _f64(BW)
    rr, rp = _rows(rows)
    n = p.n_tokens if rr is None else len(rr)
    y = np.zeros((n, p.channels))
    z = np.zeros((n, p.rank)) if p.kind == LOWRANK else None
    w = np.zeros((n, p.channels * p.ksize)) if want_w else None
    s, cu = p._c()
    rc = lib.orc_forward(ctypes.byref(s), _d(u), _d(h), _d(A) if A is not None else None, _d(BW),
                         n, rp, _d(y), _d(z), _d(w))
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return y, z, w


def filters(p: Problem, u, h, A, BW, rows=None):
    """Generated filters w [rows, C, K]."""
    _, _, w = forward(p, u, h, A, BW, rows=rows, want_w=True)
    return w.reshape(-1, p.channels, p.ksize)


def backward_rows(p: Problem, g, u, h, A, BW, rows=None):
    """Returns (du, dgen, dh) for the listed tokens: dgen = dz [.., r] (low-rank)
    or dwh [.., H*K] (head-wise)."""
    lib = _load()
    g, u, h, A, BW = _f64(g), _f64(u), _f64(h), _f64(A), _f64(BW)
    rr, rp = _rows(rows)
    n = p.n_tokens if rr is None else len(rr)
    du = np.zeros((n, p.channels))
    dg = np.zeros((n, p.gen_dim))
    dh = np.zeros((n, p.d_model))
    s, cu = p._c()
    rc = lib.orc_backward_rows(ctypes.byref(s), _d(g), _d(u), _d(h), _d(A) if A is not None else None,
                               _d(BW), n, rp, _d(du), _d(dg), _d(dh))
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return du, dg, dh


def param_grads(p: Problem, g, u, h, A, BW):
    """Full parameter gradients: (dA, dB) for low-rank, (None, dW) for head-wise."""
    lib = _load()
    g, u, h, A, BW = _f64(g), _f64(u), _f64(h), _f64(A), _f64(BW)
    dA = np.zeros((p.d_model, p.rank)) if p.kind == LOWRANK else None
    dBW = np.zeros_like(BW)
    s, cu = p._c()
    rc = lib.orc_param_grads(ctypes.byref(s), _d(g), _d(u), _d(h), _d(A) if A is not None else None,
                             _d(BW), _d(dA), _d(dBW))
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return dA, dBW


def param_grad_entries(p: Problem, g, u, h, A, BW, which: str, idx0, idx1):
    """Selected entries: which = 'dA' (a, k), 'dB' (k, col) or 'dW' (a, col)."""
    lib = _load()
    g, u, h, A, BW = _f64(g), _f64(u), _f64(h), _f64(A), _f64(BW)
    code = {"dA": 0, "dB": 1, "dW": 2}[which]
    i0 = np.ascontiguousarray(np.asarray(idx0, dtype=np.int64))
    i1 = np.ascontiguousarray(np.asarray(idx1, dtype=np.int64))
    out = np.zeros(len(i0))
    s, cu = p._c()
    ip = ctypes.POINTER(ctypes.c_int64)
    rc = lib.orc_param_grad_entries(ctypes.byref(s), _d(g), _d(u), _d(h), _d(A) if A is not None else None,
                                    _d(BW), code, len(i0), i0.ctypes.data_as(ip), i1.ctypes.data_as(ip), _d(out))
    if rc != 0:
        raise ValueError("oracle rejected the request")
    return out


def decode_step(p: Problem, u, h, A, BW, state):
    """One decode step: p.n_tokens sequences, one new token each (u [B, C], h [B, d]),
    state [B, K-1, C] = the previous K-1 conv inputs (zero before a sequence start).
    Returns (y [B, C], new state); the argument is not modified."""
    lib = _load()
    u, h, A, BW = _f64(u), _f64(h), _f64(A), _f64(BW)
    st = np.array(state, dtype=np.float64, copy=True).reshape(p.n_tokens, max(p.ksize - 1, 0), p.channels)
    st = np.ascontiguousarray(st)
    y = np.zeros((p.n_tokens, p.channels))
    s, cu = p._c()
    rc = lib.orc_decode_step(ctypes.byref(s), _d(u), _d(h), _d(A) if A is not None else None, _d(BW),
                             st.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if st.size else None, _d(y))
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return y, st


def rope(p: Problem, x, n_rot: int, head_dim: int, base: float = 10000.0, inverse: bool = False, rows=None):
    """Rotary position embedding (RoFormer's pairwise rotation) of the listed tokens' rows of x
    [rows, C]: pairs (2i, 2i+1) of each head_dim-channel head among the first n_rot channels
    turn by position * base^(-2i/head_dim); inverse=True applies the adjoint.  Returns a copy."""
    lib = _load()
    x = np.array(x, dtype=np.float64, copy=True, order="C")
    rr, rp = _rows(rows)
    n = p.n_tokens if rr is None else len(rr)
    assert x.shape == (n, p.channels)
    s, cu = p._c()
    rc = lib.orc_rope(ctypes.byref(s), n_rot, head_dim, float(base), int(bool(inverse)), n, rp, _d(x))
    if rc != 0:
        raise ValueError("oracle rejected the rotation")
    return x
