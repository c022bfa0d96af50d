"""ctypes binding of the C ABI declared in ``include/dynconv.h``.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libdynconv.so``.  The functions keep the C names and take torch
tensors (or None for nullable pointers); the stream defaults to torch's
current stream on the tensors' device.  If the shared library is missing the
import fails loudly -- there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdynconv.so")

DYNCONV_OK = 0
STATUS_NAMES = {0: "DYNCONV_OK", 1: "DYNCONV_ERR_INVALID", 2: "DYNCONV_ERR_UNSUPPORTED",
                3: "DYNCONV_ERR_WORKSPACE", 4: "DYNCONV_ERR_CUDA", 5: "DYNCONV_ERR_DEVICE_CHECK"}
LOWRANK, HEADWISE = 0, 1
F32, BF16 = 0, 1
ALGO_AUTO, ALGO_SIMT, ALGO_TC = 0, 1, 2
TOKEN_MAJOR, CHANNEL_FIRST = 0, 1

# Every entry point the header declares (checked against the library's exports by the tests).
EXPORTS = ("dynconv_workspace_bytes", "dynconv_fwd", "dynconv_fwd_varlen", "dynconv_bwd",
           "dynconv_device_status", "dynconv_last_error", "dynconv_status_string", "dynconv_version",
           "dynconv_profile_enable", "dynconv_profile_read", "dynconv_selftest_umma", "dynconv_fwd_noalloc",
           "dynconv_decode_step", "dynconv_noalloc_status", "dynconv_query_family", "dynconv_selftest_wait")


class DynConvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class dynconv_profile_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


class dynconv_desc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("dtype", ctypes.c_int32), ("batch", ctypes.c_int64),
                ("seqlen", ctypes.c_int64), ("d_model", ctypes.c_int64), ("channels", ctypes.c_int64),
                ("ksize", ctypes.c_int64), ("rank", ctypes.c_int64), ("head_dim", ctypes.c_int64),
                ("u_row_stride", ctypes.c_int64), ("h_row_stride", ctypes.c_int64),
                ("deterministic", ctypes.c_int32), ("algo", ctypes.c_int32), ("layout", ctypes.c_int32),
                ("rope_channels", ctypes.c_int64), ("rope_head_dim", ctypes.c_int64), ("rope_max_pos", ctypes.c_int64),
                ("rope_cos_sin", ctypes.c_void_p)]


_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libdynconv.so (built by ``python -m dynamic_short_convolutions_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m dynamic_short_convolutions_b200.build` "
                           "(there is no CPU or Python fallback)")
    lib = ctypes.CDLL(p)
    vp, sz, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64
    D = ctypes.POINTER(dynconv_desc)
    lib.dynconv_workspace_bytes.argtypes = [D]
    lib.dynconv_workspace_bytes.restype = sz
    lib.dynconv_fwd.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dynconv_fwd_varlen.argtypes = [D, vp, i64, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dynconv_bwd.argtypes = [D, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dynconv_device_status.argtypes = [vp, sz, vp]
    lib.dynconv_fwd_noalloc.argtypes = [D, vp, vp, vp, vp, vp, vp, vp]
    lib.dynconv_fwd_noalloc.restype = ctypes.c_int
    lib.dynconv_query_family.argtypes = [D, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
    lib.dynconv_query_family.restype = ctypes.c_int
    lib.dynconv_noalloc_status.argtypes = [vp]
    lib.dynconv_noalloc_status.restype = ctypes.c_int
    lib.dynconv_decode_step.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    for f in (lib.dynconv_fwd, lib.dynconv_fwd_varlen, lib.dynconv_bwd, lib.dynconv_device_status,
              lib.dynconv_decode_step):
        f.restype = ctypes.c_int
    lib.dynconv_last_error.restype = ctypes.c_char_p
    lib.dynconv_status_string.argtypes = [ctypes.c_int]
    lib.dynconv_status_string.restype = ctypes.c_char_p
    lib.dynconv_version.restype = ctypes.c_int
    lib.dynconv_profile_enable.argtypes = [ctypes.c_int]
    lib.dynconv_profile_enable.restype = ctypes.c_int
    lib.dynconv_profile_read.argtypes = [ctypes.POINTER(dynconv_profile_entry), ctypes.c_int, ctypes.c_int]
    lib.dynconv_profile_read.restype = ctypes.c_int
    lib.dynconv_selftest_umma.argtypes = [ctypes.c_int, vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp]
    lib.dynconv_selftest_umma.restype = ctypes.c_int
    lib.dynconv_selftest_wait.argtypes = [ctypes.c_uint64, vp, vp, vp]
    lib.dynconv_selftest_wait.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, ref: torch.Tensor):
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    dev = ref.device if ref is not None and ref.device.type == "cuda" else None
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check(status: int):
    if status != DYNCONV_OK:
        msg = load().dynconv_last_error().decode(errors="replace")
        raise DynConvError(status, msg)


def make_desc(kind: int, dtype: int, batch: int, seqlen: int, d_model: int, channels: int, ksize: int,
              rank: int = 0, head_dim: int = 0, u_row_stride: int = 0, h_row_stride: int = 0,
              deterministic: int = 0, algo: int = ALGO_AUTO, layout: int = TOKEN_MAJOR, rope_channels: int = 0,
              rope_head_dim: int = 0, rope_table: Optional[torch.Tensor] = None) -> dynconv_desc:
    """rope_table: device fp32 [max_pos, rope_head_dim] (cos, sin pairs), kept alive by the caller."""
    rope_max = int(rope_table.shape[0]) if rope_table is not None else 0
    rope_ptr = ctypes.c_void_p(rope_table.data_ptr()) if rope_table is not None else None
    return dynconv_desc(kind, dtype, batch, seqlen, d_model, channels, ksize, rank, head_dim, u_row_stride,
                        h_row_stride, deterministic, algo, layout, rope_channels, rope_head_dim, rope_max, rope_ptr)


def dynconv_workspace_bytes(desc: dynconv_desc) -> int:
    return int(load().dynconv_workspace_bytes(ctypes.byref(desc)))


def dynconv_fwd(desc, u, h, A, B_or_W, y, z_save, ws, stream=None):
    _check(load().dynconv_fwd(ctypes.byref(desc), _ptr(u), _ptr(h), _ptr(A), _ptr(B_or_W), _ptr(y),
                              _ptr(z_save), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream, u)))


def dynconv_fwd_varlen(desc, cu_seqlens, u, h, A, B_or_W, y, z_save, ws, stream=None):
    _check(load().dynconv_fwd_varlen(ctypes.byref(desc), _ptr(cu_seqlens), cu_seqlens.numel() - 1, _ptr(u),
                                     _ptr(h), _ptr(A), _ptr(B_or_W), _ptr(y), _ptr(z_save), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream, u)))


def dynconv_bwd(desc, cu_seqlens, g, u, h, A, B_or_W, z_saved, du, dh, dA, dB_or_dW, ws, stream=None):
    n_docs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(load().dynconv_bwd(ctypes.byref(desc), _ptr(cu_seqlens), n_docs, _ptr(g), _ptr(u), _ptr(h), _ptr(A),
                              _ptr(B_or_W), _ptr(z_saved), _ptr(du), _ptr(dh), _ptr(dA), _ptr(dB_or_dW),
                              _ptr(ws), ws.numel() * ws.element_size(), _stream(stream, g)))


def dynconv_fwd_noalloc(desc, u, h, A, B, y, z_save=None, stream=None):
    """Forward with no workspace argument (scratch built into the library); see include/dynconv.h."""
    _check(load().dynconv_fwd_noalloc(ctypes.byref(desc), _ptr(u), _ptr(h), _ptr(A), _ptr(B), _ptr(y), _ptr(z_save),
                                      _stream(stream, u)))


def dynconv_noalloc_status(stream=None) -> int:
    """Synchronises the stream; returns the status of the no-workspace forward calls (does not raise)."""
    st = ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)) \
        if stream is not None else ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return int(load().dynconv_noalloc_status(st))


def dynconv_decode_step(desc, u, h, A, B_or_W, state, y, ws, stream=None):
    _check(load().dynconv_decode_step(ctypes.byref(desc), _ptr(u), _ptr(h), _ptr(A), _ptr(B_or_W), _ptr(state),
                                      _ptr(y), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream, u)))


def dynconv_device_status(ws, stream=None) -> int:
    """Synchronises the stream; returns the status (does not raise)."""
    return int(load().dynconv_device_status(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream, ws)))


FAMILY_TENSOR_CORE, FAMILY_CUDA_CORE = 1, 2
FAMILY_NAMES = {FAMILY_TENSOR_CORE: "tensor_core", FAMILY_CUDA_CORE: "cuda_core"}


def dynconv_query_family(desc):
    """(forward family, backward family, reason) for a descriptor; host-only."""
    f, b = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(load().dynconv_query_family(ctypes.byref(desc), ctypes.byref(f), ctypes.byref(b)))
    return FAMILY_NAMES[f.value], FAMILY_NAMES[b.value], dynconv_last_error()


def dynconv_last_error() -> str:
    return load().dynconv_last_error().decode(errors="replace")


def dynconv_version() -> int:
    return int(load().dynconv_version())


def dynconv_profile_enable(enable: bool) -> bool:
    return bool(load().dynconv_profile_enable(int(bool(enable))))


def dynconv_profile_read(reset: bool = True):
    """{kernel name: (launches, total device ms)} since the last reset (waits for the events)."""
    lib = load()
    arr = (dynconv_profile_entry * 64)()
    n = lib.dynconv_profile_read(arr, 64, int(bool(reset)))
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(min(n, 64))}


def dynconv_selftest_wait(limit_ns: int, err_word, out2, stream=None) -> int:
    """Diagnostic bounded wait that runs out (see include/dynconv_diag.h); returns the status."""
    return int(load().dynconv_selftest_wait(int(limit_ns), _ptr(err_word), _ptr(out2), _stream(stream, err_word)))


def dynconv_selftest_umma(variant: int, A, B, D, N: int, Kd: int, err_word, stream=None) -> int:
    """Diagnostic tile D = A B^T through TMA + tcgen05 (see include/dynconv_diag.h); returns the status."""
    return int(load().dynconv_selftest_umma(variant, _ptr(A), _ptr(B), _ptr(D), N, Kd, _ptr(err_word),
                                            _stream(stream, A)))
