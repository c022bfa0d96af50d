"""Torch-facing helpers over the C ABI: output and workspace allocation, and an
autograd Function.  Marshalling only; the arithmetic runs in libdynconv.so.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib as L


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return L.BF16
    if t.dtype == torch.float32:
        return L.F32
    raise TypeError(f"storage dtype must be bf16 or fp32, got {t.dtype}")


def rope_table(max_pos: int, head_dim: int, base: float = 10000.0, device=None) -> torch.Tensor:
    """The RoPE table the C ABI reads: fp32 [max_pos, head_dim] with entries 2i, 2i+1 of row p
    the cosine and sine of p * base^(-2i/head_dim) (RoFormer's angles), computed once in fp64."""
    p = torch.arange(max_pos, dtype=torch.float64).unsqueeze(1)
    theta = base ** (-torch.arange(0, head_dim, 2, dtype=torch.float64) / head_dim)
    ang = p * theta
    return torch.stack((ang.cos(), ang.sin()), dim=-1).reshape(max_pos, head_dim).float().to(device or "cuda")


class DynConvPlan:
    """Descriptor + workspace for one problem shape.

    Token-major (default): u [N, C] (rows may be strided, channels contiguous),
    y, g, du [N, C].  Channel-first (``layout=L.CHANNEL_FIRST``): u, y, g, du
    [batch, C, seqlen] (u's channel rows ``u_row_stride`` apart, 0 = seqlen).
    h is [N, d] in both.  For packed documents pass ``cu_seqlens`` (int32 device
    tensor [docs+1]) and batch = 1, seqlen = N.
    """

    def __init__(self, kind: int, dtype: torch.dtype, batch: int, seqlen: int, d_model: int, channels: int,
                 ksize: int, rank: int = 0, head_dim: int = 0, u_row_stride: int = 0, h_row_stride: int = 0,
                 deterministic: bool = False, algo: int = L.ALGO_AUTO, device=None, layout: int = L.TOKEN_MAJOR,
                 rope_channels: int = 0, rope_head_dim: int = 0, rope_table: Optional[torch.Tensor] = None):
        self.rope_table = rope_table            # kept alive: the descriptor holds its address
        self.desc = L.make_desc(kind, L.BF16 if dtype == torch.bfloat16 else L.F32, batch, seqlen, d_model,
                                channels, ksize, rank, head_dim, u_row_stride, h_row_stride, int(deterministic),
                                algo, layout, rope_channels, rope_head_dim, rope_table)
        nbytes = L.dynconv_workspace_bytes(self.desc)
        if nbytes == 0:
            raise L.DynConvError(1, "invalid descriptor")
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")
        self.kind, self.dtype, self.layout = kind, dtype, layout
        self.N, self.d, self.C, self.K, self.r = batch * seqlen, d_model, channels, ksize, rank
        self.batch, self.seqlen = batch, seqlen

    def _conv_shape(self):
        return (self.batch, self.C, self.seqlen) if self.layout == L.CHANNEL_FIRST else (self.N, self.C)

    def forward(self, u, h, A, B_or_W, cu_seqlens=None, y=None, z_save=None, stream=None):
        if y is None:
            y = torch.empty(self._conv_shape(), dtype=self.dtype, device=u.device)
        if cu_seqlens is None:
            L.dynconv_fwd(self.desc, u, h, A, B_or_W, y, z_save, self.ws, stream)
        else:
            L.dynconv_fwd_varlen(self.desc, cu_seqlens, u, h, A, B_or_W, y, z_save, self.ws, stream)
        return y

    def backward(self, g, u, h, A, B_or_W, cu_seqlens=None, z_saved=None, want_dh=True, out=None, stream=None):
        dev = g.device
        if out is None:
            out = {"du": torch.empty(self._conv_shape(), dtype=self.dtype, device=dev),
                   "dh": torch.empty((self.N, self.d), dtype=self.dtype, device=dev) if want_dh else None,
                   "dA": torch.empty(tuple(A.shape), dtype=torch.float32, device=dev) if A is not None else None,
                   "dBW": torch.empty(tuple(B_or_W.shape), dtype=torch.float32, device=dev)}
        L.dynconv_bwd(self.desc, cu_seqlens, g, u, h, A, B_or_W, z_saved, out["du"], out["dh"], out["dA"],
                      out["dBW"], self.ws, stream)
        return out


class DynConvDecoder:
    """Decode steps for `batch` sequences (one new token each per step) with the K-1
    previous conv inputs of every sequence kept on the device (``self.state``,
    ``[batch, K-1, C]``, zero = sequence start; call :meth:`reset` to start over)."""

    def __init__(self, kind: int, dtype: torch.dtype, batch: int, d_model: int, channels: int, ksize: int,
                 rank: int = 0, head_dim: int = 0, u_row_stride: int = 0, h_row_stride: int = 0, device=None):
        self.desc = L.make_desc(kind, L.BF16 if dtype == torch.bfloat16 else L.F32, batch, 1, d_model, channels,
                                ksize, rank, head_dim, u_row_stride, h_row_stride, 0, L.ALGO_AUTO)
        nbytes = L.dynconv_workspace_bytes(self.desc)
        if nbytes == 0:
            raise L.DynConvError(1, "invalid descriptor")
        dev = device or "cuda"
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self.state = torch.zeros((batch, ksize - 1, channels), dtype=dtype, device=dev) if ksize > 1 else None
        self.dtype, self.batch, self.C = dtype, batch, channels

    def reset(self):
        if self.state is not None:
            self.state.zero_()

    def step(self, u, h, A, B_or_W, y=None, stream=None):
        if y is None:
            y = torch.empty((self.batch, self.C), dtype=self.dtype, device=u.device)
        L.dynconv_decode_step(self.desc, u, h, A, B_or_W, self.state, y, self.ws, stream)
        return y


class DynamicShortConv(torch.autograd.Function):
    """y = u + dynamic causal depthwise conv(u) with filters generated from h.

    Low-rank: pass A [d, r] and B [r, C*K].  Head-wise: A = None and B_or_W = W
    [d, (C/head_dim)*K].  Parameter gradients come back in the parameters'
    dtype (accumulated in fp32 by the kernels)."""

    @staticmethod
    def forward(ctx, u, h, A, B_or_W, ksize: int, head_dim: int, batch: int, cu_seqlens, algo: int):
        d = h.shape[1]
        kind = L.LOWRANK if A is not None else L.HEADWISE
        rank = A.shape[1] if A is not None else 0
        if u.dim() == 3:        # channel-first [batch, C, seqlen]
            batch, C, seqlen = u.shape
            if u.stride(2) != 1 or u.stride(0) != C * u.stride(1):
                u = u.contiguous()
            N, layout, us = batch * seqlen, L.CHANNEL_FIRST, u.stride(1)
        else:
            N, C = u.shape
            seqlen, layout, us = N // batch, L.TOKEN_MAJOR, u.stride(0)
        plan = DynConvPlan(kind, u.dtype, batch, seqlen, d, C, ksize, rank, head_dim, us, h.stride(0),
                           algo=algo, device=u.device, layout=layout)
        R = rank if A is not None else (C // head_dim) * ksize
        z = torch.empty((N, R), dtype=u.dtype, device=u.device)    # generator output, reused by backward
        y = plan.forward(u, h, A, B_or_W, cu_seqlens, z_save=z)
        ctx.plan = plan
        ctx.save_for_backward(u, h, A, B_or_W, cu_seqlens, z)
        return y

    @staticmethod
    def backward(ctx, gy):
        u, h, A, B_or_W, cu_seqlens, z = ctx.saved_tensors
        out = ctx.plan.backward(gy.contiguous(), u, h, A, B_or_W, cu_seqlens, z_saved=z)
        dA = out["dA"].to(A.dtype) if A is not None else None
        return out["du"], out["dh"], dA, out["dBW"].to(B_or_W.dtype), None, None, None, None, None


def dynamic_short_conv(u: torch.Tensor, h: torch.Tensor, A: Optional[torch.Tensor], B_or_W: torch.Tensor,
                       ksize: int, head_dim: int = 0, batch: int = 1,
                       cu_seqlens: Optional[torch.Tensor] = None, algo: int = L.ALGO_AUTO) -> torch.Tensor:
    """Functional form with autograd: u [N, C] token-major (N = batch * seqlen) or
    [batch, C, seqlen] channel-first; h [N, d]."""
    return DynamicShortConv.apply(u, h, A, B_or_W, ksize, head_dim, batch, cu_seqlens, algo)
