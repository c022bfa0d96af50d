"""Shared test helpers: run the CUDA path through the C ABI, run the oracle, compare."""
from __future__ import annotations

import numpy as np

from dynamic_short_convolutions_b200 import workloads as W

# Tolerances (the fp32 and bf16 bounds the hot path is held to):
#   fp32 storage: rel-L2 <= 1e-5.
#   bf16 storage, per-token outputs (y, du, dh, z): rel-L2 <= 2e-2 and, element
#     by element, |a - ref| <= 5e-2 + 2^-8 |ref|.  The second term is the
#     output's own rounding: storing a value of magnitude v in bf16 moves it by
#     up to 2^-9 v (half a unit in the last place), and 2^-8 v leaves room for
#     the rounding of the bf16 operands it was computed from; it only matters
#     for elements above ~6, whose stored value alone cannot be held to 5e-2.
#   bf16 storage, parameter gradients (dA, dB, dW; fp32 outputs): rel-L2 <=
#     2e-2 and max|a - ref| <= 5e-2 * max(1, max|ref|).  Each entry is a sum
#     over every token of products of bf16-rounded operands, so its rounding
#     error grows with the sum's size, not with the entry's own value: the
#     bound is read on the scale of the tensor.
TOL = {"f32": dict(rel_l2=1e-5, max_abs=None), "bf16": dict(rel_l2=2e-2, max_abs=5e-2)}
ELEM_REL = 2.0 ** -8
PARAM_GRADS = ("dA", "dB", "dW", "dBW")


def rel_l2(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / (den if den > 0 else 1.0))


def max_abs(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(a - ref))) if a.size else 0.0


def scaled_max_abs(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - ref)) / max(1.0, float(np.max(np.abs(ref)))))


def elem_excess(a, ref, bound):
    """max over elements of |a - ref| - (bound + 2^-8 |ref|) (<= 0 when every element passes)."""
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    if a.size == 0:
        return -bound
    return float(np.max(np.abs(a - ref) - (bound + ELEM_REL * np.abs(ref))))


def is_param_grad(name):
    return name.rsplit(":", 1)[-1] in PARAM_GRADS


def check_close(name, a, ref, dtype):
    """(ok, message) of the comparison; the message gives the observed figures."""
    t = TOL[dtype]
    e = rel_l2(a, ref)
    msg = f"{name}: rel-L2 {e:.3e} (<= {t['rel_l2']})"
    ok = e <= t["rel_l2"]
    if t["max_abs"] is not None:
        m = max_abs(a, ref)
        if is_param_grad(name):
            sm = scaled_max_abs(a, ref)
            msg += f", max-abs {m:.3e}, scaled max-abs {sm:.3e} (<= {t['max_abs']})"
            ok = ok and sm <= t["max_abs"]
        else:
            x = elem_excess(a, ref, t["max_abs"])
            msg += f", max-abs {m:.3e}, worst element over 5e-2 + 2^-8|ref| by {x:.3e} (<= 0)"
            ok = ok and x <= 0.0
    return ok, msg


def assert_close(name, a, ref, dtype):
    ok, msg = check_close(name, a, ref, dtype)
    assert ok, msg
    return msg


def oracle_problem(w: W.Workload, layer: W.Layer, cu):
    from oracle import oracle as O

    return O.Problem(O.LOWRANK if w.kind == W.LOWRANK else O.HEADWISE, w.tokens, layer.d_model, layer.channels,
                     w.ksize, [int(x) for x in cu], rank=w.rank, head_dim=w.head_dim)


def oracle_all(w, layer, x):
    """Full oracle forward + backward on fp64 host inputs x (dict)."""
    from oracle import oracle as O

    p = oracle_problem(w, layer, x["cu_seqlens"])
    A = x.get("A")
    BW = x["B"] if w.kind == W.LOWRANK else x["W"]
    y, z, _ = O.forward(p, x["u"], x["h"], A, BW)
    du, dgen, dh = O.backward_rows(p, x["g"], x["u"], x["h"], A, BW)
    dA, dBW = O.param_grads(p, x["g"], x["u"], x["h"], A, BW)
    return dict(y=y, z=z, du=du, dh=dh, dA=dA, dBW=dBW)


def gpu_run(w, layer, t, algo=0, varlen=None, z_roundtrip=True, want_dh=True, deterministic=False):
    """Forward + backward through the C ABI on torch tensors t (device, storage dtype)."""
    import torch

    from dynamic_short_convolutions_b200 import ops, _lib as L

    N, C, d = w.tokens, layer.channels, layer.d_model
    varlen = w.varlen if varlen is None else varlen
    kind = L.LOWRANK if w.kind == W.LOWRANK else L.HEADWISE
    batch, seqlen = (1, N) if varlen else (w.batch, w.seqlen)
    plan = ops.DynConvPlan(kind, W.storage_dtype(w), batch, seqlen, d, C, w.ksize, w.rank, w.head_dim,
                           t["u"].stride(0), t["h"].stride(0), deterministic=deterministic, algo=algo,
                           device=t["u"].device)
    A = t.get("A")
    BW = t["B"] if w.kind == W.LOWRANK else t["W"]
    cu = t["cu_seqlens"] if varlen else None
    R = w.rank if kind == L.LOWRANK else (C // w.head_dim) * w.ksize
    z = torch.empty((N, R), dtype=W.storage_dtype(w), device=t["u"].device) if z_roundtrip else None
    y = plan.forward(t["u"], t["h"], A, BW, cu, z_save=z)
    out = plan.backward(t["g"], t["u"], t["h"], A, BW, cu, z_saved=z, want_dh=want_dh)
    st = L.dynconv_device_status(plan.ws)
    assert st == 0, L.dynconv_last_error()
    torch.cuda.synchronize()
    res = dict(y=y, z=z if kind == L.LOWRANK else None, du=out["du"], dh=out["dh"], dA=out["dA"], dBW=out["dBW"])
    return {k: (W.to_f64(v) if v is not None else None) for k, v in res.items()}
