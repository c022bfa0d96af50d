"""Shared test helpers: run the CUDA path through the C ABI, run the oracle, compare."""
from __future__ import annotations

import numpy as np

from dynamic_short_convolutions_b200 import workloads as W

# Tolerances: fp32 storage rel-L2 <= 1e-5; bf16 storage rel-L2 <= 2e-2 and
# max-abs <= 5e-2, the max-abs read on the scale of the tensor: max|err| /
# max(1, max|ref|) (literal for tensors bounded by 1; relative above that,
# since the bf16 rounding of one stored value of magnitude v is already up to
# 2^-9 v, i.e. above 5e-2 for |v| > 25).
TOL = {"f32": dict(rel_l2=1e-5, max_abs=None), "bf16": dict(rel_l2=2e-2, max_abs=5e-2)}


def rel_l2(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / (den if den > 0 else 1.0))


def scaled_max_abs(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - ref)) / max(1.0, float(np.max(np.abs(ref)))))


def assert_close(name, a, ref, dtype):
    t = TOL[dtype]
    e = rel_l2(a, ref)
    assert e <= t["rel_l2"], f"{name}: rel-L2 {e:.3e} > {t['rel_l2']}"
    if t["max_abs"] is not None:
        m = scaled_max_abs(a, ref)
        assert m <= t["max_abs"], f"{name}: scaled max-abs {m:.3e} > {t['max_abs']}"


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
