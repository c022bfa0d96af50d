"""Full-size parity: every workload at its benchmark size, in the launch
configuration bench.py times (one plan per layer, algo AUTO, z saved by the
forward and reused by the backward), compared with the fp64 oracle on sampled
outputs it computes one by one: rows of y, z, du and dh at sequence/document
starts and ends, tile boundaries and random tokens, and sampled entries of
dA, dB (or dW)."""
import numpy as np
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from helpers import assert_close, oracle_problem

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

FULL = ["c2_qkv_150m_lowrank", "c3_qkv_2b_headwise_gqa", "c4_all_linear_2b_block", "c5_varlen_packed"]


def _rows(w, cu, rng, n_random=24):
    N = w.tokens
    rows = {0, 1, 2, 3, N - 1, N - 2, 127, 128, 129, 255, 256}
    starts = [int(c) for c in cu[:-1]]
    for s in starts[:6] + starts[-3:]:
        rows.update({s, s + 1, s + 2, s + 3, s - 1, s - 2})
    rows.update(int(x) for x in rng.integers(0, N, n_random))
    return sorted(r for r in rows if 0 <= r < N)


def _run_layer(w, layer, li):
    from dynamic_short_convolutions_b200 import _lib as L, ops

    t = W.make_inputs(w, layer, li, device="cuda")
    kind = L.LOWRANK if w.kind == W.LOWRANK else L.HEADWISE
    batch, seqlen = (1, w.tokens) if w.varlen else (w.batch, w.seqlen)
    plan = ops.DynConvPlan(kind, W.storage_dtype(w), batch, seqlen, layer.d_model, layer.channels, w.ksize, w.rank,
                           w.head_dim, device="cuda")
    A = t.get("A")
    BW = t["B"] if kind == L.LOWRANK else t["W"]
    cu = t["cu_seqlens"] if w.varlen else None
    R = w.rank if kind == L.LOWRANK else (layer.channels // w.head_dim) * w.ksize
    z = torch.empty((w.tokens, R), dtype=W.storage_dtype(w), device="cuda")
    y = plan.forward(t["u"], t["h"], A, BW, cu, z_save=z)
    out = plan.backward(t["g"], t["u"], t["h"], A, BW, cu, z_saved=z)
    assert L.dynconv_device_status(plan.ws) == 0, L.dynconv_last_error()
    torch.cuda.synchronize()
    return t, y, z, out


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    from oracle import oracle as O

    w = W.CONFIGS[name]
    rng = np.random.default_rng(4242)
    for li, layer in enumerate(w.layers):
        t, y, z, out = _run_layer(w, layer, li)
        x = {k: W.to_f64(v) for k, v in t.items() if k != "cu_seqlens"}
        cu = t["cu_seqlens"].cpu().numpy() if w.varlen else np.arange(0, w.tokens + 1, w.seqlen)
        x["cu_seqlens"] = cu
        p = oracle_problem(w, layer, cu)
        A = x.get("A")
        BW = x["B"] if w.kind == W.LOWRANK else x["W"]
        rows = _rows(w, cu, rng)
        yr, zr, _ = O.forward(p, x["u"], x["h"], A, BW, rows=rows)
        dur, _, dhr = O.backward_rows(p, x["g"], x["u"], x["h"], A, BW, rows=rows)
        tag = f"{name}:{layer.name}"
        assert_close(tag + ":y", W.to_f64(y)[rows], yr, w.dtype)
        assert_close(tag + ":du", W.to_f64(out["du"])[rows], dur, w.dtype)
        assert_close(tag + ":dh", W.to_f64(out["dh"])[rows], dhr, w.dtype)
        if zr is not None:
            assert_close(tag + ":z", W.to_f64(z)[rows], zr, w.dtype)
        d, C, K = layer.d_model, layer.channels, w.ksize
        if w.kind == W.LOWRANK:
            r = w.rank
            ka = rng.integers(0, r, 4)
            ia = rng.integers(0, d, 4)
            dA_ref = O.param_grad_entries(p, x["g"], x["u"], x["h"], A, BW, "dA", ia, ka)
            assert_close(tag + ":dA", W.to_f64(out["dA"])[ia, ka], dA_ref, w.dtype)
            kb = rng.integers(0, r, 8)
            cols = np.concatenate([[0, 63 * K + K - 1, 64 * K], rng.integers(0, C * K, 5)])
            dB_ref = O.param_grad_entries(p, x["g"], x["u"], x["h"], A, BW, "dB", kb, cols)
            assert_close(tag + ":dB", W.to_f64(out["dBW"])[kb, cols], dB_ref, w.dtype)
        else:
            G = (C // w.head_dim) * K
            ia = rng.integers(0, d, 8)
            cols = rng.integers(0, G, 8)
            dW_ref = O.param_grad_entries(p, x["g"], x["u"], x["h"], None, BW, "dW", ia, cols)
            assert_close(tag + ":dW", W.to_f64(out["dBW"])[ia, cols], dW_ref, w.dtype)
        del t, x, y, z, out
        torch.cuda.empty_cache()


def test_c2_every_element():
    """The 150M QKV layer at its benchmark size, in the bench's launch configuration,
    compared with the oracle on EVERY element of every output: y, z, du, dh and the
    full parameter gradients dA [768, 32] and dB [32, 6912] -- the cross-CTA
    reductions (bulk-tensor dz add-reduce, per-run dB partials, split-token dA
    partials) included."""
    from oracle import oracle as O

    w = W.CONFIGS["c2_qkv_150m_lowrank"]
    layer = w.layers[0]
    t, y, z, out = _run_layer(w, layer, 0)
    x = {k: W.to_f64(v) for k, v in t.items() if k != "cu_seqlens"}
    cu = np.arange(0, w.tokens + 1, w.seqlen)
    p = oracle_problem(w, layer, cu)
    yr, zr, _ = O.forward(p, x["u"], x["h"], x["A"], x["B"])
    assert_close("c2:y", W.to_f64(y), yr, w.dtype)
    assert_close("c2:z", W.to_f64(z), zr, w.dtype)
    del yr, zr
    dur, _, dhr = O.backward_rows(p, x["g"], x["u"], x["h"], x["A"], x["B"])
    assert_close("c2:du", W.to_f64(out["du"]), dur, w.dtype)
    assert_close("c2:dh", W.to_f64(out["dh"]), dhr, w.dtype)
    del dur, dhr
    dAr, dBr = O.param_grads(p, x["g"], x["u"], x["h"], x["A"], x["B"])
    assert_close("c2:dA", W.to_f64(out["dA"]), dAr, w.dtype)
    assert_close("c2:dB", W.to_f64(out["dBW"]), dBr, w.dtype)
