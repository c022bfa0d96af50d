"""GPU parity of the channel-first layout: u, y, g and du as [batch, C, seqlen]
(tokens contiguous; [C, N] for packed documents), the layout of the depthwise
convs in linear-RNN blocks.  The seeded problems of the token-major tests are
transposed on the host, every output is transposed back and compared with the
fp64 oracle element by element, and the forward is compared bitwise with the
token-major forward (both layouts run the same arithmetic in the same order)."""
import dataclasses

import numpy as np
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from helpers import assert_close, oracle_all, oracle_problem

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

C = W.CONFIGS


def _case(base, batch, seqlen, name, **kw):
    w = W.scaled(C[base], batch, seqlen, name=name)
    return dataclasses.replace(w, **kw) if kw else w


CASES = [
    # seqlen a multiple of 8 with a ragged last 128-token tile: the tiled kernels
    (_case("c2_qkv_150m_lowrank", 2, 296, "cf_c2"), 0, None),
    (_case("c2_qkv_150m_lowrank", 1, 264, "cf_k4_r64", ksize=4, rank=64), 0, None),
    (_case("c2_qkv_150m_lowrank", 2, 136, "cf_k1_r16", ksize=1, rank=16), 0, None),
    (_case("c2_qkv_150m_lowrank", 1, 200, "cf_k2_r64", ksize=2, rank=64), 0, None),
    (_case("c3_qkv_2b_headwise_gqa", 2, 296, "cf_c3"), 0, None),
    (_case("c3_qkv_2b_headwise_gqa", 1, 152, "cf_hw_k2_hd64", ksize=2, head_dim=64,
           layers=(W.Layer("qkv", 256, 640),)), 0, None),
    (_case("c3_qkv_2b_headwise_gqa", 1, 520, "cf_hw_k3_hd32", ksize=3, head_dim=32,
           layers=(W.Layer("qkv", 128, 256),)), 0, None),
    # head rows split over warps: 96 = 64 + 32 rows, and 256 rows on four warps; a third window
    (_case("c3_qkv_2b_headwise_gqa", 1, 584, "cf_hw_k4_hd96", head_dim=96,
           layers=(W.Layer("qkv", 128, 384),)), 0, None),
    (_case("c3_qkv_2b_headwise_gqa", 2, 264, "cf_hw_k4_hd256", head_dim=256,
           layers=(W.Layer("qkv", 256, 512),)), 0, None),
    # seqlen not a multiple of 8: the generic kernels
    (_case("c2_qkv_150m_lowrank", 2, 130, "cf_odd_T"), 0, None),
    (C["c1_fp32_lowrank"], 0, None),
    # packed documents, [C, N]
    (_case("c5_varlen_packed", 1, 704, "cf_varlen"), 0, [0, 1, 3, 6, 10, 15, 115, 400, 704]),
    (_case("c3_qkv_2b_headwise_gqa", 1, 704, "cf_hw_varlen", varlen=True), 0, [0, 2, 9, 130, 131, 500, 704]),
]

ALGOS = pytest.mark.parametrize("algo", [1, 0, 2], ids=["simt", "auto", "tc"])


def _cf(t, batch, seqlen, pad=0):
    """[N, C] -> [batch, C, seqlen] (channel rows seqlen + pad apart)."""
    C_ = t.shape[1]
    out = torch.zeros((batch, C_, seqlen + pad), dtype=t.dtype, device=t.device)
    out[:, :, :seqlen] = t.reshape(batch, seqlen, C_).transpose(1, 2)
    return out[:, :, :seqlen]


def _tm(t):
    """[batch, C, seqlen] -> [N, C] fp64 host array."""
    b, C_, T = t.shape
    return W.to_f64(t.transpose(1, 2).reshape(b * T, C_))


def _inputs(w, layer, cu):
    x = W.make_inputs(w, layer)
    if cu is not None:
        x["cu_seqlens"] = np.array(cu, dtype=np.int32)
    dt = W.storage_dtype(w)
    t = {k: torch.tensor(v, dtype=torch.float64).to(dt).cuda() for k, v in x.items() if k != "cu_seqlens"}
    t["cu_seqlens"] = torch.tensor(np.asarray(x["cu_seqlens"]), dtype=torch.int32).cuda()
    return x, t


def _plan(w, layer, layout, algo, us=0, deterministic=False):
    from dynamic_short_convolutions_b200 import ops, _lib as L

    kind = L.LOWRANK if w.kind == W.LOWRANK else L.HEADWISE
    batch, seqlen = (1, w.tokens) if w.varlen else (w.batch, w.seqlen)
    return ops.DynConvPlan(kind, W.storage_dtype(w), batch, seqlen, layer.d_model, layer.channels, w.ksize, w.rank,
                           w.head_dim, us, 0, deterministic=deterministic, algo=algo, device="cuda", layout=layout)


def run_cf(w, layer, t, algo, pad=0, deterministic=False):
    """Forward + backward in the channel-first layout; outputs back in [N, C] (fp64)."""
    from dynamic_short_convolutions_b200 import _lib as L

    batch, seqlen = (1, w.tokens) if w.varlen else (w.batch, w.seqlen)
    u = _cf(t["u"], batch, seqlen, pad)
    g = _cf(t["g"], batch, seqlen).contiguous()
    plan = _plan(w, layer, L.CHANNEL_FIRST, algo, u.stride(1), deterministic)
    A = t.get("A")
    BW = t["B"] if w.kind == W.LOWRANK else t["W"]
    cu = t["cu_seqlens"] if w.varlen else None
    R = w.rank if w.kind == W.LOWRANK else (layer.channels // w.head_dim) * w.ksize
    z = torch.empty((w.tokens, R), dtype=W.storage_dtype(w), device="cuda")
    y = plan.forward(u, t["h"], A, BW, cu, z_save=z)
    out = plan.backward(g, u, t["h"], A, BW, cu, z_saved=z)
    assert L.dynconv_device_status(plan.ws) == 0, L.dynconv_last_error()
    torch.cuda.synchronize()
    assert y.shape == (batch, layer.channels, seqlen) and out["du"].shape == y.shape
    return dict(y=_tm(y), du=_tm(out["du"]), dh=W.to_f64(out["dh"]), dA=W.to_f64(out["dA"]) if A is not None else None,
                dBW=W.to_f64(out["dBW"]), z=W.to_f64(z) if w.kind == W.LOWRANK else None)


def run_tm_forward(w, layer, t, algo):
    from dynamic_short_convolutions_b200 import _lib as L

    plan = _plan(w, layer, L.TOKEN_MAJOR, algo)
    A = t.get("A")
    BW = t["B"] if w.kind == W.LOWRANK else t["W"]
    y = plan.forward(t["u"], t["h"], A, BW, t["cu_seqlens"] if w.varlen else None)
    torch.cuda.synchronize()
    return W.to_f64(y)


def _run_or_skip(fn, algo):
    from dynamic_short_convolutions_b200 import _lib as L

    try:
        return fn()
    except L.DynConvError as e:
        if algo == 2 and e.status == 2:
            pytest.skip("shape outside the tensor-core kernels' coverage")
        raise


def _compare(w, gpu, ref):
    for k in ("y", "du", "dh", "dA", "dBW", "z"):
        if gpu.get(k) is None or ref.get(k) is None:
            continue
        assert_close(f"{w.name}:{k}", gpu[k], ref[k], w.dtype)


@ALGOS
@pytest.mark.parametrize("case", CASES, ids=[c[0].name for c in CASES])
def test_channel_first_parity(case, algo):
    w, li, cu = case
    layer = w.layers[li]
    x, t = _inputs(w, layer, cu)
    gpu = _run_or_skip(lambda: run_cf(w, layer, t, algo), algo)
    _compare(w, gpu, oracle_all(w, layer, x))
    # the same arithmetic in the same order as the token-major forward of the same kernel family
    # (AUTO may pick different families for the two layouts)
    if algo != 0:
        from dynamic_short_convolutions_b200 import _lib as L

        try:
            y_tm = run_tm_forward(w, layer, t, algo)
        except L.DynConvError as e:
            assert e.status == 2
            return
        assert np.array_equal(gpu["y"], y_tm)


@ALGOS
def test_channel_first_strided_u(algo):
    """u's channel rows farther apart than seqlen (a slice of a wider buffer)."""
    w = _case("c2_qkv_150m_lowrank", 2, 296, "cf_strided")
    layer = w.layers[0]
    x, t = _inputs(w, layer, None)
    gpu = _run_or_skip(lambda: run_cf(w, layer, t, algo, pad=24), algo)
    _compare(w, gpu, oracle_all(w, layer, x))


@ALGOS
def test_channel_first_headwise_strided_u(algo):
    w = _case("c3_qkv_2b_headwise_gqa", 1, 264, "cf_hw_strided")
    layer = w.layers[0]
    x, t = _inputs(w, layer, None)
    gpu = _run_or_skip(lambda: run_cf(w, layer, t, algo, pad=8), algo)
    _compare(w, gpu, oracle_all(w, layer, x))


def test_channel_first_deterministic_is_bitwise_repeatable():
    for w in (_case("c2_qkv_150m_lowrank", 2, 136, "cf_det"), _case("c3_qkv_2b_headwise_gqa", 1, 264, "cf_hw_det")):
        layer = w.layers[0]
        _, t = _inputs(w, layer, None)
        a = run_cf(w, layer, t, 0, deterministic=True)
        b = run_cf(w, layer, t, 0, deterministic=True)
        for k in a:
            if a[k] is not None:
                assert np.array_equal(a[k], b[k]), (w.name, k)


def test_channel_first_autograd():
    """The autograd Function takes a [batch, C, seqlen] u and returns y and du in that layout."""
    from dynamic_short_convolutions_b200 import ops

    w = _case("c2_qkv_150m_lowrank", 2, 136, "cf_autograd")
    layer = w.layers[0]
    x, t = _inputs(w, layer, None)
    u = _cf(t["u"], w.batch, w.seqlen).contiguous().requires_grad_(True)
    h = t["h"].clone().requires_grad_(True)
    A = t["A"].clone().requires_grad_(True)
    B = t["B"].clone().requires_grad_(True)
    y = ops.dynamic_short_conv(u, h, A, B, ksize=w.ksize, batch=w.batch)
    assert y.shape == u.shape
    y.backward(_cf(t["g"], w.batch, w.seqlen).contiguous())
    ref = oracle_all(w, layer, x)
    assert_close("autograd:y", _tm(y.detach()), ref["y"], "bf16")
    assert_close("autograd:du", _tm(u.grad), ref["du"], "bf16")
    assert_close("autograd:dh", W.to_f64(h.grad), ref["dh"], "bf16")
    assert_close("autograd:dA", W.to_f64(A.grad), ref["dA"], "bf16")
    assert_close("autograd:dB", W.to_f64(B.grad), ref["dBW"], "bf16")


def test_channel_first_argument_errors():
    from dynamic_short_convolutions_b200 import _lib as L

    # the tensor-core kernels need seqlen and the channel stride to be multiples of 8
    d = L.make_desc(L.LOWRANK, L.BF16, 1, 130, 768, 2304, 3, 32, algo=L.ALGO_TC, layout=L.CHANNEL_FIRST)
    ws = torch.zeros(L.dynconv_workspace_bytes(d), dtype=torch.uint8, device="cuda")
    u = torch.zeros((1, 2304, 130), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((130, 768), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((768, 32), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((32, 2304 * 3), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_fwd(d, u, h, A, B, torch.empty_like(u), None, ws)
    assert e.value.status == 2


FULL = ["c2_qkv_150m_lowrank", "c3_qkv_2b_headwise_gqa"]


@pytest.mark.parametrize("name", FULL)
def test_channel_first_full_size_sampled(name):
    """Benchmark-size problems in the channel-first layout, sampled rows against the oracle."""
    from dynamic_short_convolutions_b200 import _lib as L, ops
    from oracle import oracle as O

    w = W.CONFIGS[name]
    layer = w.layers[0]
    t = W.make_inputs(w, layer, 0, device="cuda")
    kind = L.LOWRANK if w.kind == W.LOWRANK else L.HEADWISE
    plan = ops.DynConvPlan(kind, W.storage_dtype(w), w.batch, w.seqlen, layer.d_model, layer.channels, w.ksize,
                           w.rank, w.head_dim, device="cuda", layout=L.CHANNEL_FIRST)
    u = _cf(t["u"], w.batch, w.seqlen).contiguous()
    g = _cf(t["g"], w.batch, w.seqlen).contiguous()
    A = t.get("A")
    BW = t["B"] if kind == L.LOWRANK else t["W"]
    R = w.rank if kind == L.LOWRANK else (layer.channels // w.head_dim) * w.ksize
    z = torch.empty((w.tokens, R), dtype=W.storage_dtype(w), device="cuda")
    y = plan.forward(u, t["h"], A, BW, z_save=z)
    out = plan.backward(g, u, t["h"], A, BW, z_saved=z)
    assert L.dynconv_device_status(plan.ws) == 0, L.dynconv_last_error()
    rng = np.random.default_rng(77)
    N = w.tokens
    rows = sorted({0, 1, 2, 3, 127, 128, 129, N - 1, N - 2, w.seqlen - 1, w.seqlen, w.seqlen + 1,
                   *(int(v) for v in rng.integers(0, N, 16))})
    bi, ti = np.array(rows) // w.seqlen, np.array(rows) % w.seqlen
    pick = lambda a: W.to_f64(a[torch.as_tensor(bi, device="cuda"), :, torch.as_tensor(ti, device="cuda")])
    x = {k: W.to_f64(v) for k, v in t.items() if k != "cu_seqlens"}
    cu = np.arange(0, N + 1, w.seqlen)
    p = oracle_problem(w, layer, cu)
    Ah = x.get("A")
    BWh = x["B"] if kind == L.LOWRANK else x["W"]
    yr, _, _ = O.forward(p, x["u"], x["h"], Ah, BWh, rows=rows)
    dur, _, dhr = O.backward_rows(p, x["g"], x["u"], x["h"], Ah, BWh, rows=rows)
    assert_close(f"{name}:cf:y", pick(y), yr, w.dtype)
    assert_close(f"{name}:cf:du", pick(out["du"]), dur, w.dtype)
    assert_close(f"{name}:cf:dh", W.to_f64(out["dh"])[rows], dhr, w.dtype)
    del t, x, y, z, out, u, g
    torch.cuda.empty_cache()
