"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element by
element, on seeded inputs that span several tiles and a ragged tail, plus edge
cases, invariants and error handling."""
import dataclasses

import numpy as np
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from helpers import assert_close, gpu_run, oracle_all

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

C = W.CONFIGS


def _case(base, batch, seqlen, name, **kw):
    w = W.scaled(C[base], batch, seqlen, name=name)
    return dataclasses.replace(w, **kw) if kw else w


SMALL = [
    (C["c1_fp32_lowrank"], 0),
    (_case("c2_qkv_150m_lowrank", 2, 300, "c2_small"), 0),
    (_case("c3_qkv_2b_headwise_gqa", 2, 200, "c3_small"), 0),
    (_case("c4_all_linear_2b_block", 1, 260, "c4_small_qkv"), 0),
    (_case("c4_all_linear_2b_block", 1, 260, "c4_small_o"), 1),
    (_case("c4_all_linear_2b_block", 1, 260, "c4_small_gate_up"), 2),
    (_case("c4_all_linear_2b_block", 1, 260, "c4_small_down"), 3),
    (_case("c2_qkv_150m_lowrank", 3, 2, "tiny_T_below_K", ksize=4), 0),
    (_case("c2_qkv_150m_lowrank", 1, 1, "single_token"), 0),
    (_case("c2_qkv_150m_lowrank", 2, 129, "k1_r16", ksize=1, rank=16), 0),
    (_case("c2_qkv_150m_lowrank", 2, 257, "k2_r64", ksize=2, rank=64), 0),
    (_case("c2_qkv_150m_lowrank", 1, 140, "k1_r64", ksize=1, rank=64), 0),
    (_case("c2_qkv_150m_lowrank", 1, 200, "k4_r8", ksize=4, rank=8), 0),
    # ranks whose last 16-wide step of the filter MMA is partly padding (r = 24: two steps, r = 48:
    # three steps of the rank-64 kernels)
    (_case("c2_qkv_150m_lowrank", 1, 270, "k3_r24", rank=24), 0),
    (_case("c2_qkv_150m_lowrank", 1, 270, "k3_r48", rank=48), 0),
    (_case("c2_qkv_150m_lowrank", 1, 200, "k4_r40", ksize=4, rank=40), 0),
    (_case("c2_qkv_150m_lowrank", 1, 130, "odd_channels", layers=(W.Layer("x", 40, 72),)), 0),
    (_case("c3_qkv_2b_headwise_gqa", 1, 150, "hw_k2_hd64", ksize=2, head_dim=64,
           layers=(W.Layer("qkv", 256, 640),)), 0),
    # head-wise: K = 3 (taps boxes at odd offsets, chunks of 3 rows), K = 1, heads of 256, 16 and 8
    # channels (32, 2 and 1 lanes per head), lengths that end runs and chunks part-way
    (_case("c3_qkv_2b_headwise_gqa", 1, 333, "hw_k3_hd32", ksize=3, head_dim=32,
           layers=(W.Layer("qkv", 128, 256),)), 0),
    (_case("c3_qkv_2b_headwise_gqa", 2, 97, "hw_k1_hd256", ksize=1, head_dim=256,
           layers=(W.Layer("qkv", 128, 2048),)), 0),
    (_case("c3_qkv_2b_headwise_gqa", 1, 301, "hw_k4_hd16", head_dim=16, layers=(W.Layer("qkv", 64, 256),)), 0),
    (_case("c3_qkv_2b_headwise_gqa", 3, 45, "hw_k4_hd8", head_dim=8, layers=(W.Layer("qkv", 64, 256),)), 0),
]

VARLEN_CU = [0, 1, 3, 6, 10, 15, 115, 400, 700]


def _varlen_case():
    return _case("c5_varlen_packed", 1, 700, "c5_small")


def _to_device(x, w):
    dt = W.storage_dtype(w)
    t = {k: torch.tensor(v, dtype=torch.float64).to(dt).cuda() for k, v in x.items() if k != "cu_seqlens"}
    t["cu_seqlens"] = torch.tensor(np.asarray(x["cu_seqlens"]), dtype=torch.int32).cuda()
    return t


def _compare(w, gpu, ref, skip=()):
    for k in ("y", "du", "dh", "dA", "dBW"):
        if k in skip or ref.get(k) is None:
            continue
        assert_close(f"{w.name}:{k}", gpu[k], ref[k], w.dtype)
    if gpu.get("z") is not None and ref.get("z") is not None:
        assert_close(f"{w.name}:z", gpu["z"], ref["z"], w.dtype)


def _run_or_skip(w, layer, t, algo, **kw):
    from dynamic_short_convolutions_b200 import _lib as L

    try:
        return gpu_run(w, layer, t, algo=algo, **kw)
    except L.DynConvError as e:
        if algo == 2 and e.status == 2:
            pytest.skip("shape outside the tensor-core kernels' coverage")
        raise


ALGOS = pytest.mark.parametrize("algo", [1, 0, 2], ids=["simt", "auto", "tc"])


@ALGOS
@pytest.mark.parametrize("case", SMALL, ids=[c[0].name for c in SMALL])
def test_small_parity(case, algo):
    w, li = case
    layer = w.layers[li]
    x = W.make_inputs(w, layer, li)
    gpu = _run_or_skip(w, layer, _to_device(x, w), algo)
    _compare(w, gpu, oracle_all(w, layer, x))


@ALGOS
def test_varlen_parity(algo):
    w = _varlen_case()
    layer = w.layers[0]
    x = W.make_inputs(w, layer)
    x["cu_seqlens"] = np.array(VARLEN_CU, dtype=np.int32)
    gpu = _run_or_skip(w, layer, _to_device(x, w), algo)
    _compare(w, gpu, oracle_all(w, layer, x))


@ALGOS
def test_varlen_parity_headwise(algo):
    """Packed documents through the head-wise kernels: runs and chunks that cross document
    starts, documents shorter than K."""
    w = _case("c3_qkv_2b_headwise_gqa", 1, 700, "hw_varlen", varlen=True, layers=(W.Layer("qkv", 128, 512),))
    layer = w.layers[0]
    x = W.make_inputs(w, layer)
    x["cu_seqlens"] = np.array(VARLEN_CU, dtype=np.int32)
    gpu = _run_or_skip(w, layer, _to_device(x, w), algo)
    _compare(w, gpu, oracle_all(w, layer, x))


@ALGOS
def test_recompute_z_and_no_dh(algo):
    w = _case("c2_qkv_150m_lowrank", 2, 140, "no_zsave")
    layer = w.layers[0]
    x = W.make_inputs(w, layer)
    gpu = _run_or_skip(w, layer, _to_device(x, w), algo, z_roundtrip=False, want_dh=False)
    _compare(w, gpu, oracle_all(w, layer, x), skip=("dh",))


@ALGOS
def test_strided_u_and_h(algo):
    """u and h as column slices of wider (fused-projection) tensors."""
    w = _case("c2_qkv_150m_lowrank", 2, 150, "strided")
    layer = w.layers[0]
    x = W.make_inputs(w, layer)
    t = _to_device(x, w)
    N, Cc, d = w.tokens, layer.channels, layer.d_model
    big_u = torch.zeros((N, Cc + 64), dtype=torch.bfloat16, device="cuda")
    big_u[:, 64:] = t["u"]
    big_h = torch.zeros((N, d + 8), dtype=torch.bfloat16, device="cuda")
    big_h[:, :d] = t["h"]
    t["u"], t["h"] = big_u[:, 64:], big_h[:, :d]
    gpu = _run_or_skip(w, layer, t, algo)
    _compare(w, gpu, oracle_all(w, layer, x))


@ALGOS
def test_causality_and_isolation_on_gpu(algo):
    """Perturbing token t* leaves every earlier output bitwise unchanged; perturbing a
    document changes nothing outside it."""
    w = _case("c5_varlen_packed", 1, 600, "causal")
    layer = W.Layer("x", 256, 512)
    w = dataclasses.replace(w, layers=(layer,))
    x = W.make_inputs(w, layer)
    cu = np.array([0, 7, 300, 301, 600], dtype=np.int32)
    x["cu_seqlens"] = cu
    t = _to_device(x, w)
    y0 = _run_or_skip(w, layer, t, algo)["y"]
    t2 = {k: v.clone() for k, v in t.items()}
    ts = 333
    t2["u"][ts] += 1.0
    t2["h"][ts] += 1.0
    y1 = gpu_run(w, layer, t2, algo=algo)["y"]
    assert np.array_equal(y1[:ts], y0[:ts])
    assert not np.array_equal(y1[ts], y0[ts])
    assert np.array_equal(y1[cu[4]:], y0[cu[4]:]) if cu[4] < w.tokens else True
    t3 = {k: v.clone() for k, v in t.items()}
    t3["u"][cu[1]:cu[2]] += 1.0
    y3 = gpu_run(w, layer, t3, algo=algo)["y"]
    outside = np.r_[0:cu[1], cu[2]:w.tokens]
    assert np.array_equal(y3[outside], y0[outside])


@ALGOS
def test_deterministic_mode_is_bitwise_repeatable(algo):
    w = _case("c2_qkv_150m_lowrank", 2, 260, "det")
    layer = w.layers[0]
    t = _to_device(W.make_inputs(w, layer), w)
    a = _run_or_skip(w, layer, t, algo, deterministic=True)
    b = gpu_run(w, layer, t, algo=algo, deterministic=True)
    for k in a:
        if a[k] is not None:
            assert np.array_equal(a[k], b[k]), k


def test_empty_input():
    from dynamic_short_convolutions_b200 import ops, _lib as L

    plan = ops.DynConvPlan(L.LOWRANK, torch.bfloat16, 0, 16, 32, 64, 3, 16)
    e = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    eh = torch.empty((0, 32), dtype=torch.bfloat16, device="cuda")
    A = torch.randn(32, 16, device="cuda").bfloat16()
    B = torch.randn(16, 192, device="cuda").bfloat16()
    y = plan.forward(e, eh, A, B)
    assert y.shape == (0, 64)
    out = plan.backward(e, e, eh, A, B)
    torch.cuda.synchronize()
    assert not torch.any(out["dA"]) and not torch.any(out["dBW"])


def test_argument_errors():
    from dynamic_short_convolutions_b200 import _lib as L

    lib = L.load()
    import ctypes

    desc = L.make_desc(L.LOWRANK, L.BF16, 1, 64, 32, 64, 3, 16)
    nbytes = L.dynconv_workspace_bytes(desc)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    u = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((64, 32), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((32, 16), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((16, 192), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros_like(u)
    with pytest.raises(L.DynConvError) as e:                   # host pointer
        L.dynconv_fwd(desc, u.cpu(), h, A, B, y, None, ws)
    assert e.value.status == 1
    with pytest.raises(L.DynConvError) as e:                   # misaligned pointer
        L.dynconv_fwd(desc, u.view(-1)[1:], h, A, B, y, None, ws)
    assert e.value.status == 1
    with pytest.raises(L.DynConvError) as e:                   # short workspace
        L.dynconv_fwd(desc, u, h, A, B, y, None, ws[: nbytes // 2])
    assert e.value.status == 3
    bad = L.make_desc(L.LOWRANK, L.BF16, 1, 64, 32, 64, 5, 16)  # K = 5
    assert L.dynconv_workspace_bytes(bad) == 0
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_fwd(bad, u, h, A, B, y, None, ws)
    assert e.value.status == 2
    st = lib.dynconv_fwd(None, None, None, None, None, None, None, None, 0, None)
    assert st == 1
    # malformed cu_seqlens: caught by the device pre-check, reported on query
    vdesc = L.make_desc(L.LOWRANK, L.BF16, 1, 64, 32, 64, 3, 16)
    cu = torch.tensor([0, 40, 30, 64], dtype=torch.int32, device="cuda")
    L.dynconv_fwd_varlen(vdesc, cu, u, h, A, B, y, None, ws)
    assert L.dynconv_device_status(ws) == 5
    assert L.dynconv_device_status(ws) == 0                    # cleared after the report
    cu2 = torch.tensor([0, 40, 63], dtype=torch.int32, device="cuda")   # does not end at N
    L.dynconv_fwd_varlen(vdesc, cu2, u, h, A, B, y, None, ws)
    assert L.dynconv_device_status(ws) == 5


def test_query_family_names_the_fallbacks():
    """On the GPU the tensor-core kernels take the workload shapes; the deterministic
    low-rank backward, ranks above 64 and fp32 storage are reported as CUDA-core runs."""
    from dynamic_short_convolutions_b200 import _lib as L

    q = L.dynconv_query_family
    assert q(L.make_desc(L.LOWRANK, L.BF16, 8, 2048, 768, 2304, 3, 32))[:2] == ("tensor_core", "tensor_core")
    assert q(L.make_desc(L.HEADWISE, L.BF16, 4, 4096, 2048, 3072, 4, head_dim=128))[:2] == \
        ("tensor_core", "tensor_core")
    f, b, why = q(L.make_desc(L.LOWRANK, L.BF16, 8, 2048, 768, 2304, 3, 32, deterministic=1))
    assert (f, b) == ("tensor_core", "cuda_core") and "deterministic" in why
    f, b, why = q(L.make_desc(L.LOWRANK, L.BF16, 1, 256, 256, 256, 3, 128))
    assert (f, b) == ("cuda_core", "cuda_core") and "rank" in why
    f, b, why = q(L.make_desc(L.LOWRANK, L.F32, 2, 128, 64, 64, 3, 4))
    assert (f, b) == ("cuda_core", "cuda_core") and "fp32" in why
