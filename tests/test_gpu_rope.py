"""GPU parity of the RoPE fused after the conv (the conv is applied to Q, K and V
before RoPE): the C ABI's y = R(u + conv(u)) and its backward against the oracle's
composite -- R applied to the oracle's y, and the oracle's conv backward fed with
R^T g -- on seeded inputs, through the tensor-core and CUDA-core kernels, dense
batches and packed documents (positions restart at each document), low-rank and
head-wise; plus the position-range errors."""
import dataclasses

import numpy as np
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from helpers import assert_close, oracle_problem

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

C = W.CONFIGS


def _case(base, batch, seqlen, name, **kw):
    w = W.scaled(C[base], batch, seqlen, name=name)
    return dataclasses.replace(w, **kw) if kw else w


def _run(w, layer, x, n_rot, hd, algo, cu=None):
    from dynamic_short_convolutions_b200 import _lib as L, ops

    dt = W.storage_dtype(w)
    t = {k: torch.tensor(v, dtype=torch.float64).to(dt).cuda() for k, v in x.items() if k != "cu_seqlens"}
    varlen = cu is not None
    batch, seqlen = (1, w.tokens) if varlen else (w.batch, w.seqlen)
    kind = L.LOWRANK if w.kind == W.LOWRANK else L.HEADWISE
    table = ops.rope_table(max(seqlen, 1), hd, device="cuda")
    plan = ops.DynConvPlan(kind, dt, batch, seqlen, layer.d_model, layer.channels, w.ksize, w.rank, w.head_dim,
                           algo=algo, device="cuda", rope_channels=n_rot, rope_head_dim=hd, rope_table=table)
    cu_t = torch.tensor(np.asarray(cu), dtype=torch.int32, device="cuda") if varlen else None
    A = t.get("A")
    BW = t["B"] if kind == L.LOWRANK else t["W"]
    y = plan.forward(t["u"], t["h"], A, BW, cu_t)
    out = plan.backward(t["g"], t["u"], t["h"], A, BW, cu_t)
    assert L.dynconv_device_status(plan.ws) == 0, L.dynconv_last_error()
    torch.cuda.synchronize()
    return {"y": W.to_f64(y), "du": W.to_f64(out["du"]), "dh": W.to_f64(out["dh"]),
            "dA": W.to_f64(out["dA"]) if out["dA"] is not None else None, "dBW": W.to_f64(out["dBW"])}


def _oracle(w, layer, x, n_rot, hd, cu):
    from oracle import oracle as O

    p = oracle_problem(w, layer, cu)
    A = x.get("A")
    BW = x["B"] if w.kind == W.LOWRANK else x["W"]
    y, _, _ = O.forward(p, x["u"], x["h"], A, BW)
    gt = O.rope(p, x["g"], n_rot, hd, inverse=True)
    du, _, dh = O.backward_rows(p, gt, x["u"], x["h"], A, BW)
    dA, dBW = O.param_grads(p, gt, x["u"], x["h"], A, BW)
    return {"y": O.rope(p, y, n_rot, hd), "du": du, "dh": dh, "dA": dA, "dBW": dBW}


CASES = [
    # (workload, layer index, rotated channels, rotary head dim)
    (_case("c2_qkv_150m_lowrank", 2, 300, "rope_c2"), 0, 1536, 64),            # Q and K of the 150M QKV
    (_case("c3_qkv_2b_headwise_gqa", 2, 200, "rope_c3"), 0, 2560, 128),        # Q (16 heads) and K (4 heads)
    (_case("c2_qkv_150m_lowrank", 1, 200, "rope_k4_r64", ksize=4, rank=64), 0, 1536, 64),
    # rotary heads narrower than a thread's 32 channels, and not dividing them: the table slice
    # wraps to the next head inside a thread's channel run
    (_case("c2_qkv_150m_lowrank", 1, 160, "rope_hd16"), 0, 1536, 16),
    (_case("c2_qkv_150m_lowrank", 1, 160, "rope_hd40"), 0, 640, 40),
    (C["c1_fp32_lowrank"], 0, 32, 16),
]


@pytest.mark.parametrize("algo", [0, 1], ids=["auto", "simt"])
@pytest.mark.parametrize("case", CASES, ids=[c[0].name for c in CASES])
def test_rope_dense(case, algo):
    w, li, n_rot, hd = case
    layer = w.layers[li]
    x = W.make_inputs(w, layer, li)
    cu = np.arange(0, w.tokens + 1, w.seqlen)
    gpu = _run(w, layer, x, n_rot, hd, algo)
    ref = _oracle(w, layer, x, n_rot, hd, cu)
    for k in ("y", "du", "dh", "dA", "dBW"):
        if ref[k] is not None and gpu[k] is not None:
            assert_close(f"{w.name}:{k}", gpu[k], ref[k], w.dtype)


@pytest.mark.parametrize("algo", [0, 1], ids=["auto", "simt"])
@pytest.mark.parametrize("kind", ["lowrank", "headwise"])
def test_rope_packed_documents(kind, algo):
    if kind == "lowrank":
        w = _case("c5_varlen_packed", 1, 700, "rope_varlen", layers=(W.Layer("x", 256, 512),))
        n_rot, hd = 256, 64
    else:
        w = _case("c3_qkv_2b_headwise_gqa", 1, 700, "rope_varlen_hw", layers=(W.Layer("x", 256, 512),),
                  head_dim=64)
        w = dataclasses.replace(w, varlen=True)
        n_rot, hd = 384, 64
    layer = w.layers[0]
    x = W.make_inputs(w, layer)
    cu = [0, 1, 3, 6, 10, 15, 115, 400, 700]
    gpu = _run(w, layer, x, n_rot, hd, algo, cu=cu)
    ref = _oracle(w, layer, x, n_rot, hd, cu)
    for k in ("y", "du", "dh", "dA", "dBW"):
        if ref[k] is not None and gpu[k] is not None:
            assert_close(f"{w.name}:{k}", gpu[k], ref[k], w.dtype)


def test_rope_families_and_errors():
    from dynamic_short_convolutions_b200 import _lib as L, ops

    table = ops.rope_table(256, 64, device="cuda")
    d = L.make_desc(L.LOWRANK, L.BF16, 2, 256, 768, 2304, 3, 32, rope_channels=1536, rope_head_dim=64,
                    rope_table=table)
    assert L.dynconv_query_family(d)[:2] == ("tensor_core", "tensor_core")
    cf = L.make_desc(L.LOWRANK, L.BF16, 2, 256, 768, 2304, 3, 32, layout=L.CHANNEL_FIRST, rope_channels=1536,
                     rope_head_dim=64, rope_table=table)
    f, b, why = L.dynconv_query_family(cf)
    assert (f, b) == ("cuda_core", "cuda_core") and "RoPE" in why
    # seqlen beyond the table: rejected before any launch
    long = L.make_desc(L.LOWRANK, L.BF16, 1, 300, 64, 128, 3, 16, rope_channels=128, rope_head_dim=64,
                       rope_table=table)
    u = torch.zeros((300, 128), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((300, 64), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((64, 16), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((16, 384), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(1, L.dynconv_workspace_bytes(long)), dtype=torch.uint8, device="cuda")
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_fwd(long, u, h, A, B, torch.empty_like(u), None, ws)
    assert e.value.status == 1
    # a packed document longer than the table: the device check reports it
    cu = torch.tensor([0, 10, 300], dtype=torch.int32, device="cuda")
    L.dynconv_fwd_varlen(long, cu, u, h, A, B, torch.empty_like(u), None, ws)
    assert L.dynconv_device_status(ws) == 5 and "rope_max_pos" in L.dynconv_last_error()
    # the decode step and the no-workspace forward do not rotate
    dec = L.make_desc(L.LOWRANK, L.BF16, 4, 1, 64, 128, 3, 16, rope_channels=128, rope_head_dim=64, rope_table=table)
    ws2 = torch.zeros(L.dynconv_workspace_bytes(dec), dtype=torch.uint8, device="cuda")
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_decode_step(dec, u[:4], h[:4], A, B, torch.zeros((4, 2, 128), dtype=torch.bfloat16,
                                                                    device="cuda"), u[:4].clone(), ws2)
    assert e.value.status == 2


@pytest.mark.parametrize("algo", [0, 1, 2], ids=["auto", "simt", "tc"])
def test_rope_workspace_guard_band(algo):
    """Forward and backward with RoPE write nothing past dynconv_workspace_bytes: the
    workspace is followed by a guard band that must come back untouched (whichever
    kernel family desc->algo asks for)."""
    from dynamic_short_convolutions_b200 import _lib as L, ops

    w = _case("c2_qkv_150m_lowrank", 2, 160, "rope_guard")
    layer = w.layers[0]
    t = W.make_inputs(w, layer, device="cuda")
    table = ops.rope_table(w.seqlen, 64, device="cuda")
    desc = L.make_desc(L.LOWRANK, L.BF16, w.batch, w.seqlen, layer.d_model, layer.channels, w.ksize, w.rank,
                       algo=algo, rope_channels=1536, rope_head_dim=64, rope_table=table)
    nbytes = L.dynconv_workspace_bytes(desc)
    guard = 1 << 20
    buf = torch.zeros(nbytes + guard, dtype=torch.uint8, device="cuda")
    buf[nbytes:] = 0xA5
    ws = buf[:nbytes]
    y = torch.empty_like(t["u"])
    L.dynconv_fwd(desc, t["u"], t["h"], t["A"], t["B"], y, None, ws)
    du, dh = torch.empty_like(t["u"]), torch.empty_like(t["h"])
    dA = torch.empty(tuple(t["A"].shape), dtype=torch.float32, device="cuda")
    dB = torch.empty(tuple(t["B"].shape), dtype=torch.float32, device="cuda")
    L.dynconv_bwd(desc, None, t["g"], t["u"], t["h"], t["A"], t["B"], None, du, dh, dA, dB, ws)
    assert L.dynconv_device_status(ws) == 0, L.dynconv_last_error()
    torch.cuda.synchronize()
    assert bool(torch.all(buf[nbytes:] == 0xA5)), "a write landed past the workspace"
