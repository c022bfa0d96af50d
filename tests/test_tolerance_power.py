"""What the bf16 parity bar (helpers.check_close) can tell apart, on the CPU.

The GPU parity tests compare the CUDA path with the oracle under that bar.  Here
the bar meets, on the same seeded inputs as the GPU case `c2_small` (150M QKV
layer shapes, 2 sequences of 300 tokens, K = 3, r = 32):
  - results a correct kernel can produce: the oracle's values rounded where the
    tensor-core path rounds (z and the staged dw tiles to bf16, fp32 sums, outputs
    stored in bf16).  The bar must pass these.
  - results of plausible kernel mistakes, each planted in the oracle's outputs
    here on the CPU: a dropped tap, a missing document mask, a du tap reading the
    wrong token, a channel chunk missing from the cross-CTA dz reduction, and one
    token tile missing from the dB reduction.  The bar must reject each of these.
The same for the head-wise generator on the inputs of the GPU case `c3_small`:
the correct rounding (bf16 taps and dwh operand) passes; a head taking its
neighbour's taps, a dwh reduction that lost half of a head's channels and a dW
missing one token tile are rejected.
The method's formulas are those of "Dynamic Short Convolutions Improve
Transformers", gist.science technical summary, section "Dynamic Short
Convolutions" (Mechanism, low-rank and head-wise Parameterization, residual
Placement); that a filter stays inside its packed document is this library's
reading of the causal Mechanism for packed sequences.
"""
import numpy as np
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from helpers import check_close, oracle_all

from oracle import oracle as O


def _bf16(a):
    return W.round_to_storage(np.asarray(a, np.float64), "bf16")


def _f32(a):
    return np.asarray(a, np.float64).astype(np.float32).astype(np.float64)


@pytest.fixture(scope="module")
def case():
    w = W.scaled(W.CONFIGS["c2_qkv_150m_lowrank"], 2, 300, name="c2_small")
    layer = w.layers[0]
    x = W.make_inputs(w, layer)
    ref = oracle_all(w, layer, x)
    N, C, K, r = w.tokens, layer.channels, w.ksize, w.rank
    cu = [int(v) for v in x["cu_seqlens"]]
    st = np.zeros(N, dtype=np.int64)
    for s in range(len(cu) - 1):
        st[cu[s]:cu[s + 1]] = cu[s]
    # u[n - j] where the tap stays inside token n's sequence, else 0
    ush = np.zeros((K, N, C))
    for j in range(K):
        ok = (np.arange(N) - j) >= st
        ush[j, ok] = x["u"][np.arange(N)[ok] - j]
    p = O.Problem(O.LOWRANK, N, layer.d_model, C, K, cu, rank=r)
    wf = O.filters(p, x["u"], x["h"], x["A"], x["B"])            # [N, C, K]
    return dict(w=w, layer=layer, x=x, ref=ref, st=st, ush=ush, wf=wf, N=N, C=C, K=K, r=r, cu=cu)


def _ok(name, a, ref):
    return check_close(name, a, ref, "bf16")


def test_rounding_of_a_correct_kernel_passes(case):
    x, ref, ush, K = case["x"], case["ref"], case["ush"], case["K"]
    B3 = x["B"].reshape(case["r"], case["C"], K)
    # forward: z rounded to bf16 before the filter MMA, filters and conv in fp32, y stored in bf16
    zb = _bf16(x["h"] @ x["A"])
    wt = _f32(np.einsum("nk,kcj->ncj", zb, B3))
    y = _bf16(_f32(x["u"] + np.einsum("ncj,jnc->nc", wt, ush)))
    ok, msg = _ok("y", y, ref["y"])
    assert ok, msg
    # backward: the staged dw tiles rounded to bf16 for the dz MMA; dz, dB, dA summed in fp32
    dw = _bf16(x["g"][None] * ush)                                 # [K, N, C]
    dz = _f32(np.einsum("jnc,kcj->nk", dw, B3))
    dB = _f32(np.einsum("nk,jnc->kcj", zb, dw).reshape(case["r"], -1))
    dA = _f32(x["h"].T @ dz)
    dh = _bf16(dz @ x["A"].T)
    for name, a, b in (("dh", dh, ref["dh"]), ("dA", dA, ref["dA"]), ("dB", dB, ref["dBW"])):
        ok, msg = _ok(name, a, b)
        assert ok, msg
    ok, msg = _ok("du", _bf16(ref["du"]), ref["du"])
    assert ok, msg


def test_dropped_tap_is_rejected(case):
    K = case["K"]
    y_bad = case["ref"]["y"] - case["wf"][:, :, K - 1] * case["ush"][K - 1]
    assert not _ok("y", _bf16(y_bad), case["ref"]["y"])[0]


def test_missing_document_mask_is_rejected(case):
    # the filter of the second sequence's first tokens reaching back into the first sequence
    w, layer, x = case["w"], case["layer"], case["x"]
    p_one = O.Problem(O.LOWRANK, case["N"], layer.d_model, case["C"], case["K"], [0, case["N"]], rank=w.rank)
    y_bad, _, _ = O.forward(p_one, x["u"], x["h"], x["A"], x["B"])
    assert not np.array_equal(y_bad, case["ref"]["y"])
    assert not _ok("y", _bf16(y_bad), case["ref"]["y"])[0]


def test_du_tap_reading_the_wrong_token_is_rejected(case):
    # tap j = 1 of du[m] takes g[m + 2] where it should take g[m + 1]
    x, wf, st, N = case["x"], case["wf"], case["st"], case["N"]
    du_bad = case["ref"]["du"].copy()
    for m in range(N - 2):
        if m >= st[m + 1] and m >= st[m + 2]:
            du_bad[m] += wf[m + 1, :, 1] * (x["g"][m + 2] - x["g"][m + 1])
    assert not _ok("du", _bf16(du_bad), case["ref"]["du"])[0]


def test_lost_dz_chunk_is_rejected(case):
    # one 64-channel chunk's contribution missing from the dz reduction (a reduction that did not land)
    x, ush, K, r, C = case["x"], case["ush"], case["K"], case["r"], case["C"]
    B3 = x["B"].reshape(r, C, K)
    sl = slice(64 * 7, 64 * 8)
    part = np.einsum("jnc,kcj->nk", x["g"][None, :, sl] * ush[:, :, sl], B3[:, sl, :])
    _, dz_ref, _ = O.backward_rows(O.Problem(O.LOWRANK, case["N"], case["layer"].d_model, C, K, case["cu"], rank=r),
                                   x["g"], x["u"], x["h"], x["A"], x["B"])
    dz_bad = dz_ref - part
    assert not _ok("dh", _bf16(dz_bad @ x["A"].T), case["ref"]["dh"])[0]
    assert not _ok("dA", _f32(x["h"].T @ dz_bad), case["ref"]["dA"])[0]


def test_lost_dB_tile_is_rejected(case):
    # one 128-token tile missing from the dB reduction over tokens
    x, ush, K, r = case["x"], case["ush"], case["K"], case["r"]
    z = x["h"] @ x["A"]
    t = slice(128, 256)
    part = np.einsum("nk,jnc->kcj", z[t], x["g"][None, t] * ush[:, t]).reshape(r, -1)
    assert not _ok("dB", _f32(case["ref"]["dBW"] - part), case["ref"]["dBW"])[0]


# ---- head-wise: the inputs of the GPU case `c3_small` (2B head-wise GQA layer shapes,
# 2 sequences of 200 tokens, K = 4, 24 heads of 128 channels)

@pytest.fixture(scope="module")
def hcase():
    w = W.scaled(W.CONFIGS["c3_qkv_2b_headwise_gqa"], 2, 200, name="c3_small")
    layer = w.layers[0]
    x = W.make_inputs(w, layer)
    ref = oracle_all(w, layer, x)
    N, C, K, hd = w.tokens, layer.channels, w.ksize, w.head_dim
    H = C // hd
    cu = [int(v) for v in x["cu_seqlens"]]
    st = np.zeros(N, dtype=np.int64)
    for s in range(len(cu) - 1):
        st[cu[s]:cu[s + 1]] = cu[s]
    ush = np.zeros((K, N, C))
    for j in range(K):
        ok = (np.arange(N) - j) >= st
        ush[j, ok] = x["u"][np.arange(N)[ok] - j]
    return dict(x=x, ref=ref, ush=ush, N=N, C=C, K=K, hd=hd, H=H)


def _expand(wh, H, K, hd):
    # wh [N, H*K] (head q, tap j at q*K + j) -> [K, N, H*hd]
    return np.repeat(wh.reshape(-1, H, K).transpose(2, 0, 1), hd, axis=2)


def test_headwise_rounding_of_a_correct_kernel_passes(hcase):
    x, ref, ush, H, K, hd = hcase["x"], hcase["ref"], hcase["ush"], hcase["H"], hcase["K"], hcase["hd"]
    # the generator's taps stored in bf16, the conv in fp32, y stored in bf16
    whb = _bf16(x["h"] @ x["W"])
    y = _bf16(_f32(x["u"] + np.einsum("jnc,jnc->nc", _expand(whb, H, K, hd), ush)))
    ok, msg = _ok("y", y, ref["y"])
    assert ok, msg
    # dwh summed in fp32 over each head's channels, rounded to bf16 as the generator backward's operand
    dwh = _f32(np.einsum("jnqc->nqj", (x["g"][None] * ush).reshape(K, -1, H, hd)).reshape(-1, H * K))
    dwhb = _bf16(dwh)
    for name, a, b in (("dh", _bf16(dwhb @ x["W"].T), ref["dh"]), ("dW", _f32(x["h"].T @ dwhb), ref["dBW"])):
        ok, msg = _ok(name, a, b)
        assert ok, msg


def test_headwise_filter_of_the_wrong_head_is_rejected(hcase):
    x, ush, H, K, hd = hcase["x"], hcase["ush"], hcase["H"], hcase["K"], hcase["hd"]
    wh = (x["h"] @ x["W"]).reshape(-1, H, K)
    wrong = np.roll(wh, 1, axis=1).reshape(-1, H * K)           # head q takes head q-1's taps
    y_bad = x["u"] + np.einsum("jnc,jnc->nc", _expand(wrong, H, K, hd), ush)
    assert not _ok("y", _bf16(y_bad), hcase["ref"]["y"])[0]


def test_headwise_dwh_missing_half_a_head_is_rejected(hcase):
    # the shuffle reduction over a head's lanes losing its last level: half the channels summed
    x, ush, H, K, hd = hcase["x"], hcase["ush"], hcase["H"], hcase["K"], hcase["hd"]
    prod = (x["g"][None] * ush).reshape(K, -1, H, hd)
    dwh_bad = np.einsum("jnqc->nqj", prod[..., : hd // 2]).reshape(-1, H * K)
    assert not _ok("dh", _bf16(dwh_bad @ x["W"].T), hcase["ref"]["dh"])[0]
    assert not _ok("dW", _f32(x["h"].T @ dwh_bad), hcase["ref"]["dBW"])[0]


def test_headwise_lost_dW_tile_is_rejected(hcase):
    x, ush, H, K, hd = hcase["x"], hcase["ush"], hcase["H"], hcase["K"], hcase["hd"]
    dwh = np.einsum("jnqc->nqj", (x["g"][None] * ush).reshape(K, -1, H, hd)).reshape(-1, H * K)
    t = slice(128, 256)
    assert not _ok("dW", _f32(hcase["ref"]["dBW"] - x["h"][t].T @ dwh[t]), hcase["ref"]["dBW"])[0]
