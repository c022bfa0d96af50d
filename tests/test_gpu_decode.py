"""Decode step on the GPU (dynconv_decode_step) against the fp64 oracle: a rollout of
several steps per case, the state carried on the GPU, outputs compared step by step and the
final state compared exactly (it only moves stored inputs)."""
import numpy as np
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from helpers import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [  # kind, dtype, batch, d, C, K, r, head_dim
    ("lowrank", "bf16", 1, 64, 256, 3, 32, 0),
    ("lowrank", "bf16", 13, 768, 2304, 3, 32, 0),      # ragged over the 8-sequence blocks
    ("lowrank", "bf16", 9, 200, 200, 4, 64, 0),        # channels not a multiple of the block
    ("lowrank", "f32", 5, 48, 96, 2, 8, 0),
    ("lowrank", "bf16", 4, 64, 128, 1, 16, 0),          # K = 1: no state
    ("headwise", "bf16", 6, 256, 512, 4, 0, 128),
    ("headwise", "f32", 3, 40, 80, 3, 0, 16),
]


def _tensors(kind, dtype, Bs, T, d, C, K, r, hd, seed):
    rnd = lambda tag, n, std=1.0: W.round_to_storage(W.normal(seed, tag, n, std), dtype)
    x = {"u": rnd("u", T * Bs * C).reshape(T, Bs, C), "h": rnd("h", T * Bs * d).reshape(T, Bs, d)}
    if kind == "lowrank":
        x["A"] = rnd("A", d * r, 1 / np.sqrt(d)).reshape(d, r)
        x["BW"] = rnd("B", r * C * K, 1 / np.sqrt(r)).reshape(r, C * K)
    else:
        x["A"] = None
        x["BW"] = rnd("W", d * (C // hd) * K, 1 / np.sqrt(d)).reshape(d, (C // hd) * K)
    return x


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_decode_rollout(case):
    from dynamic_short_convolutions_b200 import _lib as L
    from oracle import oracle as O

    kind, dtype, Bs, d, C, K, r, hd = case
    T = 5
    x = _tensors(kind, dtype, Bs, T, d, C, K, r, hd, seed=7 + K)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    dev = lambda a: None if a is None else torch.tensor(a, dtype=torch.float64).to(tdt).cuda().contiguous()
    desc = L.make_desc(L.LOWRANK if kind == "lowrank" else L.HEADWISE, L.BF16 if dtype == "bf16" else L.F32,
                       Bs, 1, d, C, K, r, hd)
    ws = torch.zeros(L.dynconv_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    state = torch.zeros((Bs, K - 1, C), dtype=tdt, device="cuda") if K > 1 else None
    A, BW = dev(x["A"]), dev(x["BW"])
    p = O.Problem(O.LOWRANK if kind == "lowrank" else O.HEADWISE, Bs, d, C, K, [0, Bs], rank=r, head_dim=hd)
    ostate = np.zeros((Bs, K - 1, C))
    for t in range(T):
        u, h = dev(x["u"][t]), dev(x["h"][t])
        y = torch.empty((Bs, C), dtype=tdt, device="cuda")
        L.dynconv_decode_step(desc, u, h, A, BW, state, y, ws)
        yr, ostate = O.decode_step(p, x["u"][t], x["h"][t], x["A"], x["BW"], ostate)
        torch.cuda.synchronize()
        assert_close(f"step{t}:y", W.to_f64(y), yr, dtype)
    assert L.dynconv_device_status(ws) == 0
    if K > 1:
        assert np.array_equal(W.to_f64(state), ostate), "state after the rollout"


def test_decode_matches_forward_rows():
    """Token-by-token decode from a zero state equals the forward over the whole sequence."""
    from dynamic_short_convolutions_b200 import _lib as L, ops

    Bs, T, d, C, K, r = 4, 9, 128, 512, 4, 32
    x = _tensors("lowrank", "bf16", Bs, T, d, C, K, r, 0, seed=3)
    dev = lambda a: torch.tensor(a, dtype=torch.float64).to(torch.bfloat16).cuda().contiguous()
    u_seq = dev(np.transpose(x["u"], (1, 0, 2)).reshape(Bs * T, C))     # [b, t] -> token b*T + t
    h_seq = dev(np.transpose(x["h"], (1, 0, 2)).reshape(Bs * T, d))
    A, B = dev(x["A"]), dev(x["BW"])
    plan = ops.DynConvPlan(L.LOWRANK, torch.bfloat16, Bs, T, d, C, K, r, algo=L.ALGO_SIMT, device="cuda")
    y_fwd = plan.forward(u_seq, h_seq, A, B)
    desc = L.make_desc(L.LOWRANK, L.BF16, Bs, 1, d, C, K, r, 0)
    ws = torch.zeros(L.dynconv_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    state = torch.zeros((Bs, K - 1, C), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        y = torch.empty((Bs, C), dtype=torch.bfloat16, device="cuda")
        L.dynconv_decode_step(desc, dev(x["u"][t]), dev(x["h"][t]), A, B, state, y, ws)
        rows = torch.arange(Bs, device="cuda") * T + t
        torch.cuda.synchronize()
        # both fp32-accumulated; the decode generator sums over d in eight warp-slices, the
        # forward's in one loop, so z (and then y) may round differently: compare within tolerance
        assert_close(f"step{t}", W.to_f64(y), W.to_f64(y_fwd[rows]), "bf16")


def test_decode_argument_errors():
    from dynamic_short_convolutions_b200 import _lib as L

    t = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    desc = L.make_desc(L.LOWRANK, L.BF16, 2, 2, 8, 8, 3, 8, 0)             # seqlen 2
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_decode_step(desc, t, t, t, t, t, t, ws)
    assert e.value.status == 1
    desc = L.make_desc(L.LOWRANK, L.BF16, 2, 1, 8, 8, 3, 8, 0)
    with pytest.raises(L.DynConvError) as e:                                   # K = 3 needs a state
        L.dynconv_decode_step(desc, t, t, t, t, None, t, ws)
    assert e.value.status == 1
    desc1 = L.make_desc(L.LOWRANK, L.BF16, 2, 1, 8, 8, 1, 8, 0)               # K = 1: no state needed
    L.dynconv_decode_step(desc1, t, t, t, t, None, t, ws)
    torch.cuda.synchronize()


def test_decode_channel_first_descriptor():
    """A channel-first [batch, C, 1] token is the same memory as [batch, C]: a channel-first
    descriptor decodes bitwise like the token-major one; other channel strides are refused."""
    from dynamic_short_convolutions_b200 import _lib as L

    Bs, d, C, K, r = 3, 64, 128, 3, 16
    x = _tensors("lowrank", "bf16", Bs, 2, d, C, K, r, 0, seed=5)
    dev = lambda a: torch.tensor(a, dtype=torch.float64).to(torch.bfloat16).cuda().contiguous()
    A, B = dev(x["A"]), dev(x["BW"])
    outs = []
    for layout in (L.TOKEN_MAJOR, L.CHANNEL_FIRST):
        desc = L.make_desc(L.LOWRANK, L.BF16, Bs, 1, d, C, K, r, 0, layout=layout)
        ws = torch.zeros(L.dynconv_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
        state = torch.zeros((Bs, K - 1, C), dtype=torch.bfloat16, device="cuda")
        ys = []
        for t in range(2):
            y = torch.empty((Bs, C), dtype=torch.bfloat16, device="cuda")
            L.dynconv_decode_step(desc, dev(x["u"][t]), dev(x["h"][t]), A, B, state, y, ws)
            ys.append(y)
        torch.cuda.synchronize()
        outs.append((torch.stack(ys), state.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    desc = L.make_desc(L.LOWRANK, L.BF16, Bs, 1, d, C, K, r, 0, u_row_stride=2, layout=L.CHANNEL_FIRST)
    ws = torch.zeros(L.dynconv_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    t = torch.zeros((Bs, 2 * C), dtype=torch.bfloat16, device="cuda")
    state = torch.zeros((Bs, K - 1, C), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_decode_step(desc, t, dev(x["h"][0]), A, B, state, torch.empty((Bs, C), dtype=torch.bfloat16,
                                                                                  device="cuda"), ws)
    assert e.value.status == 2
