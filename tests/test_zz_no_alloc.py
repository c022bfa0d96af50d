"""The forward entry point that allocates nothing (dynconv_fwd_noalloc) and its
status query (dynconv_noalloc_status).

It exists for callers that cannot call cudaMalloc -- code that must not enter
the CUDA allocator or that only ever receives device pointers from elsewhere.
Its scratch is a buffer built into the library, shared by every call.  This
file checks, through the C ABI, on two calls in a row with different inputs
(so a stale Bp or z left in the shared buffer would show):
  - y and z are bitwise equal to dynconv_fwd's with a caller workspace (the
    same kernels on the same inputs), with and without z_save;
  - y is within the bf16 parity bounds of the fp64 oracle;
  - dynconv_noalloc_status reports DYNCONV_OK after each call;
and that a problem too large for the built-in buffer is rejected with a clear
error.  The file name makes pytest collect it last.
"""
import numpy as np
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from helpers import assert_close, oracle_problem

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _inputs(seed_offset):
    import dataclasses

    w = W.scaled(W.CONFIGS["c2_qkv_150m_lowrank"], 2, 300, name="noalloc")
    w = dataclasses.replace(w, seed=w.seed + seed_offset)
    layer = w.layers[0]
    x = W.make_inputs(w, layer)
    t = {k: torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).cuda() for k, v in x.items()
         if k != "cu_seqlens"}
    return w, layer, x, t


def _workspace_forward(w, layer, t):
    from dynamic_short_convolutions_b200 import _lib as L, ops

    plan = ops.DynConvPlan(L.LOWRANK, torch.bfloat16, w.batch, w.seqlen, layer.d_model, layer.channels, w.ksize,
                           w.rank, algo=L.ALGO_TC, device="cuda")
    z = torch.empty((w.tokens, w.rank), dtype=torch.bfloat16, device="cuda")
    y = plan.forward(t["u"], t["h"], t["A"], t["B"], z_save=z)
    assert L.dynconv_device_status(plan.ws) == 0, L.dynconv_last_error()
    return y, z


def test_noalloc_forward_matches_workspace_forward_twice():
    from dynamic_short_convolutions_b200 import _lib as L
    from oracle import oracle as O

    for call, seed_offset in enumerate((0, 17)):
        w, layer, x, t = _inputs(seed_offset)
        y_ref, z_ref = _workspace_forward(w, layer, t)
        desc = L.make_desc(L.LOWRANK, L.BF16, w.batch, w.seqlen, layer.d_model, layer.channels, w.ksize, w.rank)
        y = torch.full_like(y_ref, float("nan"))
        L.dynconv_fwd_noalloc(desc, t["u"], t["h"], t["A"], t["B"], y)
        assert L.dynconv_noalloc_status() == 0, L.dynconv_last_error()
        z = torch.full_like(z_ref, float("nan"))
        y2 = torch.full_like(y_ref, float("nan"))
        L.dynconv_fwd_noalloc(desc, t["u"], t["h"], t["A"], t["B"], y2, z)
        assert L.dynconv_noalloc_status() == 0, L.dynconv_last_error()
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), f"call {call}: y differs from the workspace forward"
        assert torch.equal(y2, y_ref), f"call {call}: y (z_save given) differs from the workspace forward"
        assert torch.equal(z, z_ref), f"call {call}: z differs from the workspace forward"
        if call == 0:
            cu = np.arange(0, w.tokens + 1, w.seqlen)
            yr, zr, _ = O.forward(oracle_problem(w, layer, cu), x["u"], x["h"], x["A"], x["B"])
            assert_close("noalloc:y", W.to_f64(y), yr, "bf16")
            assert_close("noalloc:z", W.to_f64(z), zr, "bf16")


def test_noalloc_rejects_oversize_and_unsupported():
    from dynamic_short_convolutions_b200 import _lib as L

    dummy = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    big = L.make_desc(L.LOWRANK, L.BF16, 1, 1 << 17, 64, 64, 3, 64)    # z needs 16 MiB > 8 MiB
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_fwd_noalloc(big, dummy, dummy, dummy, dummy, dummy)
    assert e.value.status == 2 and "scratch" in str(e.value)
    f32 = L.make_desc(L.LOWRANK, L.F32, 1, 64, 64, 64, 3, 8)
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_fwd_noalloc(f32, dummy, dummy, dummy, dummy, dummy)
    assert e.value.status == 2
    assert L.dynconv_noalloc_status() == 0
