"""The forward entry point that allocates nothing (dynconv_fwd_noalloc).

It exists for callers that cannot call cudaMalloc -- code that must not enter
the CUDA allocator or that only ever receives device pointers from elsewhere.
Its scratch is a buffer built into the library, shared by every call.  This
file checks, through the C ABI, that two calls in a row (different inputs, so a
stale buffer would show) give the same outputs as dynconv_fwd with a caller
workspace, within the bf16 tolerances of the other parity tests, and that a
problem too large for the built-in buffer is rejected with a clear error.
The file name makes pytest collect it last.
"""
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from helpers import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _inputs(seed_offset):
    import dataclasses

    w = W.scaled(W.CONFIGS["c2_qkv_150m_lowrank"], 2, 300, name="noalloc")
    w = dataclasses.replace(w, seed=w.seed + seed_offset)
    layer = w.layers[0]
    t = W.make_inputs(w, layer, device="cuda")
    return w, layer, t


def _reference(w, layer, t):
    from dynamic_short_convolutions_b200 import _lib as L, ops

    plan = ops.DynConvPlan(L.LOWRANK, torch.bfloat16, w.batch, w.seqlen, layer.d_model, layer.channels, w.ksize,
                           w.rank, algo=L.ALGO_TC, device="cuda")
    z = torch.empty((w.tokens, w.rank), dtype=torch.bfloat16, device="cuda")
    y = plan.forward(t["u"], t["h"], t["A"], t["B"], z_save=z)
    return y, z


def test_noalloc_forward_matches_workspace_forward_twice():
    from dynamic_short_convolutions_b200 import _lib as L

    for call, seed_offset in enumerate((0, 17)):
        w, layer, t = _inputs(seed_offset)
        y_ref, z_ref = _reference(w, layer, t)
        desc = L.make_desc(L.LOWRANK, L.BF16, w.batch, w.seqlen, layer.d_model, layer.channels, w.ksize, w.rank)
        y = torch.full_like(y_ref, float("nan"))
        L.dynconv_fwd_noalloc(desc, t["u"], t["h"], t["A"], t["B"], y)
        z = torch.full_like(z_ref, float("nan"))
        y2 = torch.full_like(y_ref, float("nan"))
        L.dynconv_fwd_noalloc(desc, t["u"], t["h"], t["A"], t["B"], y2, z)
        torch.cuda.synchronize()
        assert_close(f"call{call}:y", W.to_f64(y), W.to_f64(y_ref), "bf16")
        assert_close(f"call{call}:y_zsave", W.to_f64(y2), W.to_f64(y_ref), "bf16")
        assert_close(f"call{call}:z", W.to_f64(z), W.to_f64(z_ref), "bf16")


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
