"""The tensor-core building blocks (TMA 128-byte-swizzled tiles, UMMA descriptors
for K-major and MN-major operands, TMEM loads) on one tile, against torch."""
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [(0, 64, 64), (0, 192, 64), (0, 256, 64), (0, 96, 64), (0, 192, 192), (0, 64, 128),
         (1, 64, 64), (1, 64, 16), (1, 96, 128), (1, 256, 128), (1, 128, 32),
         (2, 64, 64), (2, 192, 64), (2, 256, 64), (2, 96, 64)]
SHIFTED = [(3, 64, 1), (3, 64, 2), (3, 64, 3), (3, 64, 5), (4, 64, 1), (4, 64, 3)]


@pytest.mark.parametrize("variant,N,Kd", CASES)
def test_umma_tile(variant, N, Kd):
    from dynamic_short_convolutions_b200 import _lib as L

    g = torch.Generator(device="cuda").manual_seed(1000 * variant + N + Kd)
    if variant == 0:
        A = torch.randn(128, Kd, device="cuda", generator=g).bfloat16()
        B = torch.randn(N, Kd, device="cuda", generator=g).bfloat16()
        ref = A.double() @ B.double().T
    elif variant == 2:
        A = torch.randn(128, Kd, device="cuda", generator=g).bfloat16()
        B = torch.randn(Kd, N, device="cuda", generator=g).bfloat16()
        ref = A.double() @ B.double()
    else:
        A = torch.randn(Kd, 128, device="cuda", generator=g).bfloat16()
        B = torch.randn(Kd, N, device="cuda", generator=g).bfloat16()
        ref = A.double().T @ B.double()
    D = torch.full((128, N), float("nan"), device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert L.dynconv_selftest_umma(variant, A, B, D, N, Kd, err) == 0
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    torch.testing.assert_close(D.double(), ref, rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("variant,N,shift", SHIFTED)
def test_umma_row_shifted_operand(variant, N, shift):
    """A K-major operand that starts a few rows into a 128-byte-swizzled tile.
    Variant 3 (base offset 0) is the form the backward kernel relies on; variant 4
    is recorded for information and is allowed to differ."""
    from dynamic_short_convolutions_b200 import _lib as L

    g = torch.Generator(device="cuda").manual_seed(77 + shift)
    A = torch.randn(136, 64, device="cuda", generator=g).bfloat16()
    B = torch.randn(N, 64, device="cuda", generator=g).bfloat16()
    ref = A[shift:shift + 128].double() @ B.double().T
    D = torch.full((128, N), float("nan"), device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert L.dynconv_selftest_umma(variant, A, B, D, N, shift, err) == 0
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    ok = torch.allclose(D.double(), ref, rtol=1e-5, atol=1e-4)
    print(f"variant {variant} shift {shift}: {'match' if ok else 'MISMATCH'}")
    if variant == 3:
        assert ok


def test_bounded_wait_runs_out_and_reports():
    """A wait on an mbarrier that nothing completes ends after its limit (20 ms), raises the
    wait-timeout bit, takes the other waiting warp of the CTA down with it through the abort
    flag, and leaves the context usable: a tensor-core tile computes correctly afterwards."""
    import time

    from dynamic_short_convolutions_b200 import _lib as L

    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.zeros(2, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert L.dynconv_selftest_wait(20_000_000, err, out) == 0
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert out.tolist() == [2, 2]                  # both waits gave up
    assert int(err[0]) & 2                         # the wait-timeout bit
    assert 0.015 < elapsed < 1.0                   # the short limit, not the kernels' 2 s
    # invalid arguments are refused before any launch
    assert L.STATUS_NAMES[L.dynconv_selftest_wait(0, err, out)] == "DYNCONV_ERR_INVALID"
    assert L.STATUS_NAMES[L.dynconv_selftest_wait(3_000_000_000, err, out)] == "DYNCONV_ERR_INVALID"
    # the context still runs work
    g = torch.Generator(device="cuda").manual_seed(5)
    A = torch.randn(128, 64, device="cuda", generator=g).bfloat16()
    B = torch.randn(64, 64, device="cuda", generator=g).bfloat16()
    D = torch.full((128, 64), float("nan"), device="cuda")
    err2 = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert L.dynconv_selftest_umma(0, A, B, D, 64, 64, err2) == 0
    torch.cuda.synchronize()
    assert int(err2[0]) == 0
    torch.testing.assert_close(D.double(), A.double() @ B.double().T, rtol=1e-5, atol=1e-4)
