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
