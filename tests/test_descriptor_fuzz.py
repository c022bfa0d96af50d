"""Property test of the C ABI's descriptor validation, on the CPU (host logic only:
dynconv_workspace_bytes and dynconv_query_family launch nothing).

For random descriptors, including negative, zero and near-2^63 fields, the library
must accept exactly those that keep the rules the header states: kind, dtype, algo
and layout from their enums; batch, seqlen >= 0; d_model, channels >= 1; ksize
1..4; low-rank rank 1..128; head-wise head_dim dividing channels; row strides at
least the row and, token-major, a multiple of 16 bytes; and every operand's byte
count below 2^56 without a wrapped product.  An accepted descriptor gets a
non-zero workspace size and a kernel family for both passes (or, when it forces
the tensor-core kernels on a shape they do not cover, DYNCONV_ERR_UNSUPPORTED)."""
import os

import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "dynamic_short_convolutions_b200", "libdynconv.so")
I64 = (1 << 63) - 1
MAX_BYTES = 1 << 56


def _expected_ok(kind, dtype, algo, layout, batch, seqlen, d, C, K, r, hd, us, hs):
    if kind not in (0, 1) or dtype not in (0, 1) or algo not in (0, 1, 2) or layout not in (0, 1):
        return False
    if batch < 0 or seqlen < 0 or d < 1 or C < 1 or K < 1 or K > 4:
        return False
    N = batch * seqlen
    if N > I64:
        return False
    vec = 8 if dtype == 1 else 4
    es = 2 if dtype == 1 else 4
    if layout == 0:
        us = us or C
        if us < C or us % vec:
            return False
    else:
        us = us or seqlen
        if us < seqlen:
            return False
        if seqlen == 1 and us == 1 and C % vec == 0:
            layout, us = 0, C
    hs = hs or d
    if hs < d or hs % vec:
        return False
    if kind == 0:
        if r < 1 or r > 128:
            return False
        R = r
    else:
        if hd < 1 or C % hd:
            return False
        R, r = (C // hd) * K, 0
    rows = N if layout == 0 else batch * C
    return (rows * us * es <= MAX_BYTES and N * hs * es <= MAX_BYTES and N * R * 4 <= MAX_BYTES
            and d * R * 4 <= MAX_BYTES and C * K * max(r, 1) * 4 <= MAX_BYTES)


def _size():
    # mostly small values, with the edges and huge values that make products wrap
    edges = st.sampled_from([-1, 0, 1, 2, 3, 7, 8, 16, 64, 128, 129, 4096, 1 << 31, 1 << 40, 1 << 55,
                             1 << 62, I64])
    return st.one_of(edges, st.integers(-4, 300), st.integers(-(1 << 63), I64))


@settings(max_examples=600, deadline=None)
@given(kind=st.integers(-1, 2), dtype=st.integers(-1, 2), algo=st.integers(-1, 3), layout=st.integers(-1, 2),
       batch=_size(), seqlen=_size(), d=_size(), C=_size(), K=st.integers(-1, 6), r=_size(), hd=_size(),
       us=st.one_of(st.just(0), _size()), hs=st.one_of(st.just(0), _size()))
def test_validation_follows_the_documented_rules(kind, dtype, algo, layout, batch, seqlen, d, C, K, r, hd, us, hs):
    if not os.path.exists(LIB):
        pytest.skip("library not built")
    from dynamic_short_convolutions_b200 import _lib as L

    desc = L.make_desc(kind, dtype, batch, seqlen, d, C, K, rank=r, head_dim=hd, u_row_stride=us,
                       h_row_stride=hs, algo=algo, layout=layout)
    nbytes = L.dynconv_workspace_bytes(desc)
    want = _expected_ok(kind, dtype, algo, layout, batch, seqlen, d, C, K, r, hd, us, hs)
    assert (nbytes > 0) == want, (nbytes, L.dynconv_last_error())
    if want:
        try:
            fwd, bwd, _ = L.dynconv_query_family(desc)
        except L.DynConvError as e:
            # ALGO_TC on a shape outside the tensor-core kernels is refused (UNSUPPORTED), nothing else
            assert algo == 2 and e.status == 2, (e.status, str(e))
        else:
            assert fwd in ("tensor_core", "cuda_core") and bwd in ("tensor_core", "cuda_core")
