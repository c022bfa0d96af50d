"""Pins of the oracle's rotary position embedding (orc_rope), the rotation fused
after the Q/K convolution ("Placement": the conv runs on Q, K and V before RoPE).
The pages name RoPE without a variant; the oracle follows the rotation of Su et al.,
"RoFormer: Enhanced Transformer with Rotary Position Embedding" (section 3.4.2):
channel pairs (2i, 2i+1) of each head turn by position * base^(-2i/head_dim).
These checks pin it to values and properties that do not restate that formula:
  - literal cosines and sines at position 1 (pair 0 turns by exactly 1 rad; for a
    head of 8 channels the four pairs turn by 1, 0.1, 0.01 and 0.001 rad at base 1e4;
    with two heads rotated, each head's pairs turn by the same angles);
  - the relative-position property that defines RoPE: <R_m q, R_n k> depends only
    on m - n;
  - orthogonality (the inverse undoes it, pair norms are kept, the adjoint identity);
  - position 0 and channels past n_rot are left bitwise unchanged, and positions
    restart at every packed-document boundary;
  - the gradient of L = <g, rope(conv(...))> by central differences equals the
    conv backward applied to rope^T(g) (the rule the fused backward uses).
A planted mistake (the rotation turned the wrong way) is caught."""
import numpy as np
import pytest

from oracle import oracle as O


def _prob(n, C, cu=None, K=3, r=2, d=3):
    return O.Problem(O.LOWRANK, n, d, C, K, cu if cu is not None else [0, n], rank=r)


def test_literal_values_at_position_one():
    p = _prob(2, 8)
    x = np.zeros((2, 8))
    x[:, 0::2] = 1.0                       # every pair (1, 0)
    y = O.rope(p, x, 8, 8)
    # position 1, base 1e4, head of 8: pair i turns by 10^(-i) rad
    cos = [0.5403023058681398, 0.9950041652780258, 0.9999500004166653, 0.9999995000000417]
    sin = [0.8414709848078965, 0.09983341664682815, 0.009999833334166664, 0.0009999998333333417]
    np.testing.assert_allclose(y[1, 0::2], cos, rtol=0, atol=1e-15)
    np.testing.assert_allclose(y[1, 1::2], sin, rtol=0, atol=1e-15)
    assert np.array_equal(y[0], x[0])      # position 0: identity


def test_head_of_four_two_pairs():
    p = _prob(2, 4)
    x = np.array([[1.0, 0.0, 0.0, 1.0]] * 2)
    y = O.rope(p, x, 4, 4)
    # pair 1 of a 4-channel head turns by 1e4^(-1/2) = 0.01 rad: (0, 1) -> (-sin 0.01, cos 0.01)
    np.testing.assert_allclose(y[1], [0.5403023058681398, 0.8414709848078965, -0.009999833334166664,
                                      0.9999500004166653], rtol=0, atol=1e-15)


def test_every_head_turns_by_the_same_angles():
    # two 4-channel heads, both rotated: the pair index restarts in each head, so at
    # position 1 the second head's pairs turn by 1 and 0.01 rad like the first head's
    p = _prob(2, 8)
    x = np.array([[1.0, 0.0, 0.0, 1.0, 1.0, 0.0, 0.0, 1.0]] * 2)
    y = O.rope(p, x, 8, 4)
    head = [0.5403023058681398, 0.8414709848078965, -0.009999833334166664, 0.9999500004166653]
    np.testing.assert_allclose(y[1], head + head, rtol=0, atol=1e-15)


def test_relative_position_property():
    rng = np.random.default_rng(0)
    n, hd = 40, 16
    p = _prob(n, hd)
    q = rng.standard_normal((1, hd))
    k = rng.standard_normal((1, hd))
    Q = O.rope(p, np.repeat(q, n, 0), hd, hd)
    Kr = O.rope(p, np.repeat(k, n, 0), hd, hd)
    for delta in (0, 1, 5, 17):
        dots = [Q[m] @ Kr[m - delta] for m in range(delta, n)]
        np.testing.assert_allclose(dots, dots[0], rtol=0, atol=1e-12)
        # and it equals rotating q alone by the difference
        assert abs(dots[0] - Q[delta] @ k[0]) < 1e-12


def test_orthogonal_inverse_adjoint():
    rng = np.random.default_rng(1)
    n, C, hd = 30, 24, 8
    p = _prob(n, C)
    x = rng.standard_normal((n, C))
    y = rng.standard_normal((n, C))
    rx = O.rope(p, x, 16, hd)
    np.testing.assert_allclose(O.rope(p, rx, 16, hd, inverse=True), x, rtol=0, atol=1e-14)
    np.testing.assert_allclose(rx[:, 0:16:2] ** 2 + rx[:, 1:16:2] ** 2, x[:, 0:16:2] ** 2 + x[:, 1:16:2] ** 2,
                               rtol=1e-14, atol=0)
    assert np.array_equal(rx[:, 16:], x[:, 16:])     # channels past n_rot untouched
    lhs = np.sum(rx * y)
    rhs = np.sum(x * O.rope(p, y, 16, hd, inverse=True))
    assert abs(lhs - rhs) < 1e-12 * max(1.0, abs(lhs))


def test_positions_restart_at_document_boundaries():
    rng = np.random.default_rng(2)
    cu = [0, 5, 6, 13]
    p = _prob(13, 8, cu=cu)
    row = rng.standard_normal(8)
    x = np.tile(row, (13, 1))
    y = O.rope(p, x, 8, 8)
    for s in cu[:-1]:
        assert np.array_equal(y[s], row)                    # each document's first token
    np.testing.assert_array_equal(y[6 + 3], y[0 + 3])       # same position in two documents
    one = O.rope(_prob(7, 8), x[6:13], 8, 8)                # document 3 alone
    np.testing.assert_array_equal(y[6:13], one)


def test_fused_gradient_by_central_differences():
    """d/dtheta <g, rope(y(u, h, A, B))> equals the conv backward fed with rope^T(g)."""
    rng = np.random.default_rng(3)
    n, C, K, r, d, hd = 9, 8, 3, 2, 3, 4
    cu = [0, 4, 9]
    p = O.Problem(O.LOWRANK, n, d, C, K, cu, rank=r)
    u, h, g = rng.standard_normal((n, C)), rng.standard_normal((n, d)), rng.standard_normal((n, C))
    A, B = rng.standard_normal((d, r)), rng.standard_normal((r, C * K))

    def loss(u_, h_, A_, B_):
        y, _, _ = O.forward(p, u_, h_, A_, B_)
        return float(np.sum(g * O.rope(p, y, 8, hd)))

    gt = O.rope(p, g, 8, hd, inverse=True)
    du, _, dh = O.backward_rows(p, gt, u, h, A, B)
    dA, dB = O.param_grads(p, gt, u, h, A, B)
    eps = 1e-6
    for name, arr, grad in (("u", u, du), ("h", h, dh), ("A", A, dA), ("B", B, dB)):
        for idx in [tuple(rng.integers(0, s) for s in arr.shape) for _ in range(6)]:
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += eps
            a2[idx] -= eps
            args1 = {"u": u, "h": h, "A": A, "B": B}
            args2 = dict(args1)
            args1[name], args2[name] = a1, a2
            fd = (loss(args1["u"], args1["h"], args1["A"], args1["B"]) -
                  loss(args2["u"], args2["h"], args2["A"], args2["B"])) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_planted_wrong_direction_is_caught():
    """Rotating the other way (the adjoint in place of the rotation) breaks the literal pin."""
    p = _prob(2, 8)
    x = np.zeros((2, 8))
    x[:, 0::2] = 1.0
    wrong = O.rope(p, x, 8, 8, inverse=True)
    with pytest.raises(AssertionError):
        np.testing.assert_allclose(wrong[1, 1::2], [0.8414709848078965, 0.09983341664682815,
                                                    0.009999833334166664, 0.0009999998333333417], atol=1e-15)
