"""Pins of the oracle's decode step (CPU): feeding each sequence token by token from a
zero state must reproduce the oracle's full-sequence forward (an independently pinned
code path), and the state must hold the last K-1 inputs."""
import numpy as np
import pytest

from dynamic_short_convolutions_b200 import workloads as W
from oracle import oracle as O


def _params(kind, d, C, K, r, hd, seed):
    if kind == O.LOWRANK:
        A = W.normal(seed, "A", d * r, 1.0 / np.sqrt(d)).reshape(d, r)
        B = W.normal(seed, "B", r * C * K, 1.0 / np.sqrt(r)).reshape(r, C * K)
        return A, B
    H = C // hd
    return None, W.normal(seed, "W", d * H * K, 1.0 / np.sqrt(d)).reshape(d, H * K)


@pytest.mark.parametrize("kind", [O.LOWRANK, O.HEADWISE])
@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_decode_rollout_equals_forward(kind, K):
    Bs, T, d, C, r, hd = 3, 7, 6, 8, 3, 4
    seed = 11 * K + (kind == O.HEADWISE)
    A, BW = _params(kind, d, C, K, r, hd, seed)
    u = W.normal(seed, "u", Bs * T * C).reshape(Bs * T, C)
    h = W.normal(seed, "h", Bs * T * d).reshape(Bs * T, d)
    full = O.Problem(kind, Bs * T, d, C, K, list(range(0, Bs * T + 1, T)), rank=r, head_dim=hd)
    y_full, _, _ = O.forward(full, u, h, A, BW)
    step = O.Problem(kind, Bs, d, C, K, [0, Bs], rank=r, head_dim=hd)
    state = np.zeros((Bs, K - 1, C))
    for t in range(T):
        rows = np.arange(Bs) * T + t
        y, state = O.decode_step(step, u[rows], h[rows], A, BW, state)
        np.testing.assert_allclose(y, y_full[rows], rtol=0, atol=1e-12)
    for b in range(Bs):                      # the state holds the last K-1 inputs, newest first
        for j in range(K - 1):
            assert np.array_equal(state[b, j], u[b * T + T - 1 - j])


def test_decode_state_shift_is_exact_and_input_untouched():
    Bs, d, C, K, r = 2, 5, 6, 4, 2
    A, B = _params(O.LOWRANK, d, C, K, r, 0, 3)
    u = W.normal(3, "u", Bs * C).reshape(Bs, C)
    h = W.normal(3, "h", Bs * d).reshape(Bs, d)
    state = W.normal(3, "s", Bs * (K - 1) * C).reshape(Bs, K - 1, C)
    keep = state.copy()
    p = O.Problem(O.LOWRANK, Bs, d, C, K, [0, Bs], rank=r)
    y, new = O.decode_step(p, u, h, A, B, state)
    assert np.array_equal(state, keep)
    assert np.array_equal(new[:, 0], u) and np.array_equal(new[:, 1:], keep[:, :-1])
    # y against the definition written out with the oracle's own filters
    w = O.filters(O.Problem(O.LOWRANK, Bs, d, C, K, [0, 1, 2], rank=r), u, h, A, B)
    x = np.concatenate([u[:, None], keep], axis=1)           # x_j, j = 0 .. K-1
    ref = u + np.einsum("bcj,bjc->bc", w, x)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def test_decode_planted_mistake_is_caught():
    """A state rolled the wrong way round must fail the rollout pin."""
    Bs, T, d, C, K, r = 1, 5, 4, 4, 3, 2
    A, B = _params(O.LOWRANK, d, C, K, r, 0, 5)
    u = W.normal(5, "u", T * C).reshape(T, C)
    h = W.normal(5, "h", T * d).reshape(T, d)
    y_full, _, _ = O.forward(O.Problem(O.LOWRANK, T, d, C, K, [0, T], rank=r), u, h, A, B)
    step = O.Problem(O.LOWRANK, 1, d, C, K, [0, 1], rank=r)
    state = np.zeros((1, K - 1, C))
    worst = 0.0
    for t in range(T):
        y, state = O.decode_step(step, u[t:t + 1], h[t:t + 1], A, B, state)
        state = state[:, ::-1].copy()          # the planted mistake: oldest first
        worst = max(worst, float(np.max(np.abs(y - y_full[t:t + 1]))))
    assert worst > 1e-6
