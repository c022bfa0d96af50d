"""Pins for the fp64 oracle: each check ties the oracle to something other than
itself -- a closed form, an invariant the method must have, a brute force or
library routine, or a hand-derived example.

Source for what the method computes: "Dynamic Short Convolutions Improve
Transformers", gist.science technical summary, section "Dynamic Short
Convolutions" (Mechanism formula, the low-rank and head-wise Parameterization,
the residual Placement) and "Key Contributions" (the primitive generalizes
static short convolutions).
"""
import math

import numpy as np
import pytest

from oracle import oracle as O

RNG = np.random.default_rng(12345)


def _lowrank_problem(N, d, C, K, r, cu=None):
    cu = [0, N] if cu is None else cu
    return O.Problem(O.LOWRANK, N, d, C, K, cu, rank=r)


def _rand_lowrank(N, d, C, K, r, rng=RNG):
    return dict(u=rng.standard_normal((N, C)), h=rng.standard_normal((N, d)),
                A=rng.standard_normal((d, r)), B=rng.standard_normal((r, C * K)),
                g=rng.standard_normal((N, C)))


def _loss_and_grads(p, x):
    """L = <g, y> and its gradients from the oracle (all inputs)."""
    BW = x["B"] if p.kind == O.LOWRANK else x["W"]
    A = x.get("A")
    y, _, _ = O.forward(p, x["u"], x["h"], A, BW)
    du, _, dh = O.backward_rows(p, x["g"], x["u"], x["h"], A, BW)
    dA, dBW = O.param_grads(p, x["g"], x["u"], x["h"], A, BW)
    return float(np.sum(x["g"] * y)), dict(u=du, h=dh, A=dA, B=dBW) if p.kind == O.LOWRANK \
        else dict(u=du, h=dh, W=dBW)


# 1. Hand-derived example (integers, exact in fp64).  Derivation:
#    h = [[1,0],[0,1],[1,1]], A = [[2],[1]]  ->  z = [2, 1, 3]
#    B = [[1,-1,0,2]] (column c*K+j)         ->  w[n] = z[n] * B
#    u = [[1,2],[3,-1],[0,5]], K = 2, one sequence of 3 tokens
#    y[0] = (1 + 2*1,  2 + 0*2)                      = (3, 2)
#    y[1] = (3 + 1*3 - 1*1,  -1 + 0*(-1) + 2*2)       = (5, 3)
#    y[2] = (0 + 3*0 - 3*3,  5 + 0*5 + 6*(-1))        = (-9, -1)
#    g = [[1,0],[0,1],[1,-1]]
#    dw[n,c,j] = g[n,c] u[n-j,c]: n0 (1,0 | 0,0), n1 (0,0 | -1,2), n2 (0,3 | -5,1)
#    du[0] = (1 + 2*1 + (-1)*0,  0 + 0 + 2*1)         = (3, 2)
#    du[1] = (0 + 1*0 + (-3)*1,  1 + 0 + 6*(-1))       = (-3, -5)
#    du[2] = (1 + 3*1,  -1 + 0*(-1))                   = (4, -1)
#    dz = dw . B = (1, 4, -1); dB = sum_n z[n] dw[n] = (2, 9, -16, 5)
#    dA = h^T dz = (0, 3); dh = dz A^T = ((2,1),(8,4),(-2,-1))
def test_hand_worked_lowrank_example():
    p = _lowrank_problem(3, 2, 2, 2, 1)
    h = np.array([[1., 0.], [0., 1.], [1., 1.]])
    A = np.array([[2.], [1.]])
    B = np.array([[1., -1., 0., 2.]])
    u = np.array([[1., 2.], [3., -1.], [0., 5.]])
    g = np.array([[1., 0.], [0., 1.], [1., -1.]])
    y, z, _ = O.forward(p, u, h, A, B)
    assert np.array_equal(z[:, 0], [2., 1., 3.])
    assert np.array_equal(y, [[3., 2.], [5., 3.], [-9., -1.]])
    du, dz, dh = O.backward_rows(p, g, u, h, A, B)
    assert np.array_equal(du, [[3., 2.], [-3., -5.], [4., -1.]])
    assert np.array_equal(dz[:, 0], [1., 4., -1.])
    assert np.array_equal(dh, [[2., 1.], [8., 4.], [-2., -1.]])
    dA, dB = O.param_grads(p, g, u, h, A, B)
    assert np.array_equal(dA[:, 0], [0., 3.])
    assert np.array_equal(dB[0], [2., 9., -16., 5.])


# 2. Constant filter => static depthwise causal conv ("generalizes static short
#    convolutions"): with h[n,:] = h0 for every token the filter is constant, and
#    y - u must equal a per-channel np.convolve restricted to each sequence.
@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_constant_filter_is_static_conv(K):
    N, d, C, r = 23, 5, 6, 3
    cu = [0, 9, 23]
    p = _lowrank_problem(N, d, C, K, r, cu)
    x = _rand_lowrank(N, d, C, K, r)
    h = np.tile(RNG.standard_normal(d), (N, 1))
    w0 = O.filters(p, x["u"], h, x["A"], x["B"], rows=[0])[0]        # [C, K]
    wall = O.filters(p, x["u"], h, x["A"], x["B"])
    assert np.array_equal(wall, np.broadcast_to(w0, wall.shape))
    y, _, _ = O.forward(p, x["u"], h, x["A"], x["B"])
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        for c in range(C):
            static = np.convolve(x["u"][a:b, c], w0[c, :])[: b - a]
            np.testing.assert_allclose(y[a:b, c] - x["u"][a:b, c], static, rtol=1e-13, atol=1e-13)


# 3. Zero filter => identity (the residual alone), bitwise.
def test_zero_filter_is_identity():
    N, d, C, K, r = 17, 4, 5, 3, 2
    p = _lowrank_problem(N, d, C, K, r, [0, 6, 17])
    x = _rand_lowrank(N, d, C, K, r)
    B0 = np.zeros_like(x["B"])
    y, _, _ = O.forward(p, x["u"], x["h"], x["A"], B0)
    assert np.array_equal(y, x["u"])
    du, dz, dh = O.backward_rows(p, x["g"], x["u"], x["h"], x["A"], B0)
    assert np.array_equal(du, x["g"])
    assert not np.any(dz) and not np.any(dh)
    dA, _ = O.param_grads(p, x["g"], x["u"], x["h"], x["A"], B0)
    assert not np.any(dA)
    h0 = np.zeros_like(x["h"])                    # zero hidden state: z = 0, w = 0
    y, _, _ = O.forward(p, x["u"], h0, x["A"], x["B"])
    assert np.array_equal(y, x["u"])
    dA, dB = O.param_grads(p, x["g"], x["u"], h0, x["A"], x["B"])
    assert not np.any(dA) and not np.any(dB)


# 4. Causality: perturbing token t* (its u and h) leaves every earlier output
#    bitwise unchanged, and changes y[t*].
@pytest.mark.parametrize("kind", [O.LOWRANK, O.HEADWISE])
def test_causality(kind):
    N, d, C, K = 20, 4, 8, 4
    if kind == O.LOWRANK:
        p = _lowrank_problem(N, d, C, K, 3)
        x = _rand_lowrank(N, d, C, K, 3)
        BW, A = x["B"], x["A"]
    else:
        p = O.Problem(O.HEADWISE, N, d, C, K, [0, N], head_dim=4)
        x = _rand_lowrank(N, d, C, K, 1)
        BW, A = RNG.standard_normal((d, 2 * K)), None
    y0, _, _ = O.forward(p, x["u"], x["h"], A, BW)
    for t in (0, 7, N - 1):
        u1, h1 = x["u"].copy(), x["h"].copy()
        u1[t] += RNG.standard_normal(C)
        h1[t] += RNG.standard_normal(d)
        y1, _, _ = O.forward(p, u1, h1, A, BW)
        assert np.array_equal(y1[:t], y0[:t])
        assert not np.array_equal(y1[t], y0[t])


# 5. Document isolation: a packed run equals independent runs per document
#    (bitwise for per-token outputs; parameter gradients are sums over documents).
@pytest.mark.parametrize("kind", [O.LOWRANK, O.HEADWISE])
def test_document_isolation(kind):
    lens = [1, 2, 5, 3, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    N, d, C, K = int(cu[-1]), 3, 8, 3
    x = _rand_lowrank(N, d, C, K, 2)
    if kind == O.LOWRANK:
        mk = lambda n, c: _lowrank_problem(n, d, C, K, 2, c)
        A, BW = x["A"], x["B"]
    else:
        mk = lambda n, c: O.Problem(O.HEADWISE, n, d, C, K, c, head_dim=2)
        A, BW = None, RNG.standard_normal((d, 4 * K))
    p = mk(N, cu)
    y, _, _ = O.forward(p, x["u"], x["h"], A, BW)
    du, dg, dh = O.backward_rows(p, x["g"], x["u"], x["h"], A, BW)
    dA, dBW = O.param_grads(p, x["g"], x["u"], x["h"], A, BW)
    sA, sBW = 0.0, 0.0
    for s in range(len(lens)):
        a, b = int(cu[s]), int(cu[s + 1])
        q = mk(b - a, [0, b - a])
        sl = lambda k: x[k][a:b]
        ys, _, _ = O.forward(q, sl("u"), sl("h"), A, BW)
        dus, dgs, dhs = O.backward_rows(q, sl("g"), sl("u"), sl("h"), A, BW)
        assert np.array_equal(ys, y[a:b])
        assert np.array_equal(dus, du[a:b]) and np.array_equal(dgs, dg[a:b]) and np.array_equal(dhs, dh[a:b])
        dAs, dBWs = O.param_grads(q, sl("g"), sl("u"), sl("h"), A, BW)
        sBW = sBW + dBWs
        if dAs is not None:
            sA = sA + dAs
    np.testing.assert_allclose(dBW, sBW, rtol=1e-12, atol=1e-12)
    if dA is not None:
        np.testing.assert_allclose(dA, sA, rtol=1e-12, atol=1e-12)
    # perturbing document 2 changes nothing outside it
    u1 = x["u"].copy()
    u1[cu[2]:cu[3]] += 1.0
    y1, _, _ = O.forward(p, u1, x["h"], A, BW)
    outside = np.r_[0:cu[2], cu[3]:N]
    assert np.array_equal(y1[outside], y[outside])


# 6. Central finite differences in fp64.  L = <g, y> is a polynomial of degree
#    <= 2 in every single input entry, so the central difference is exact up to
#    rounding; every gradient entry must agree to 1e-7 (relative to the largest).
@pytest.mark.parametrize("kind", [O.LOWRANK, O.HEADWISE])
def test_finite_differences(kind):
    N, d, C, K = 7, 3, 4, 3
    cu = [0, 3, 7]                                # includes a document boundary
    x = _rand_lowrank(N, d, C, K, 2)
    if kind == O.LOWRANK:
        p = _lowrank_problem(N, d, C, K, 2, cu)
        names = ["u", "h", "A", "B"]
    else:
        p = O.Problem(O.HEADWISE, N, d, C, K, cu, head_dim=2)
        x["W"] = RNG.standard_normal((d, 2 * K))
        del x["A"], x["B"]
        names = ["u", "h", "W"]
    _, grads = _loss_and_grads(p, x)
    eps = 1e-6
    for nm in names:
        fd = np.zeros_like(x[nm])
        for idx in np.ndindex(*x[nm].shape):
            xp = {k: v.copy() for k, v in x.items()}
            xm = {k: v.copy() for k, v in x.items()}
            xp[nm][idx] += eps
            xm[nm][idx] -= eps
            fd[idx] = (_loss_and_grads(p, xp)[0] - _loss_and_grads(p, xm)[0]) / (2 * eps)
        scale = max(1.0, np.abs(fd).max())
        assert np.abs(fd - grads[nm]).max() / scale <= 1e-7, nm


# 7. Adjoint identity <g, J d> = <J^T g, d> for a random direction d over all
#    inputs at once.  y(x + t d) is a polynomial of degree <= 4 in t, so the
#    five-point stencil gives J d exactly up to rounding.
def test_adjoint_identity():
    N, d, C, K, r = 11, 4, 6, 4, 3
    p = _lowrank_problem(N, d, C, K, r, [0, 5, 11])
    x = _rand_lowrank(N, d, C, K, r)
    dirn = {k: RNG.standard_normal(x[k].shape) for k in ("u", "h", "A", "B")}

    def y_at(t):
        return O.forward(p, x["u"] + t * dirn["u"], x["h"] + t * dirn["h"], x["A"] + t * dirn["A"],
                         x["B"] + t * dirn["B"])[0]

    Jd = (y_at(-2.0) - 8.0 * y_at(-1.0) + 8.0 * y_at(1.0) - y_at(2.0)) / 12.0
    lhs = float(np.sum(x["g"] * Jd))
    _, gr = _loss_and_grads(p, x)
    rhs = sum(float(np.sum(gr[k] * dirn[k])) for k in ("u", "h", "A", "B"))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


# 8. Head-wise is the low-rank form with A = W (r = H*K) and the fixed expansion
#    B = E, E[(q,j'), c*K+j] = [q == c // head_dim][j == j'].  The two oracle
#    paths share no generator code, so this cross-checks both.
def test_headwise_equals_lowrank_with_expansion():
    N, d, hd, H, K = 13, 5, 3, 4, 3
    C = hd * H
    cu = [0, 4, 13]
    x = _rand_lowrank(N, d, C, K, 1)
    W = RNG.standard_normal((d, H * K))
    E = np.zeros((H * K, C * K))
    for q in range(H):
        for j in range(K):
            for c in range(q * hd, (q + 1) * hd):
                E[q * K + j, c * K + j] = 1.0
    ph = O.Problem(O.HEADWISE, N, d, C, K, cu, head_dim=hd)
    pl = O.Problem(O.LOWRANK, N, d, C, K, cu, rank=H * K)
    yh, _, _ = O.forward(ph, x["u"], x["h"], None, W)
    yl, _, _ = O.forward(pl, x["u"], x["h"], W, E)
    np.testing.assert_allclose(yh, yl, rtol=1e-12, atol=1e-12)
    duh, dwh, dhh = O.backward_rows(ph, x["g"], x["u"], x["h"], None, W)
    dul, dzl, dhl = O.backward_rows(pl, x["g"], x["u"], x["h"], W, E)
    np.testing.assert_allclose(duh, dul, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dwh, dzl, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dhh, dhl, rtol=1e-12, atol=1e-12)
    _, dW = O.param_grads(ph, x["g"], x["u"], x["h"], None, W)
    dA, _ = O.param_grads(pl, x["g"], x["u"], x["h"], W, E)
    np.testing.assert_allclose(dW, dA, rtol=1e-12, atol=1e-12)


# 9. K = 1 closed form: y = u * (1 + w[:, :, 0]) elementwise, with the filter the
#    plain two-matrix product h A B; and y is linear in u for a fixed h.
def test_k1_closed_form_and_linearity():
    N, d, C, r = 9, 4, 5, 2
    p = _lowrank_problem(N, d, C, 1, r, [0, 2, 9])
    x = _rand_lowrank(N, d, C, 1, r)
    w = x["h"] @ x["A"] @ x["B"]                  # [N, C] for K = 1
    y, _, _ = O.forward(p, x["u"], x["h"], x["A"], x["B"])
    np.testing.assert_allclose(y, x["u"] * (1.0 + w), rtol=1e-13, atol=1e-13)
    p3 = _lowrank_problem(N, d, C, 3, r, [0, 2, 9])
    x3 = _rand_lowrank(N, d, C, 3, r)
    u2 = RNG.standard_normal((N, C))
    ya, _, _ = O.forward(p3, x3["u"], x3["h"], x3["A"], x3["B"])
    yb, _, _ = O.forward(p3, u2, x3["h"], x3["A"], x3["B"])
    yab, _, _ = O.forward(p3, 2.0 * x3["u"] - 3.0 * u2, x3["h"], x3["A"], x3["B"])
    np.testing.assert_allclose(yab, 2.0 * ya - 3.0 * yb, rtol=1e-12, atol=1e-12)


# 10. Independent restatement in PyTorch fp64 (autograd on an explicit [N,C,K]
#     filter tensor built with einsum, taps gathered with a padded shift per
#     sequence): forward and every gradient agree to 1e-12.
@pytest.mark.parametrize("kind", [O.LOWRANK, O.HEADWISE])
def test_torch_autograd_restatement(kind):
    torch = pytest.importorskip("torch")
    N, d, C, K, hd = 12, 5, 6, 3, 3
    cu = [0, 1, 5, 12]
    x = _rand_lowrank(N, d, C, K, 4)
    if kind == O.LOWRANK:
        p = _lowrank_problem(N, d, C, K, 4, cu)
        A, BW = x["A"], x["B"]
    else:
        p = O.Problem(O.HEADWISE, N, d, C, K, cu, head_dim=hd)
        A, BW = None, RNG.standard_normal((d, (C // hd) * K))
    T = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True)
         for k, v in dict(u=x["u"], h=x["h"], BW=BW).items()}
    if A is not None:
        T["A"] = torch.tensor(A, dtype=torch.float64, requires_grad=True)
        wt = torch.einsum("nr,rck->nck", T["h"] @ T["A"], T["BW"].reshape(-1, C, K))
    else:
        wh = torch.einsum("nd,dqk->nqk", T["h"], T["BW"].reshape(d, C // hd, K))
        wt = wh.repeat_interleave(hd, dim=1)
    outs = []
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        useg = torch.nn.functional.pad(T["u"][a:b], (0, 0, K - 1, 0))    # K-1 zero rows in front
        taps = torch.stack([useg[K - 1 - j: K - 1 - j + (b - a)] for j in range(K)], dim=-1)
        outs.append(T["u"][a:b] + (wt[a:b] * taps).sum(-1))
    y = torch.cat(outs)
    g = torch.tensor(x["g"])
    (y * g).sum().backward()
    yo, _, _ = O.forward(p, x["u"], x["h"], A, BW)
    np.testing.assert_allclose(yo, y.detach().numpy(), rtol=1e-12, atol=1e-12)
    du, _, dh = O.backward_rows(p, x["g"], x["u"], x["h"], A, BW)
    dA, dBW = O.param_grads(p, x["g"], x["u"], x["h"], A, BW)
    np.testing.assert_allclose(du, T["u"].grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dh, T["h"].grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dBW, T["BW"].grad.numpy(), rtol=1e-12, atol=1e-12)
    if A is not None:
        np.testing.assert_allclose(dA, T["A"].grad.numpy(), rtol=1e-12, atol=1e-12)


# 11. Sampled entries agree with the full reductions (they are what the
#     full-size GPU tests compare against).
def test_sampled_entries_match_full():
    N, d, C, K, r = 15, 4, 6, 3, 3
    p = _lowrank_problem(N, d, C, K, r, [0, 7, 15])
    x = _rand_lowrank(N, d, C, K, r)
    dA, dB = O.param_grads(p, x["g"], x["u"], x["h"], x["A"], x["B"])
    ia, ka = [0, 3, 2], [2, 0, 1]
    np.testing.assert_allclose(O.param_grad_entries(p, x["g"], x["u"], x["h"], x["A"], x["B"], "dA", ia, ka),
                               dA[ia, ka], rtol=1e-12)
    kb, cb = [0, 2, 1], [17, 0, 5]
    np.testing.assert_allclose(O.param_grad_entries(p, x["g"], x["u"], x["h"], x["A"], x["B"], "dB", kb, cb),
                               dB[kb, cb], rtol=1e-12)
    rows = [14, 0, 6, 7]
    y, z, _ = O.forward(p, x["u"], x["h"], x["A"], x["B"])
    ys, zs, _ = O.forward(p, x["u"], x["h"], x["A"], x["B"], rows=rows)
    assert np.array_equal(ys, y[rows]) and np.array_equal(zs, z[rows])
    du, dz, dh = O.backward_rows(p, x["g"], x["u"], x["h"], x["A"], x["B"])
    dus, dzs, dhs = O.backward_rows(p, x["g"], x["u"], x["h"], x["A"], x["B"], rows=rows)
    assert np.array_equal(dus, du[rows]) and np.array_equal(dzs, dz[rows]) and np.array_equal(dhs, dh[rows])
    hd, H = 2, 3
    W = RNG.standard_normal((d, H * K))
    ph = O.Problem(O.HEADWISE, N, d, C, K, [0, 7, 15], head_dim=hd)
    _, dW = O.param_grads(ph, x["g"], x["u"], x["h"], None, W)
    np.testing.assert_allclose(O.param_grad_entries(ph, x["g"], x["u"], x["h"], None, W, "dW", [1, 3], [8, 0]),
                               dW[[1, 3], [8, 0]], rtol=1e-12)


# 12. A planted mistake is caught: an oracle variant that drops the j = 0 tap
#     (emulated here by subtracting its contribution) fails the static-conv pin.
def test_planted_mistake_is_caught():
    N, d, C, K, r = 10, 3, 4, 3, 2
    p = _lowrank_problem(N, d, C, K, r)
    x = _rand_lowrank(N, d, C, K, r)
    h = np.tile(RNG.standard_normal(d), (N, 1))
    w0 = O.filters(p, x["u"], h, x["A"], x["B"], rows=[0])[0]
    y, _, _ = O.forward(p, x["u"], h, x["A"], x["B"])
    y_bad = y - w0[None, :, 0] * x["u"]
    static = np.stack([np.convolve(x["u"][:, c], w0[c])[:N] for c in range(C)], axis=1)
    assert np.allclose(y - x["u"], static, rtol=1e-13, atol=1e-13)
    assert not np.allclose(y_bad - x["u"], static, rtol=1e-6, atol=1e-6)
