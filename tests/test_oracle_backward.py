"""Pins for the backward oracle (``oracle.backward``).

Each gradient is checked against something other than its own formula: the
adjoint identity with the independently pinned forward oracle, central
finite differences of the forward oracle (fp64, or exactly representable
fp32 logit steps), closed forms of silu', and the softmax's shift
invariance.  Planted mistakes (a dropped term of silu', a halved gradient,
a forgotten routing weight) must fail the same checks.
"""

import numpy as np
import pytest

import oracle
from oracle import backward as bw

E, K_TOP, H, I, T = 4, 2, 64, 64, 5


def _stack(seed):
    rng = np.random.default_rng(seed)
    w_gu = (rng.standard_normal((E, 2 * I, H)) * 0.1).astype(np.float32)
    w_d = (rng.standard_normal((E, H, I)) * 0.1).astype(np.float32)
    p_gu, a_gu = oracle.quantize_blockwise(w_gu)
    p_d, a_d = oracle.quantize_blockwise(w_d)
    return oracle.ExpertStack(p_gu, a_gu.reshape(E, -1), p_d, a_d.reshape(E, -1))


def _logits(rng, shape):
    # multiples of 2^-6 with top-k margins >= 2^-3, so that steps of 2^-12 are
    # exact in fp32 and never change the selection
    while True:
        lg = np.round(rng.standard_normal(shape) * 64) / 64
        s = np.sort(lg, axis=1)[:, ::-1]
        gaps = np.abs(np.diff(s, axis=1))
        if np.all(gaps >= 2 ** -3):
            return lg.astype(np.float32)


def test_grouped_gemm_t_is_the_adjoint_of_grouped_gemm():
    st = _stack(0)
    rng = np.random.default_rng(1)
    counts = [3, 0, 5, 1]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(off[-1])
    X = rng.standard_normal((M, H))
    G = rng.standard_normal((M, 2 * I))
    fwd = oracle.grouped_gemm(X, st.packed_gu, st.absmax_gu, off)
    back = bw.grouped_gemm_t(G, st.packed_gu, st.absmax_gu, off)
    assert back.shape == X.shape
    np.testing.assert_allclose(np.sum(G * fwd), np.sum(back * X), rtol=1e-12)
    # row by row as well: the identity holds per routed row
    np.testing.assert_allclose(np.sum(G * fwd, axis=1), np.sum(back * X, axis=1), rtol=1e-10,
                               atol=1e-12)


def _fd_dir(f, x, v, eps):
    return (f(x + eps * v) - f(x - eps * v)) / (2 * eps)


def test_swiglu_backward_matches_finite_differences():
    rng = np.random.default_rng(2)
    gu = rng.standard_normal((6, 2 * 16)) * 3
    dh = rng.standard_normal((6, 16))
    d = bw.swiglu_backward(gu, dh)
    for _ in range(4):
        v = rng.standard_normal(gu.shape)
        fd = _fd_dir(lambda z: np.sum(dh * oracle.swiglu(z)), gu, v, 1e-6)
        np.testing.assert_allclose(np.sum(d * v), fd, rtol=1e-7)


def test_silu_derivative_closed_forms():
    # d/dg [g sigmoid(g)] at g = 0 is 1/2; it tends to 1 for large g and 0 for
    # very negative g; its maximum is about 1.0998 near g = 2.3994
    g = np.array([[0.0, 40.0, -40.0, 2.399357280515]])
    d = bw.swiglu_backward(np.concatenate([g, np.ones_like(g)], axis=1), np.ones_like(g))
    dg = d[0, :4]
    np.testing.assert_allclose(dg[:3], [0.5, 1.0, 0.0], atol=1e-12)
    np.testing.assert_allclose(dg[3], 1.0998393194, rtol=1e-9)
    # du = silu(g): silu(0) = 0
    assert d[0, 4] == 0.0


def test_combine_backward_is_the_adjoint_and_dw_is_exact():
    rng = np.random.default_rng(3)
    idx = np.array([[0, 2], [1, 0], [3, 1]], dtype=np.int32)
    _, _, inv = oracle.permute_by_expert(idx, E)
    w = rng.random((3, 2))
    Yp = rng.standard_normal((6, H))
    dY = rng.standard_normal((3, H))
    dYp, dw = bw.combine_backward(dY, Yp, inv, w)
    V = rng.standard_normal(Yp.shape)
    np.testing.assert_allclose(np.sum(dY * oracle.unpermute_combine(V, inv, w)), np.sum(dYp * V),
                               rtol=1e-12)
    for t in range(3):
        for j in range(2):
            e = np.zeros_like(w)
            e[t, j] = 1.0
            # the combine is linear in w: the difference quotient is exact
            dq = np.sum(dY * (oracle.unpermute_combine(Yp, inv, w + e)
                              - oracle.unpermute_combine(Yp, inv, w)))
            np.testing.assert_allclose(dw[t, j], dq, rtol=1e-10)


@pytest.mark.parametrize("renorm", [True, False])
def test_route_backward_matches_exact_logit_steps(renorm):
    rng = np.random.default_rng(4 + renorm)
    lg = _logits(rng, (4, 6))
    idx, _ = oracle.route_topk(lg, 3, renorm)
    dw = rng.standard_normal((4, 3))
    dl = bw.route_backward(lg, idx, dw, renorm)
    h = np.float32(2 ** -12)
    for t in range(4):
        for i in range(6):
            up, dn = lg.copy(), lg.copy()
            up[t, i] += h
            dn[t, i] -= h
            iu, wu = oracle.route_topk(up, 3, renorm)
            idn, wd = oracle.route_topk(dn, 3, renorm)
            assert np.array_equal(iu, idx) and np.array_equal(idn, idx)
            fd = np.sum(dw[t] * (wu[t] - wd[t])) / (2 * float(h))
            np.testing.assert_allclose(dl[t, i], fd, rtol=1e-6, atol=1e-9)
    # shifting all logits of a token changes no weight: the gradient sums to 0
    np.testing.assert_allclose(dl.sum(axis=1), 0.0, atol=1e-12)
    if renorm:
        # only the selected logits receive gradient
        mask = np.zeros_like(dl, dtype=bool)
        np.put_along_axis(mask, idx.astype(np.int64), True, axis=1)
        assert np.all(dl[~mask] == 0.0)


@pytest.mark.parametrize("renorm", [True, False])
def test_layer_backward_matches_finite_differences(renorm):
    st = _stack(5)
    rng = np.random.default_rng(6)
    x = rng.standard_normal((T, H))
    lg = _logits(rng, (T, E))
    dY = rng.standard_normal((T, H))
    dx, dl = bw.moe_layer_backward(x, lg, st, K_TOP, renorm, dY)

    def loss_x(z):
        return np.sum(dY * oracle.moe_layer(z, lg, st, K_TOP, renorm))

    for _ in range(3):
        v = rng.standard_normal(x.shape)
        np.testing.assert_allclose(np.sum(dx * v), _fd_dir(loss_x, x, v, 1e-6), rtol=1e-6)
    h = np.float32(2 ** -12)
    for t, i in [(0, 0), (1, 3), (4, 2), (2, 1)]:
        up, dn = lg.copy(), lg.copy()
        up[t, i] += h
        dn[t, i] -= h
        fd = (np.sum(dY * oracle.moe_layer(x, up, st, K_TOP, renorm))
              - np.sum(dY * oracle.moe_layer(x, dn, st, K_TOP, renorm))) / (2 * float(h))
        np.testing.assert_allclose(dl[t, i], fd, rtol=1e-5, atol=1e-9)


def test_permuted_backward_equals_per_token_backward():
    st = _stack(7)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((T, H))
    lg = _logits(rng, (T, E))
    dY = rng.standard_normal((T, H))
    a = bw.moe_layer_backward(x, lg, st, K_TOP, True, dY)
    b = bw.moe_layer_backward_permuted(x, lg, st, K_TOP, True, dY)
    np.testing.assert_allclose(b[0], a[0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(b[1], a[1], rtol=1e-10, atol=1e-12)


def test_planted_mistakes_fail_the_finite_difference_check():
    rng = np.random.default_rng(9)
    gu = rng.standard_normal((4, 2 * 8)) * 2
    dh = rng.standard_normal((4, 8))
    v = rng.standard_normal(gu.shape)
    fd = _fd_dir(lambda z: np.sum(dh * oracle.swiglu(z)), gu, v, 1e-6)
    g, u = gu[:, :8], gu[:, 8:]
    s = 1 / (1 + np.exp(-g))
    # silu' without its g (1 - s) term
    wrong = np.concatenate([dh * u * s, dh * g * s], axis=1)
    assert abs(np.sum(wrong * v) - fd) > 1e-3 * abs(fd)
    # a gradient halved everywhere: invisible to any check of its direction
    # alone, caught by the finite difference
    half = 0.5 * bw.swiglu_backward(gu, dh)
    assert abs(np.sum(half * v) - fd) > 0.1 * abs(fd)
    # the combine adjoint without the routing weight
    idx = np.array([[0, 2], [1, 0]], dtype=np.int32)
    _, _, inv = oracle.permute_by_expert(idx, E)
    w = np.array([[0.7, 0.3], [0.6, 0.4]])
    Yp = rng.standard_normal((4, 8))
    dY = rng.standard_normal((2, 8))
    V = rng.standard_normal(Yp.shape)
    dYp_wrong = np.zeros_like(Yp)
    for t in range(2):
        for j in range(2):
            dYp_wrong[inv[t * 2 + j]] = dY[t]
    assert abs(np.sum(dY * oracle.unpermute_combine(V, inv, w)) - np.sum(dYp_wrong * V)) > 1e-3


def test_lora_backward_matches_finite_differences():
    rng = np.random.default_rng(10)
    Ee, N, Kk, r = 3, 12, 16, 4
    off = np.array([0, 2, 2, 5], dtype=np.int32)
    X = rng.standard_normal((5, Kk))
    A = rng.standard_normal((Ee, r, Kk))
    B = rng.standard_normal((Ee, N, r))
    G = rng.standard_normal((5, N))
    scale = 0.75
    dX, dA, dB = bw.lora_backward(X, off, A, B, scale, G)

    def loss(Xv, Av, Bv):
        return np.sum(G * oracle.lora_delta(Xv, off, Av, Bv, scale))

    for which, base, grad in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        v = rng.standard_normal(base.shape)
        args = {"X": X, "A": A, "B": B}

        def f(z, which=which):
            a = dict(args)
            a[which] = z
            return loss(a["X"], a["A"], a["B"])

        np.testing.assert_allclose(np.sum(grad * v), _fd_dir(f, base, v, 1e-6), rtol=1e-7,
                                   err_msg=which)
    # expert 1 has no rows: its adapters get no gradient
    assert not np.any(dA[1]) and not np.any(dB[1])
