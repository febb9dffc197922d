"""Pins for the oracle's backward pass (T = 1), CPU only.

The gradients of sum(O * dO) with respect to q, k and v are checked against
(i) central finite differences of the oracle's own forward pass, on untiled
and uneven tiled shapes, and (ii) the degenerate block sizes b1 = 1 and
b2 = 1, where the method equals dense softmax attention as a function, so
its gradient must equal dense attention's, written here in closed form.
"""
import numpy as np
import pytest
from scipy.special import softmax

from oracle import monarch_attention, monarch_attention_backward


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _fd_grads(q, k, v, dO, b1, b2, c1, c2, eps=1e-6):
    def f(qq, kk, vv):
        return (monarch_attention(qq, kk, vv, b1, b2, 1, c1, c2) * dO).sum()
    out = []
    for which in range(3):
        x = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(x[which])
        it = np.nditer(g, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[which][idx] += eps
            xm[which][idx] -= eps
            g[idx] = (f(*xp) - f(*xm)) / (2 * eps)
        out.append(g)
    return out


@pytest.mark.parametrize("b1,b2,c1,c2", [(3, 4, 1, 1), (3, 4, 2, 2), (5, 3, 2, 3), (4, 5, 3, 2)])
def test_backward_matches_finite_differences(b1, b2, c1, c2):
    N, d = b1 * b2, 3
    q, k, v, dO = (_rand((2, N, d), s) for s in (1, 2, 3, 4))
    dq, dk, dv = monarch_attention_backward(q, k, v, dO, b1, b2, c1, c2)
    fq, fk, fv = _fd_grads(q, k, v, dO, b1, b2, c1, c2)
    for got, ref in ((dq, fq), (dk, fk), (dv, fv)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=2e-7 * max(1.0, np.abs(ref).max()))


def _dense_grads(q, k, v, dO):
    """Gradients of sum(softmax(q k^T / sqrt(d)) v * dO), closed form."""
    sc = 1 / np.sqrt(q.shape[-1])
    P = softmax(sc * q @ np.swapaxes(k, -1, -2), axis=-1)
    dv = np.swapaxes(P, -1, -2) @ dO
    dP = dO @ np.swapaxes(v, -1, -2)
    dS = P * (dP - (P * dP).sum(-1, keepdims=True))
    return sc * dS @ k, sc * np.swapaxes(dS, -1, -2) @ q, dv


@pytest.mark.parametrize("b1,b2,c1,c2", [(1, 12, 1, 1), (1, 12, 1, 3), (12, 1, 1, 1),
                                         (12, 1, 4, 1), (4, 3, 4, 3)])
def test_degenerate_blocks_have_dense_attention_gradients(b1, b2, c1, c2):
    N, d = b1 * b2, 6
    q, k, v, dO = (_rand((3, N, d), s) for s in (5, 6, 7, 8))
    got = monarch_attention_backward(q, k, v, dO, b1, b2, c1, c2)
    for g, r in zip(got, _dense_grads(q, k, v, dO)):
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-12)


def test_backward_is_linear_in_dO():
    b1, b2, c1, c2, d = 4, 5, 2, 2, 4
    q, k, v, a, b = (_rand((1, b1 * b2, d), s) for s in (9, 10, 11, 12, 13))
    ga = monarch_attention_backward(q, k, v, a, b1, b2, c1, c2)
    gb = monarch_attention_backward(q, k, v, b, b1, b2, c1, c2)
    gab = monarch_attention_backward(q, k, v, 2 * a - b, b1, b2, c1, c2)
    for x, y, z in zip(ga, gb, gab):
        np.testing.assert_allclose(z, 2 * x - y, rtol=0, atol=1e-12)
