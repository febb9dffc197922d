"""Pins for the oracle's padding (N_real < b1 * b2), CPU only.

Source: MonarchAttention OpenReview discussion, author response on choosing
the block sizes (m is the ceiling of N / b; ViT's N = 197 is pre-padded).
Reading: the objective is taken over the real tokens only.  Pad keys get zero
R weight, column groups without a real key get zero L weight, and pad query
rows are left out.  Each pin compares the oracle with something other than
itself: dense softmax attention over the real tokens, closed forms, the dense
objective over the real sub-matrix, and a generic optimiser.
"""
import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

from oracle import (
    LFactor,
    RFactor,
    dense_logits,
    group_valid,
    groups,
    l_update,
    materialise,
    monarch_attention,
    objective,
    objective_dense,
    r_update,
    token_mask,
)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def exact_attention(q, k, v):
    S = q @ np.swapaxes(k, -1, -2) / np.sqrt(q.shape[-1])
    return softmax(S, axis=-1) @ v


def test_token_mask_places_pads_first_or_last():
    m = token_mask(3, 4, 5, True)
    assert m.reshape(-1).tolist() == [False] * 5 + [True] * 7
    m = token_mask(3, 4, 5, False)
    assert m.reshape(-1).tolist() == [True] * 7 + [False] * 5
    assert token_mask(3, 4, 0).all()
    with pytest.raises(ValueError):
        token_mask(3, 4, 12)
    real = token_mask(4, 6, 8, True)              # chunk 0 all pad, chunk 1 keys 2..5 real
    assert group_valid(real, groups(6, 3)).tolist() == [[False] * 3, [False, True, True],
                                                         [True] * 3, [True] * 3]


@pytest.mark.parametrize("b1,b2,c1,c2,n_pad", [(1, 12, 1, 1, 3), (1, 12, 1, 3, 5),
                                               (12, 1, 1, 1, 4), (12, 1, 3, 1, 7),
                                               (4, 3, 4, 3, 5), (3, 5, 3, 5, 6)])
@pytest.mark.parametrize("pad_front", [True, False])
@pytest.mark.parametrize("T", [1, 2])
def test_padded_degenerate_blocks_are_dense_attention_over_real_tokens(b1, b2, c1, c2, n_pad,
                                                                       pad_front, T):
    n, d = b1 * b2 - n_pad, 8
    q, k, v = (_rand((2, n, d), s) for s in (1, 2, 3))
    O = monarch_attention(q, k, v, b1, b2, T, c1, c2, n_pad=n_pad, pad_front=pad_front)
    np.testing.assert_allclose(O, exact_attention(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("b1,b2,c1,c2,n_pad", [(5, 7, 1, 1, 3), (5, 7, 2, 3, 9), (4, 6, 2, 3, 7)])
@pytest.mark.parametrize("pad_front", [True, False])
@pytest.mark.parametrize("T", [1, 2])
def test_padded_zero_logits_give_the_mean_of_real_values(b1, b2, c1, c2, n_pad, pad_front, T):
    """q = 0: softmax over the real keys is uniform, which the method reaches at
    T >= 1; pad keys must carry no weight, and a group without real keys none."""
    n, d = b1 * b2 - n_pad, 4
    q = np.zeros((1, n, d))
    k, v = _rand((1, n, d), 1), _rand((1, n, d), 2)
    O = monarch_attention(q, k, v, b1, b2, T, c1, c2, n_pad=n_pad, pad_front=pad_front)
    np.testing.assert_allclose(O[0], np.broadcast_to(v[0].mean(0), O[0].shape), atol=1e-13)


@pytest.mark.parametrize("pad_front", [True, False])
def test_padded_T0_is_the_mean_over_valid_groups_of_real_key_means(pad_front):
    b1, b2, c2, n_pad, d = 4, 6, 3, 7, 5
    n = b1 * b2 - n_pad
    v = _rand((1, n, d), 3)
    q = k = _rand((1, n, d), 4)
    O = monarch_attention(q, k, v, b1, b2, 0, 1, c2, n_pad=n_pad, pad_front=pad_front)
    real = token_mask(b1, b2, n_pad, pad_front).reshape(-1)
    vp = np.zeros((b1 * b2, d))
    vp[real] = v[0]
    vp = vp.reshape(b1, b2, d)
    rm = real.reshape(b1, b2)
    means = [vp[kk, j0:j1][rm[kk, j0:j1]].mean(0) for kk in range(b1)
             for j0, j1 in groups(b2, c2) if rm[kk, j0:j1].any()]
    np.testing.assert_allclose(O[0], np.broadcast_to(np.mean(means, axis=0), (n, d)),
                               atol=1e-13)


def _real_submatrix(M, real):
    r = real.reshape(-1)
    return M[:, r][:, :, r], M[:, r][:, :, ~r]


@pytest.mark.parametrize("b1,b2,c1,c2,n_pad", [(4, 6, 1, 1, 5), (5, 4, 2, 2, 3), (6, 5, 3, 2, 8),
                                               (4, 6, 2, 3, 7)])
@pytest.mark.parametrize("pad_front", [True, False])
@pytest.mark.parametrize("T", [0, 1, 3])
def test_padded_M_is_row_stochastic_on_real_tokens_and_gives_the_output(b1, b2, c1, c2, n_pad,
                                                                        pad_front, T):
    n, d = b1 * b2 - n_pad, 6
    q, k, v = (_rand((2, n, d), s) * 2 for s in (7, 8, 9))
    O, st = monarch_attention(q, k, v, b1, b2, T, c1, c2, return_state=True, n_pad=n_pad,
                              pad_front=pad_front)
    M = materialise(st["L"], st["R"], st["rows"], st["cols"])
    Mr, Mpad = _real_submatrix(M, st["real"])
    assert Mr.min() >= 0
    assert np.abs(Mpad).max(initial=0) == 0
    np.testing.assert_allclose(Mr.sum(-1), 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Mr @ v, O, rtol=0, atol=1e-12)
    S = dense_logits(st["q"], st["k"])
    Sr, _ = _real_submatrix(S, st["real"])
    np.testing.assert_allclose(
        objective_dense(Mr, Sr),
        objective(st["q"], st["L"], st["R"], st["rows"], st["sc"], st["real"]),
        rtol=1e-12, atol=1e-10)


@pytest.mark.parametrize("b1,b2,c1,c2,n_pad", [(6, 6, 1, 1, 8), (8, 5, 2, 2, 11), (5, 8, 1, 3, 9)])
@pytest.mark.parametrize("pad_front", [True, False])
def test_padded_objective_monotone_with_exact_gap(b1, b2, c1, c2, n_pad, pad_front):
    """Each half-step raises f over the real tokens; f* - f is the KL divergence of
    M's real rows from softmax over the real keys."""
    n, d = b1 * b2 - n_pad, 8
    q, k, v = (_rand((3, n, d), s) * 1.5 for s in (11, 12, 13))
    _, st = monarch_attention(q, k, v, b1, b2, 0, c1, c2, return_state=True, n_pad=n_pad,
                              pad_front=pad_front)
    qh, kh, vh, real = st["q"], st["k"], st["v"], st["real"]
    rows, cols, sc = groups(b1, c1), groups(b2, c2), 1 / np.sqrt(d)
    L, rf = st["L"], st["R"]
    Sr, _ = _real_submatrix(dense_logits(qh, kh), real)
    fstar = logsumexp(Sr, axis=-1).sum(-1)
    trace = [objective(qh, L, rf, rows, sc, real)]
    for _ in range(4):
        rf = r_update(qh, kh, vh, L, rows, cols, sc, real)
        trace.append(objective(qh, L, rf, rows, sc, real))
        L = l_update(qh, rf, rows, cols, sc)
        trace.append(objective(qh, L, rf, rows, sc, real))
        Mr, _ = _real_submatrix(materialise(L, rf, rows, cols), real)
        P = softmax(Sr, axis=-1)
        with np.errstate(divide="ignore", invalid="ignore"):
            kl = np.where(Mr > 0, Mr * (np.log(Mr) - np.log(P)), 0.0).sum(axis=(1, 2))
        np.testing.assert_allclose(fstar - trace[-1], kl, rtol=1e-9, atol=1e-10)
    trace = np.array(trace)
    assert (np.diff(trace, axis=0) >= -1e-10).all()
    assert (trace <= fstar + 1e-10).all()


def test_padded_updates_beat_random_competitors():
    b1, b2, c1, c2, n_pad, d = 5, 6, 2, 2, 8, 4
    n = b1 * b2 - n_pad
    q, k, v = (_rand((1, n, d), s) * 2 for s in (21, 22, 23))
    _, st = monarch_attention(q, k, v, b1, b2, 1, c1, c2, return_state=True, n_pad=n_pad)
    qh, kh, vh, rows, cols, sc, real = (st[x] for x in ("q", "k", "v", "rows", "cols", "sc",
                                                         "real"))
    L = st["L"]
    rf_opt = r_update(qh, kh, vh, L, rows, cols, sc, real)
    f_opt = objective(qh, L, rf_opt, rows, sc, real)[0]
    rng = np.random.default_rng(0)
    for _ in range(20):   # competitors stay on the constraint set: zero on pad keys
        R = rf_opt.R * np.exp(0.3 * rng.standard_normal(rf_opt.R.shape))
        for j0, j1 in cols:
            z = R[..., j0:j1].sum(-1, keepdims=True)
            R[..., j0:j1] = np.where(z > 0, R[..., j0:j1] / np.where(z > 0, z, 1), 0)
        assert objective(qh, L, RFactor(R, kh, vh, cols, real), rows, sc, real)[0] < f_opt
    Lu = l_update(qh, rf_opt, rows, cols, sc)
    g_opt = objective(qh, Lu, rf_opt, rows, sc, real)[0]
    Larr = Lu.materialise()
    for _ in range(20):
        A = Larr * np.exp(0.3 * rng.standard_normal(Larr.shape))
        A /= A.sum(axis=(-1, -2), keepdims=True)
        Lc = LFactor.explicit(A, rows, cols, valid=rf_opt.valid)
        assert objective(qh, Lc, rf_opt, rows, sc, real)[0] < g_opt


def _brute_force_padded(q, k, v, b1, b2, T, c1, c2, real):
    """Alternating maximisation of the dense objective over the real tokens by
    LBFGS, with M built entry by entry on the padded grid: L a softmax over the
    pairs (k, q) holding a real key, R a softmax over the real keys of each
    column group, f summed over real rows and columns."""
    N = b1 * b2
    r = torch.tensor(real.reshape(-1))
    qp = torch.zeros(N, q.shape[-1], dtype=torch.float64)
    kp = torch.zeros_like(qp)
    qp[r], kp[r] = torch.tensor(q), torch.tensor(k)
    S = (qp @ kp.T / q.shape[-1] ** 0.5)[r][:, r]
    prow = np.concatenate([[g] * len(a) for g, a in enumerate(np.array_split(np.arange(b1), c1))])
    qcol = np.concatenate([[g] * len(a) for g, a in enumerate(np.array_split(np.arange(b2), c2))])
    kreal = torch.tensor(real)                                            # (k, j)
    valid = torch.stack([kreal[:, torch.tensor(qcol == g)].any(1) for g in range(c2)], 1)
    neg = torch.tensor(-1e300, dtype=torch.float64)

    def L_of(th):
        th = torch.where(valid.reshape(-1), th, neg)
        return torch.softmax(th, dim=-1).reshape(b2, b1, b1, c2)

    def R_of(th):
        out = torch.zeros_like(th)
        for g in range(c2):
            m = torch.tensor(qcol == g)
            t = torch.where(kreal[:, m][:, None, None, :], th[..., m], neg)
            out[..., m] = torch.where(valid[:, g][:, None, None, None], torch.softmax(t, -1), 0.0)
        return out

    l_, i_, k_, j_ = (torch.tensor(a.reshape(-1)) for a in
                      np.meshgrid(np.arange(b1), np.arange(b2), np.arange(b1), np.arange(b2),
                                  indexing="ij"))
    p_, q_ = torch.tensor(prow)[l_], torch.tensor(qcol)[j_]

    def M_of(thL, thR):
        L, R = L_of(thL), R_of(thR)
        return (L[i_, l_, k_, q_] * R[k_, p_, i_, j_]).reshape(N, N)[r][:, r]

    def f_of(M):
        return (M * S).sum() - torch.special.xlogy(M, M).sum()

    def argmax(th, other, which):
        th = th.clone().requires_grad_(True)
        opt = torch.optim.LBFGS([th], lr=1, max_iter=500, tolerance_grad=1e-13,
                                tolerance_change=1e-15, line_search_fn="strong_wolfe")

        def closure():
            opt.zero_grad()
            loss = -f_of(M_of(th, other) if which == "L" else M_of(other, th))
            loss.backward()
            return loss
        for _ in range(6):
            opt.step(closure)
        return th.detach()

    thL = torch.zeros(b2, b1, b1 * c2, dtype=torch.float64)
    thR = torch.zeros(b1, c1, b2, b2, dtype=torch.float64)
    for _ in range(T):
        thR = argmax(thR, thL, "R")
        thL = argmax(thL, thR, "L")
    with torch.no_grad():
        return (M_of(thL, thR) @ torch.tensor(v)).numpy()


@pytest.mark.parametrize("b1,b2,c1,c2,n_pad,pad_front,T", [(2, 3, 1, 1, 2, True, 1),
                                                           (3, 3, 1, 1, 4, False, 2),
                                                           (3, 3, 2, 2, 3, True, 2),
                                                           (3, 4, 1, 2, 5, True, 1)])
def test_padded_matches_brute_force_alternating_maximisation(b1, b2, c1, c2, n_pad, pad_front, T):
    n, d = b1 * b2 - n_pad, 2
    q, k, v = (_rand((n, d), s) * 1.5 for s in (31, 32, 33))
    O = monarch_attention(q, k, v, b1, b2, T, c1, c2, n_pad=n_pad, pad_front=pad_front)
    Ob = _brute_force_padded(q, k, v, b1, b2, T, c1, c2, token_mask(b1, b2, n_pad, pad_front))
    np.testing.assert_allclose(O, Ob, rtol=0, atol=2e-6)


def test_vit_197_prepadded_is_finite_and_differs_from_zero_filled_tokens():
    """ViT's 197 tokens in 15 x 14 blocks with 13 pad tokens in front.  Masking
    matters: feeding zero vectors as if they were real tokens gives another result."""
    n, d = 197, 16
    q, k, v = (_rand((1, n, d), s) for s in (51, 52, 53))
    O = monarch_attention(q, k, v, 15, 14, 3, n_pad=13, pad_front=True)
    assert O.shape == (1, n, d) and np.isfinite(O).all()
    z = np.zeros((1, 13, d))
    Oz = monarch_attention(np.concatenate([z, q], 1), np.concatenate([z, k], 1),
                           np.concatenate([z, v], 1), 15, 14, 3)[:, 13:]
    assert np.abs(O - Oz).max() > 1e-3
