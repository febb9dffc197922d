"""Pins for the float64 oracle: every check here compares it with something
other than itself (dense softmax attention, closed forms, invariants, a brute
force optimiser over the pages' objective).  CPU only.

Sources: MonarchAttention (AI summary "Approach"; OpenReview discussion:
eq. (6) objective, concavity of each sub-problem, positivity of L and R,
block-size choice "b = 1 or N gives back dense"); MonarchRT summary ("Key
claims": six aligned block sizes, misaligned splits collapse, tiled Monarch
strictly contains untiled; "Method" (1)-(2)).
"""
import itertools

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

from oracle import (
    LFactor,
    RFactor,
    dense_logits,
    groups,
    l_update,
    materialise,
    monarch_attention,
    objective,
    objective_dense,
    r_update,
)
from oracle.monarch_ref import as_heads
from structured_sub_quadratic_b200.inputs import video_qkv


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def exact_attention(q, k, v):
    """Textbook softmax(q k^T / sqrt(d)) v, float64."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    S = q @ np.swapaxes(k, -1, -2) / np.sqrt(q.shape[-1])
    return softmax(S, axis=-1) @ v


def _state(q, k, v, b1, b2, T, c1, c2):
    return monarch_attention(q, k, v, b1, b2, T, c1, c2, return_state=True)


# --------------------------------------------------------------------------
# grouping reading (uneven split, larger first)
# --------------------------------------------------------------------------
def test_groups_uneven_split():
    assert groups(945, 2) == [(0, 473), (473, 945)]
    assert groups(80, 2) == [(0, 40), (40, 80)]
    assert groups(7, 3) == [(0, 3), (3, 5), (5, 7)]
    for n, c in [(10, 1), (10, 10), (13, 4)]:
        g = groups(n, c)
        sizes = [b - a for a, b in g]
        assert sum(sizes) == n and max(sizes) - min(sizes) <= 1
        assert sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        groups(4, 5)


# --------------------------------------------------------------------------
# P1: degenerate block sizes give dense softmax attention
# --------------------------------------------------------------------------
@pytest.mark.parametrize("b1,b2,c1,c2", [(1, 12, 1, 1), (12, 1, 1, 1), (1, 12, 1, 3),
                                         (4, 3, 4, 3), (3, 5, 3, 5)])
@pytest.mark.parametrize("T", [1, 2])
def test_degenerate_blocks_are_exact(b1, b2, c1, c2, T):
    N, d = b1 * b2, 8
    q, k, v = (_rand((2, N, d), s) for s in (1, 2, 3))
    O = monarch_attention(q, k, v, b1, b2, T, c1, c2)
    np.testing.assert_allclose(O, exact_attention(q, k, v), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# P2 / P3: separable positional logits; aligned vs misaligned block sizes
# --------------------------------------------------------------------------
def _aligned_perms(f, h, w):
    """The six aligned (b1, b2) layouts as token permutations of (f,h,w)."""
    idx = np.arange(f * h * w).reshape(f, h, w)
    out = {}
    for name, axes, b1 in [("(fh,w)", (0, 1, 2), f * h), ("(w,fh)", (2, 0, 1), w),
                           ("(f,hw)", (0, 1, 2), f), ("(hw,f)", (1, 2, 0), h * w),
                           ("(fw,h)", (0, 2, 1), f * w), ("(h,fw)", (1, 0, 2), h)]:
        out[name] = (idx.transpose(axes).reshape(-1), b1)
    return out


@pytest.mark.parametrize("latent", [(2, 3, 4), (3, 4, 5), (2, 5, 6)])
def test_separable_logits_exact_for_all_six_aligned_layouts(latent):
    f, h, w = latent
    N = f * h * w
    q, k, v = (x.double().numpy() for x in video_qkv(1, 2, latent, 32, torch.float32,
                                                      seed=5, noise=False))
    E = exact_attention(q, k, v)
    for name, (perm, b1) in _aligned_perms(f, h, w).items():
        O = monarch_attention(q[..., perm, :], k[..., perm, :], v[..., perm, :], b1, N // b1, 1)
        np.testing.assert_allclose(O, E[..., perm, :], rtol=0, atol=1e-12, err_msg=name)


@pytest.mark.parametrize("latent,mis", [((3, 6, 8), (12, 12)), ((2, 5, 6), (15, 4))])
def test_misaligned_split_does_not_converge(latent, mis):
    f, h, w = latent
    q, k, v = (x.double().numpy() for x in video_qkv(1, 1, latent, 32, torch.float32,
                                                      seed=0, noise=False))
    E = exact_attention(q, k, v)
    for T in (1, 2, 3):
        Oa = monarch_attention(q, k, v, f * h, w, T)
        Om = monarch_attention(q, k, v, mis[0], mis[1], T)
        rel_a = np.linalg.norm(Oa - E) / np.linalg.norm(E)
        rel_m = np.linalg.norm(Om - E) / np.linalg.norm(E)
        assert rel_a < 1e-12
        assert rel_m > 0.1


# --------------------------------------------------------------------------
# P4 / P8: M is nonnegative, row-stochastic, and M V equals the output
# --------------------------------------------------------------------------
@pytest.mark.parametrize("b1,b2,c1,c2", [(4, 6, 1, 1), (5, 4, 2, 2), (6, 5, 3, 2), (7, 3, 2, 3)])
@pytest.mark.parametrize("T", [0, 1, 3])
def test_row_stochastic_and_output_equals_MV(b1, b2, c1, c2, T):
    N, d = b1 * b2, 6
    q, k, v = (_rand((2, N, d), s) * 2 for s in (7, 8, 9))
    O, st = _state(q, k, v, b1, b2, T, c1, c2)
    M = materialise(st["L"], st["R"], st["rows"], st["cols"])
    assert M.min() >= 0
    np.testing.assert_allclose(M.sum(-1), 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(M @ v.reshape(2, N, d), O, rtol=0, atol=1e-12)
    S = dense_logits(st["q"], st["k"])
    np.testing.assert_allclose(objective_dense(M, S),
                               objective(st["q"], st["L"], st["R"], st["rows"], st["sc"]),
                               rtol=1e-12, atol=1e-10)


def test_block_rank_one_structure():
    """Untiled: every (i,k) block over (l, j) is rank one; tiled: every sub-tile is."""
    b1, b2, d = 6, 5, 4
    q, k, v = (_rand((1, b1 * b2, d), s) for s in (1, 2, 3))
    for c1, c2 in [(1, 1), (2, 2), (3, 2)]:
        _, st = _state(q, k, v, b1, b2, 2, c1, c2)
        M = materialise(st["L"], st["R"], st["rows"], st["cols"])[0].reshape(b1, b2, b1, b2)
        for i, kk in itertools.product(range(b2), range(b1)):
            blk = M[:, i, kk, :]                              # (l, j)
            for (l0, l1), (j0, j1) in itertools.product(st["rows"], st["cols"]):
                sv = np.linalg.svd(blk[l0:l1, j0:j1], compute_uv=False)
                assert sv[1:].max(initial=0) < 1e-12 * max(sv[0], 1e-300)


# --------------------------------------------------------------------------
# T = 0 and zero logits: closed forms
# --------------------------------------------------------------------------
@pytest.mark.parametrize("c2", [1, 2, 3])
def test_T0_is_uniform_group_mean(c2):
    b1, b2, d = 4, 7, 5
    v = _rand((1, b1 * b2, d), 3)
    q = k = _rand((1, b1 * b2, d), 4)
    O = monarch_attention(q, k, v, b1, b2, 0, 1, c2)
    vb = v.reshape(b1, b2, d)
    cols = np.array_split(np.arange(b2), c2)
    expect = np.mean([vb[kk, c].mean(0) for kk in range(b1) for c in cols], axis=0)
    np.testing.assert_allclose(O[0], np.broadcast_to(expect, (b1 * b2, d)), atol=1e-13)


@pytest.mark.parametrize("c1,c2", [(1, 1), (2, 3), (3, 2)])
@pytest.mark.parametrize("T", [1, 2])
def test_zero_logits_give_the_global_mean(c1, c2, T):
    """q = 0: softmax(S) is uniform, which the method must reach at T >= 1.

    With uneven column groups this needs the entropy bias of the L-update.
    """
    b1, b2, d = 5, 7, 4
    q = np.zeros((1, b1 * b2, d))
    k, v = _rand((1, b1 * b2, d), 1), _rand((1, b1 * b2, d), 2)
    O = monarch_attention(q, k, v, b1, b2, T, c1, c2)
    np.testing.assert_allclose(O[0], np.broadcast_to(v[0].mean(0), O[0].shape), atol=1e-13)


# --------------------------------------------------------------------------
# P5 / P6: monotone objective, and its gap to the softmax optimum
# --------------------------------------------------------------------------
@pytest.mark.parametrize("b1,b2,c1,c2", [(6, 6, 1, 1), (8, 5, 2, 2), (5, 8, 1, 3)])
def test_objective_monotone_and_bounded(b1, b2, c1, c2):
    N, d = b1 * b2, 8
    q, k, v = (_rand((3, N, d), s) * 1.5 for s in (11, 12, 13))
    qh, _ = as_heads(q, b1, b2)
    kh, _ = as_heads(k, b1, b2)
    vh, _ = as_heads(v, b1, b2)
    rows, cols, sc = groups(b1, c1), groups(b2, c2), 1 / np.sqrt(d)
    L = LFactor.uniform(3, b1, b2, rows, cols)
    rf = RFactor.uniform(kh, vh, rows, cols)
    S = dense_logits(qh, kh)
    fstar = logsumexp(S, axis=-1).sum(-1)
    trace = [objective(qh, L, rf, rows, sc)]
    for _ in range(4):
        rf = r_update(qh, kh, vh, L, rows, cols, sc)
        trace.append(objective(qh, L, rf, rows, sc))
        L = l_update(qh, rf, rows, cols, sc)
        trace.append(objective(qh, L, rf, rows, sc))
        M = materialise(L, rf, rows, cols)
        P = softmax(S, axis=-1)
        kl = (M * (np.log(M) - np.log(P))).sum(axis=(1, 2))
        np.testing.assert_allclose(fstar - trace[-1], kl, rtol=1e-9, atol=1e-10)
    trace = np.array(trace)
    assert (np.diff(trace, axis=0) >= -1e-10).all()
    assert (trace <= fstar + 1e-10).all()


def test_objective_after_l_update_is_sum_of_lse():
    b1, b2, d = 5, 6, 4
    q, k, v = (_rand((1, b1 * b2, d), s) for s in (1, 2, 3))
    _, st = _state(q, k, v, b1, b2, 2, 2, 2)
    L = st["L"]
    lse = sum(logsumexp(L.logits(i).reshape(1, b1, -1), axis=-1).sum() for i in range(b2))
    np.testing.assert_allclose(objective(st["q"], L, st["R"], st["rows"], st["sc"])[0], lse,
                               rtol=1e-12)


# --------------------------------------------------------------------------
# P7: each update is the block-coordinate maximiser (random competitors)
# --------------------------------------------------------------------------
def test_updates_beat_random_competitors():
    b1, b2, c1, c2, d = 5, 6, 2, 2, 4
    q, k, v = (_rand((1, b1 * b2, d), s) * 2 for s in (21, 22, 23))
    _, st = _state(q, k, v, b1, b2, 1, c1, c2)
    qh, kh, vh, rows, cols, sc = (st[x] for x in ("q", "k", "v", "rows", "cols", "sc"))
    L = st["L"]
    rf_opt = r_update(qh, kh, vh, L, rows, cols, sc)
    f_opt = objective(qh, L, rf_opt, rows, sc)[0]
    rng = np.random.default_rng(0)
    for _ in range(20):
        R = rf_opt.R * np.exp(0.3 * rng.standard_normal(rf_opt.R.shape))
        for j0, j1 in cols:
            R[..., j0:j1] /= R[..., j0:j1].sum(-1, keepdims=True)
        assert objective(qh, L, RFactor(R, kh, vh, cols), rows, sc)[0] < f_opt
    Lu = l_update(qh, rf_opt, rows, cols, sc)
    g_opt = objective(qh, Lu, rf_opt, rows, sc)[0]
    Larr = Lu.materialise()
    for _ in range(20):
        A = Larr * np.exp(0.3 * rng.standard_normal(Larr.shape))
        A /= A.sum(axis=(-1, -2), keepdims=True)
        assert objective(qh, LFactor.explicit(A, rows, cols), rf_opt, rows, sc)[0] < g_opt


# --------------------------------------------------------------------------
# Brute force: alternating maximisation of the dense objective by a generic
# optimiser, with the Monarch matrix built entry by entry from its definition.
# --------------------------------------------------------------------------
def _brute_force_monarch(q, k, v, b1, b2, T, c1, c2):
    q, k, v = (torch.tensor(x, dtype=torch.float64) for x in (q, k, v))
    N, d = q.shape
    S = q @ k.T / d ** 0.5
    prow = np.concatenate([[g] * len(a) for g, a in
                           enumerate(np.array_split(np.arange(b1), c1))])
    qcol = np.concatenate([[g] * len(a) for g, a in
                           enumerate(np.array_split(np.arange(b2), c2))])
    col_masks = [torch.tensor(qcol == g) for g in range(c2)]

    def L_of(th):                     # th: (b2, b1, b1*c2) -> softmax over (k, q)
        return torch.softmax(th, dim=-1).reshape(b2, b1, b1, c2)

    def R_of(th):                     # th: (b1, c1, b2, b2) -> softmax inside column groups
        out = torch.zeros_like(th)
        for m in col_masks:
            out[..., m] = torch.softmax(th[..., m], dim=-1)
        return out

    # every entry (l, i, k, j) of M, row index l*b2 + i and column k*b2 + j
    l_, i_, k_, j_ = (torch.tensor(a.reshape(-1)) for a in
                      np.meshgrid(np.arange(b1), np.arange(b2), np.arange(b1), np.arange(b2),
                                  indexing="ij"))
    p_, q_ = torch.tensor(prow)[l_], torch.tensor(qcol)[j_]

    def M_of(thL, thR):
        L, R = L_of(thL), R_of(thR)
        return (L[i_, l_, k_, q_] * R[k_, p_, i_, j_]).reshape(N, N)

    def f_of(M):
        return (M * S).sum() - torch.special.xlogy(M, M).sum()

    def argmax(th, other, which):
        th = th.clone().requires_grad_(True)
        opt = torch.optim.LBFGS([th], lr=1, max_iter=500, tolerance_grad=1e-13,
                                tolerance_change=1e-15, line_search_fn="strong_wolfe")

        def closure():
            opt.zero_grad()
            M = M_of(th, other) if which == "L" else M_of(other, th)
            loss = -f_of(M)
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
        return (M_of(thL, thR) @ v).numpy()


@pytest.mark.parametrize("b1,b2,c1,c2,T", [(2, 3, 1, 1, 1), (3, 2, 1, 1, 2),
                                           (3, 3, 2, 2, 2), (2, 3, 2, 2, 1)])
def test_matches_brute_force_alternating_maximisation(b1, b2, c1, c2, T):
    N, d = b1 * b2, 2
    q, k, v = (_rand((N, d), s) * 1.5 for s in (31, 32, 33))
    O = monarch_attention(q, k, v, b1, b2, T, c1, c2)
    Ob = _brute_force_monarch(q, k, v, b1, b2, T, c1, c2)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=2e-6)


# --------------------------------------------------------------------------
# P9 / P10: tiled Monarch contains untiled Monarch, strictly
# --------------------------------------------------------------------------
def test_c1_c2_one_is_untiled_and_embedding_is_exact():
    b1, b2, d = 6, 4, 5
    q, k, v = (_rand((2, b1 * b2, d), s) for s in (41, 42, 43))
    _, st = _state(q, k, v, b1, b2, 2, 1, 1)
    M1 = materialise(st["L"], st["R"], st["rows"], st["cols"])
    # embed the untiled (L, R) into the 2 x 2 tiled parameterisation
    rows2, cols2 = groups(b1, 2), groups(b2, 2)
    La = st["L"].materialise()[..., 0]                        # (G, i, l, k)
    Rt = st["R"].R[:, :, 0]                                   # (G, k, i, j)
    Lt = np.empty(La.shape + (2,))
    R2 = np.empty(Rt.shape[:2] + (2,) + Rt.shape[2:])
    for qi, (j0, j1) in enumerate(cols2):
        mass = Rt[..., j0:j1].sum(-1)                         # (G, k, i)
        Lt[..., qi] = La * np.swapaxes(mass, 1, 2)[:, :, None, :]
        for pi in range(2):
            R2[:, :, pi, :, j0:j1] = Rt[..., j0:j1] / mass[..., None]
    kh, vh = st["k"], st["v"]
    M2 = materialise(LFactor.explicit(Lt, rows2, cols2), RFactor(R2, kh, vh, cols2),
                     rows2, cols2)
    np.testing.assert_allclose(M2, M1, atol=1e-13)
    # one tiled step from the embedding can only raise the objective
    qh, sc = st["q"], st["sc"]
    f_un = objective(qh, st["L"], st["R"], st["rows"], sc)
    Lemb = LFactor.explicit(Lt, rows2, cols2)
    rf = r_update(qh, kh, vh, Lemb, rows2, cols2, sc)
    L2 = l_update(qh, rf, rows2, cols2, sc)
    assert (objective(qh, L2, rf, rows2, sc) >= f_un - 1e-10).all()


def test_two_spike_block_needs_tiling():
    """A target whose blocks have rank > 1 is reached exactly by c1 = c2 = 2."""
    b1, b2, N = 4, 4, 16
    rng = np.random.default_rng(1)
    rows, cols = groups(b1, 2), groups(b2, 2)
    Larr = rng.random((1, b2, b1, b1, 2)) + 0.05
    Larr /= Larr.sum(axis=(-1, -2), keepdims=True)
    R = rng.random((1, b1, 2, b2, b2)) + 0.05
    for j0, j1 in cols:
        R[..., j0:j1] /= R[..., j0:j1].sum(-1, keepdims=True)
    z = np.zeros((1, b1, b2, 1))
    Mt = materialise(LFactor.explicit(Larr, rows, cols), RFactor(R, z, z, cols), rows, cols)[0]
    blk = Mt.reshape(b1, b2, b1, b2)[:, 1, 2, :]
    assert np.linalg.svd(blk, compute_uv=False)[1] > 1e-3       # rank > 1 block
    # logits whose softmax is the target: q = sqrt(N) log Mt, k = I (d = N)
    q = np.sqrt(N) * np.log(Mt)[None]
    k = np.eye(N)[None]
    v = rng.standard_normal((1, N, 3))
    for T in (1, 3):
        O2 = monarch_attention(q, k, v, b1, b2, T, 2, 2)
        O1 = monarch_attention(q, k, v, b1, b2, T, 1, 1)
        np.testing.assert_allclose(O2[0], Mt @ v[0], atol=1e-12)
        assert np.abs(O1[0] - Mt @ v[0]).max() > 1e-2
