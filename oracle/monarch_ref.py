"""MonarchAttention forward pass in float64 on the CPU: the oracle.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
leg of the benchmark use this file.  It is deliberately plain and slow: numpy
float64, one step of the method per function, no blocking or fusion beyond
what the method itself states.  Library primitives (matmul, einsum, exp, log)
serve as steps.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
against dense softmax attention, closed forms, invariants and brute force.
The one thing left unpinned is the ViT-B objective table printed in the
MonarchAttention OpenReview discussion (f(M) = 418, 937, 940, 940 for T = 0..3):
it needs trained ViT-B weights and ImageNet images, so that table is
"parity unpinned".

Notation (one head)
-------------------
N = b1 * b2 tokens.  Token n = l * b2 + i with l in [b1] (the chunk) and
i in [b2] (the position inside the chunk); keys are n' = k * b2 + j likewise.
For a (f, h, w) video latent flattened row-major, the aligned block sizes
(b1, b2) = (f h, w) give l = (f, h) and i = w (MonarchRT summary, "Key claims":
the six aligned configurations).

Logits S[(l,i),(k,j)] = sc * q_(l,i) . k_(k,j) with sc = 1 / sqrt(d).

Monarch matrix M = P L P^T R with L, R block diagonal (MonarchRT summary,
"Method" (1)).  Entry by entry:

    M[(l,i),(k,j)] = L_i[l,k] * R_k[i,j]

Tiled Monarch (MonarchRT summary, "Key claims" and "Method" (2), Theorem 4.1):
every (i,k) block is cut into c1 x c2 sub-tiles, each independently rank one.
With p(l) in [c1] the contiguous row group of l and q(j) in [c2] the
contiguous column group of j:

    M[(l,i),(k,j)] = L_i[l,(k,q(j))] * R_{k,p(l)}[i,j]

Constraints (OpenReview discussion, response to reviewer nTcP: L and R are
kept positive, "Alternating Maximization with Constraints"): each row of L_i
lies on the simplex over the b1*c2 pairs (k,q); each row of R_{k,p} lies on the
simplex separately inside every column group q.  Then M >= 0 and every row of
M sums to one.  c1 = c2 = 1 is the untiled model.

Softmax variational objective (MonarchAttention AI summary, "Approach";
OpenReview discussion, f(M) of eq. (6)):

    f(M) = sum over rows of  <M_row, S_row> + H(M_row),   H(m) = -sum m ln m

Over row-stochastic M >= 0 its maximiser is softmax(S) row by row.  For the
Monarch model the row entropy splits as

    H(M_(l,i)) = H(L_i[l,:]) + sum_{k,q} L_i[l,(k,q)] Hs_{k,p(l),q,i}

with Hs_{k,p,q,i} = H(R_{k,p}[i, j in q]).  Writing
Kt_{k,p,q,i} = sum_{j in q} R_{k,p}[i,j] k_(k,j):

    f = sum_{l,i} [ sum_{k,q} L_i[l,(k,q)] (sc q_(l,i).Kt_{k,p(l),q,i} + Hs_{k,p(l),q,i})
                    + H(L_i[l,:]) ]

Alternating maximisation.  With L fixed the objective is concave in R and with
R fixed concave in L (OpenReview discussion, response to reviewer nTcP on
concavity); each sub-problem splits into independent entropy-regularised
linear problems on simplices, whose maximiser is a softmax:

  R-update, for every (k, p, q, i):
      c  = sum_{l in p} L_i[l,(k,q)]
      Qt = sum_{l in p} L_i[l,(k,q)] q_(l,i) / c          (the aggregated query)
      R_{k,p}[i, j in q] = softmax_{j in q}( sc Qt . k_(k,j) )
  L-update, for every (l, i):
      L_i[l,(k,q)] = softmax_{(k,q)}( sc q_(l,i).Kt_{k,p(l),q,i} + Hs_{k,p(l),q,i} )

Output without forming the N x N matrix (MonarchRT summary, "Method" (3);
MonarchAttention abstract: Theta(N sqrt(N) d) compute, Theta(N d) I/O):

    O_(l,i) = sum_{k,q} L_i[l,(k,q)] Y_{k,p(l),q,i},   Y_{k,p,q,i} = sum_{j in q} R_{k,p}[i,j] v_(k,j)

Padding (OpenReview discussion, author response on choosing block sizes:
m is the ceiling of N / b, and for ViT's N = 197 the pad tokens go before the
class token): a sequence of N_real < b1 * b2 tokens is padded to b1 * b2,
with the pad tokens before the real ones (pre-padding) or after them.  The
pages do not say how pad tokens enter the softmaxes; the reading taken here
keeps the objective over the real tokens only:
  * a pad key gets zero R weight (R rows are softmaxes over the real keys of
    each column group);
  * a column group (k, q) with no real key gets zero L weight (L rows are
    softmaxes over the pairs (k, q) that hold a real key);
  * pad query rows are left out of the aggregated queries and of the
    objective, and their outputs are dropped.
With no pad tokens every mask is all true and nothing changes.

Readings where the pages are silent:
  * L starts uniform, 1 / (b1 c2); R starts uniform inside every column group.
  * One step is an R-update followed by an L-update; T = 0 returns the
    uniform initial Monarch matrix; the output uses the last L and R.
  * Uneven groups: sizes differ by at most one, larger groups first.
  * If c == 0 (underflow) the aggregated query is 0 (that R row then is
    uniform and carries zero weight in M).
  * Natural logarithm, 0 ln 0 = 0, softmax is max-subtracted.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def groups(n: int, c: int):
    """Split range(n) into c contiguous (start, end) groups.

    Sizes differ by at most one, the larger groups first (945 rows in two
    groups give 473 and 472).
    """
    if not (1 <= c <= n):
        raise ValueError(f"need 1 <= c <= n, got c={c}, n={n}")
    base, extra = divmod(n, c)
    out, s = [], 0
    for g in range(c):
        z = base + (1 if g < extra else 0)
        out.append((s, s + z))
        s += z
    return out


def _xlogx(p):
    """p ln p with 0 ln 0 = 0."""
    pos = p > 0
    return np.where(pos, p * np.log(np.where(pos, p, 1.0)), 0.0)


def _masked_softmax_last(s, mask):
    """softmax over the last axis restricted to mask (broadcast to s); entries
    outside the mask are 0, and a row with no entry inside it is all 0."""
    mask = np.broadcast_to(mask, s.shape)
    sm = np.where(mask, s, -np.inf)
    m = sm.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(mask, np.exp(sm - m), 0.0)
    z = e.sum(axis=-1, keepdims=True)
    return np.where(z > 0, e / np.where(z > 0, z, 1.0), 0.0)


def token_mask(b1: int, b2: int, n_pad: int = 0, pad_front: bool = True):
    """(b1, b2) bool: True where token l*b2 + i is real.  The n_pad pad tokens
    come first (pre-padding) or last."""
    N = b1 * b2
    if not (0 <= n_pad < N):
        raise ValueError(f"need 0 <= n_pad < b1*b2, got {n_pad}")
    m = np.zeros(N, dtype=bool)
    if pad_front:
        m[n_pad:] = True
    else:
        m[:N - n_pad] = True
    return m.reshape(b1, b2)


def group_valid(real, cols):
    """(b1, c2) bool: column group q of chunk k holds at least one real key."""
    return np.stack([real[:, j0:j1].any(axis=1) for j0, j1 in cols], axis=1)


def as_heads(x, b1: int, b2: int):
    """(..., N, d) -> float64 (G, b1, b2, d) with token n = l*b2 + i."""
    x = np.asarray(x, dtype=np.float64)
    *lead, N, d = x.shape
    if N != b1 * b2:
        raise ValueError(f"N={N} != b1*b2={b1 * b2}")
    return x.reshape(-1, b1, b2, d), tuple(lead)


# ----------------------------------------------------------------------------
# the two factors
# ----------------------------------------------------------------------------
class RFactor:
    """R_{k,p}[i,j] for all chunks k and row groups p, with its contractions.

    ``R`` has shape (G, b1[k], c1[p], b2[i], b2[j]); inside every column group
    q the entries of a row sum to one (all zero for a group with no real
    key).  From it:
      Kt (G, b1[k], c1[p], c2[q], b2[i], d) = sum_{j in q} R k_(k,j)
      Y  (same)                             = sum_{j in q} R v_(k,j)
      Hs (G, b1[k], c1[p], c2[q], b2[i])    = entropy of R over j in q
      valid (b1[k], c2[q])                  = group q of chunk k holds a real key
    """

    def __init__(self, R, k, v, cols, real=None):
        self.R = R
        G, b1, c1, b2, _ = R.shape
        c2 = len(cols)
        d, dv = k.shape[-1], v.shape[-1]
        if real is None:
            real = np.ones((b1, b2), dtype=bool)
        self.valid = group_valid(real, cols)
        self.Kt = np.empty((G, b1, c1, c2, b2, d))
        self.Y = np.empty((G, b1, c1, c2, b2, dv))
        self.Hs = np.empty((G, b1, c1, c2, b2))
        for qi, (j0, j1) in enumerate(cols):
            Rq = R[..., j0:j1]                               # (G, k, p, i, j in q)
            self.Kt[:, :, :, qi] = Rq @ k[:, :, None, j0:j1]  # (G, k, p, i, d)
            self.Y[:, :, :, qi] = Rq @ v[:, :, None, j0:j1]
            self.Hs[:, :, :, qi] = -_xlogx(Rq).sum(axis=-1)

    @classmethod
    def uniform(cls, k, v, rows, cols, real=None):
        """R uniform over the real keys of every column group."""
        G, b1, b2, _ = k.shape
        if real is None:
            real = np.ones((b1, b2), dtype=bool)
        R = np.zeros((G, b1, len(rows), b2, b2))
        for j0, j1 in cols:
            w = real[:, j0:j1].astype(np.float64)            # (k, j in q)
            cnt = w.sum(axis=1, keepdims=True)
            w = np.where(cnt > 0, w / np.where(cnt > 0, cnt, 1.0), 0.0)
            R[..., j0:j1] = w[None, :, None, None, :]
        return cls(R, k, v, cols, real)


class LFactor:
    """L_i[l,(k,q)] for every position i, produced one block at a time.

    ``block(i)`` returns an array of shape (G, b1[l], b1[k], c2[q]) whose rows
    sum to one over the valid pairs (k, q), those whose column group holds a
    real key, and are zero on the others.  The factor is either uniform, an
    explicit array of shape (G, b2[i], b1[l], b1[k], c2[q]), or the L-update
    of an RFactor.
    """

    def __init__(self, G, b1, b2, rows, cols, *, arr=None, q=None, rf=None, sc=None,
                 valid=None):
        self.G, self.b1, self.b2 = G, b1, b2
        self.rows, self.cols = rows, cols
        self.arr, self.q, self.rf, self.sc = arr, q, rf, sc
        if valid is None:
            valid = rf.valid if rf is not None else np.ones((b1, len(cols)), dtype=bool)
        self.valid = valid

    @classmethod
    def uniform(cls, G, b1, b2, rows, cols, valid=None):
        """L uniform over the valid pairs (k, q)."""
        return cls(G, b1, b2, rows, cols, valid=valid)

    @classmethod
    def explicit(cls, arr, rows, cols, valid=None):
        G, b2, b1, _, _ = arr.shape
        return cls(G, b1, b2, rows, cols, arr=arr, valid=valid)

    def logits(self, i):
        """sc q_(l,i).Kt_{k,p(l),q,i} + Hs_{k,p(l),q,i}, shape (G, l, k, q)."""
        rf, q = self.rf, self.q
        out = np.empty((self.G, self.b1, self.b1, len(self.cols)))
        for pi, (l0, l1) in enumerate(self.rows):
            nk = self.b1 * len(self.cols)
            Kt = rf.Kt[:, :, pi, :, i, :].reshape(self.G, nk, -1)   # (G, (k,q), d)
            Hs = rf.Hs[:, :, pi, :, i].reshape(self.G, 1, nk)       # (G, 1, (k,q))
            s = self.sc * (q[:, l0:l1, i] @ np.swapaxes(Kt, -1, -2)) + Hs
            out[:, l0:l1] = s.reshape(self.G, l1 - l0, self.b1, len(self.cols))
        return out

    def block(self, i):
        c2 = len(self.cols)
        if self.arr is not None:
            return self.arr[:, i]
        if self.rf is None:
            w = self.valid / self.valid.sum()
            return np.broadcast_to(w, (self.G, self.b1, self.b1, c2)).copy()
        s = self.logits(i)
        flat = s.reshape(self.G, self.b1, self.b1 * c2)
        return _masked_softmax_last(flat, self.valid.reshape(-1)).reshape(s.shape)

    def materialise(self):
        return np.stack([self.block(i) for i in range(self.b2)], axis=1)


# ----------------------------------------------------------------------------
# the steps
# ----------------------------------------------------------------------------
def r_update(q, k, v, L: LFactor, rows, cols, sc, real=None) -> RFactor:
    """Exact maximiser of f over R with L fixed (a softmax per (k, p, q, i)).

    ``real`` (b1, b2) marks the real tokens: pad rows l are left out of the
    aggregated queries and pad keys get zero weight."""
    G, b1, b2, d = q.shape
    c1, c2 = len(rows), len(cols)
    if real is None:
        real = np.ones((b1, b2), dtype=bool)
    Qt = np.zeros((G, b1, c1, c2, b2, d))                    # [k, p, q, i]
    for i in range(b2):
        Lb = L.block(i)                                      # (G, l, k, q)
        for pi, (l0, l1) in enumerate(rows):
            Lp = Lb[:, l0:l1] * real[l0:l1, i][None, :, None, None]
            c = Lp.sum(axis=1)                               # (G, k, q)
            num = np.einsum("glkq,gld->gkqd", Lp, q[:, l0:l1, i], optimize=True)
            safe = np.where(c > 0, c, 1.0)
            Qt[:, :, pi, :, i] = np.where((c > 0)[..., None], num / safe[..., None], 0.0)
    R = np.empty((G, b1, c1, b2, b2))
    for pi in range(c1):
        for qi, (j0, j1) in enumerate(cols):
            s = sc * (Qt[:, :, pi, qi] @ np.swapaxes(k[:, :, j0:j1], -1, -2))  # (G, k, i, j)
            R[:, :, pi, :, j0:j1] = _masked_softmax_last(s, real[None, :, None, j0:j1])
    return RFactor(R, k, v, cols, real)


def l_update(q, rf: RFactor, rows, cols, sc) -> LFactor:
    """Exact maximiser of f over L with R fixed (a softmax per row (l, i))."""
    G, b1, b2, _ = q.shape
    return LFactor(G, b1, b2, rows, cols, q=q, rf=rf, sc=sc)


def output(L: LFactor, rf: RFactor, rows):
    """O_(l,i) = sum_{k,q} L_i[l,(k,q)] Y_{k,p(l),q,i}; shape (G, b1, b2, d)."""
    G, b1, _, _, b2, dv = rf.Y.shape
    O = np.empty((G, b1, b2, dv))
    for i in range(b2):
        Lb = L.block(i)
        nk = Lb.shape[2] * Lb.shape[3]
        for pi, (l0, l1) in enumerate(rows):
            Lp = Lb[:, l0:l1].reshape(G, l1 - l0, nk)                # (G, l, (k,q))
            O[:, l0:l1, i] = Lp @ rf.Y[:, :, pi, :, i].reshape(G, nk, dv)
    return O


def objective(q, L: LFactor, rf: RFactor, rows, sc, real=None):
    """f(M) of the factored Monarch matrix over the real rows, per head (shape (G,))."""
    G = q.shape[0]
    if real is None:
        real = np.ones(q.shape[1:3], dtype=bool)
    f = np.zeros(G)
    for i in range(q.shape[2]):
        Lb = L.block(i)
        for pi, (l0, l1) in enumerate(rows):
            nk = Lb.shape[2] * Lb.shape[3]
            Kt = rf.Kt[:, :, pi, :, i].reshape(G, nk, -1)
            lin = sc * (q[:, l0:l1, i] @ np.swapaxes(Kt, -1, -2)) \
                + rf.Hs[:, :, pi, :, i].reshape(G, 1, nk)
            Lp = Lb[:, l0:l1].reshape(G, l1 - l0, nk)
            rw = real[l0:l1, i][None, :, None]
            f += (rw * (Lp * lin - _xlogx(Lp))).sum(axis=(1, 2))
    return f


def materialise(L: LFactor, rf: RFactor, rows, cols):
    """Dense M (G, N, N) with M[(l,i),(k,j)] = L_i[l,(k,q(j))] R_{k,p(l)}[i,j]."""
    G, b1, _, b2, _ = rf.R.shape
    M = np.zeros((G, b1, b2, b1, b2))
    for i in range(b2):
        Lb = L.block(i)
        for pi, (l0, l1) in enumerate(rows):
            for qi, (j0, j1) in enumerate(cols):
                M[:, l0:l1, i, :, j0:j1] = Lb[:, l0:l1, :, qi][..., None] \
                    * rf.R[:, :, pi, i, j0:j1][:, None]
    return M.reshape(G, b1 * b2, b1 * b2)


def dense_logits(q, k):
    """S = q k^T / sqrt(d) for (G, b1, b2, d) inputs, shape (G, N, N)."""
    G, b1, b2, d = q.shape
    qf = q.reshape(G, b1 * b2, d)
    kf = k.reshape(G, b1 * b2, d)
    return (qf @ np.swapaxes(kf, -1, -2)) / np.sqrt(d)


def objective_dense(M, S):
    """f(M) = sum M o S - sum M ln M per head, straight from the definition."""
    return (M * S).sum(axis=(1, 2)) - _xlogx(M).sum(axis=(1, 2))


# ----------------------------------------------------------------------------
# the forward pass
# ----------------------------------------------------------------------------
def monarch_attention(q, k, v, b1, b2, T, c1=1, c2=1, return_state=False, n_pad=0,
                      pad_front=True):
    """MonarchAttention forward: T alternating steps, then O = M V.

    q, k, v: arrays (..., N_real, d) with N_real = b1*b2 - n_pad (any float
    dtype; read as float64).  The n_pad pad tokens are placed before the real
    tokens (``pad_front``) or after them.  Returns O (..., N_real, d) in
    float64, the real tokens' rows; with ``return_state`` also the final
    (L, R) factors, the head-major padded inputs and the real-token mask.
    """
    real = token_mask(b1, b2, n_pad, pad_front)
    qa, ka, va = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    *lead, n_in, d = qa.shape
    if n_in != b1 * b2 - n_pad:
        raise ValueError(f"N={n_in} != b1*b2 - n_pad = {b1 * b2 - n_pad}")
    if T < 0:
        raise ValueError("T must be >= 0")

    def padded(x):
        x = x.reshape(-1, n_in, x.shape[-1])
        out = np.zeros((x.shape[0], b1 * b2, x.shape[-1]))
        out[:, real.reshape(-1)] = x
        return out.reshape(-1, b1, b2, x.shape[-1])

    qh, kh, vh = padded(qa), padded(ka), padded(va)
    G = qh.shape[0]
    sc = 1.0 / np.sqrt(d)
    rows, cols = groups(b1, c1), groups(b2, c2)
    L = LFactor.uniform(G, b1, b2, rows, cols, valid=group_valid(real, cols))
    rf = RFactor.uniform(kh, vh, rows, cols, real)
    for _ in range(T):
        rf = r_update(qh, kh, vh, L, rows, cols, sc, real)
        L = l_update(qh, rf, rows, cols, sc)
    O = output(L, rf, rows).reshape(G, b1 * b2, vh.shape[-1])[:, real.reshape(-1)]
    O = O.reshape(*lead, n_in, vh.shape[-1])
    if return_state:
        return O, dict(L=L, R=rf, q=qh, k=kh, v=vh, rows=rows, cols=cols, sc=sc, real=real)
    return O


# ----------------------------------------------------------------------------
# the backward pass (T = 1)
# ----------------------------------------------------------------------------
def monarch_attention_backward(q, k, v, dO, b1, b2, c1=1, c2=1):
    """Gradients (dq, dk, dv) of sum(O * dO) for the T = 1 forward pass.

    One refinement step is what the pages finetune with (MonarchRT summary:
    finetuning collapses the refinement to one iteration; forward and
    backward kernels).  The chain rule through the steps of the forward pass,
    in reverse:

      O_(l,i) = sum_{k,q} L Y                  dY  = sum_{l in p} L dO_(l,i)
                                               dL  = dO_(l,i) . Y
      L = softmax_{(k,q)}(S_L)                 dS_L = L (dL - sum_{k,q} L dL)
      S_L = sc q . Kt + Hs                     dq += sc sum_{k,q} dS_L Kt
                                               dKt = sc sum_{l in p} dS_L q_(l,i)
                                               dHs = sum_{l in p} dS_L
      Kt, Y, Hs from R (per (k,p,q,i))         dR_j = dKt . k_j + dY . v_j - dHs (ln R_j + 1)
      R = softmax_{j in q}(S_R)                dS_R = R (dR - sum_j R dR)
      S_R = sc Qt0 . k_(k,j)                   dk_j += sum R dKt + sc sum dS_R Qt0
                                               dv_j += sum R dY
                                               dQt0 = sc sum_{k,j} dS_R k_j
      Qt0_{p,i} = mean_{l in p} q_(l,i)        dq_(l,i) += dQt0_{p(l),i} / |p|

    q, k, v, dO: (..., N, d) with N = b1*b2.  Returns float64 arrays of the
    same shapes.
    """
    O, st = monarch_attention(q, k, v, b1, b2, 1, c1, c2, return_state=True)
    L, rf, qh, kh, vh = st["L"], st["R"], st["q"], st["k"], st["v"]
    rows, cols, sc = st["rows"], st["cols"], st["sc"]
    G, _, _, d = qh.shape
    dOh = np.asarray(dO, dtype=np.float64).reshape(G, b1, b2, -1)
    Oh = np.asarray(O).reshape(G, b1, b2, -1)
    nk = b1 * c2
    dq = np.zeros_like(qh)
    dKt = np.zeros_like(rf.Kt)                     # (G, k, p, q, i, d)
    dY = np.zeros_like(rf.Y)
    dHs = np.zeros_like(rf.Hs)                     # (G, k, p, q, i)
    # ---- L side, one position i and row group p at a time ----
    for i in range(b2):
        Lb = L.block(i)                                          # (G, l, k, q)
        for pi, (l0, l1) in enumerate(rows):
            Lp = Lb[:, l0:l1].reshape(G, l1 - l0, nk)            # (G, l, kq)
            Kt = rf.Kt[:, :, pi, :, i].reshape(G, nk, d)         # (G, kq, d)
            Yp = rf.Y[:, :, pi, :, i].reshape(G, nk, -1)
            g = dOh[:, l0:l1, i]                                 # (G, l, dv)
            dL = g @ np.swapaxes(Yp, -1, -2)                     # (G, l, kq)
            delta = (g * Oh[:, l0:l1, i]).sum(-1, keepdims=True)  # sum_{kq} L dL = dO . O
            dS = Lp * (dL - delta)
            dq[:, l0:l1, i] += sc * (dS @ Kt)
            dKt[:, :, pi, :, i] = (sc * (np.swapaxes(dS, -1, -2) @ qh[:, l0:l1, i])
                                   ).reshape(G, b1, c2, d)
            dHs[:, :, pi, :, i] = dS.sum(axis=1).reshape(G, b1, c2)
            dY[:, :, pi, :, i] = (np.swapaxes(Lp, -1, -2) @ g).reshape(G, b1, c2, -1)
    # ---- R side: every (k, p, q, i) row over j in q ----
    dk = np.zeros_like(kh)
    dv = np.zeros_like(vh)
    dQt0 = np.zeros((G, len(rows), b2, d))
    Qt0 = np.stack([qh[:, l0:l1].mean(axis=1) for l0, l1 in rows], axis=1)  # (G, p, i, d)
    for pi in range(len(rows)):
        for qi, (j0, j1) in enumerate(cols):
            R = rf.R[:, :, pi, :, j0:j1]                         # (G, k, i, j)
            kq, vq = kh[:, :, j0:j1], vh[:, :, j0:j1]            # (G, k, j, d)
            a = dKt[:, :, pi, qi]                                # (G, k, i, d)
            y = dY[:, :, pi, qi]
            h = dHs[:, :, pi, qi][..., None]                     # (G, k, i, 1)
            with np.errstate(divide="ignore"):
                lnR = np.where(R > 0, np.log(np.where(R > 0, R, 1.0)), 0.0)
            dR = a @ np.swapaxes(kq, -1, -2) + y @ np.swapaxes(vq, -1, -2) - h * (lnR + 1.0)
            dS = R * (dR - (R * dR).sum(-1, keepdims=True))     # (G, k, i, j)
            dk[:, :, j0:j1] += np.swapaxes(R, -1, -2) @ a + \
                sc * (np.swapaxes(dS, -1, -2) @ Qt0[:, None, pi])
            dv[:, :, j0:j1] += np.swapaxes(R, -1, -2) @ y
            dQt0[:, pi] += sc * np.einsum("gkij,gkjd->gid", dS, kq)
    for pi, (l0, l1) in enumerate(rows):
        dq[:, l0:l1] += dQt0[:, pi][:, None] / (l1 - l0)
    shape = np.asarray(q).shape
    return (dq.reshape(shape), dk.reshape(np.asarray(k).shape), dv.reshape(np.asarray(v).shape))
