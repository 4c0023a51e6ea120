"""Element-wise error bounds for the fp32 training step (test infrastructure).

Every gradient of the training step is a sum of terms (a batch sum for the
MLP weights and biases, a sum over occurrences for a table row, a sum over the
interaction partners for a pooled vector). An fp32 program that evaluates the
step correctly, in any order, differs from the fp64 oracle by rounding, and
that rounding is bounded by a small multiple of u (2^-24) times the size of the
computation, the same computation carried out on absolute values. How deep
that absolute evaluation goes decides whether the bound is honest or vacuous:

  level 0: |value| only;
  level 1: the sum's own terms, |dY| |a| (the gradient's last operation);
  level 2: the terms with each operand taken at its own level-1 size, i.e. the
           last two operations (|dY_next| |W| for a gradient, |W| |a_prev| + |b|
           for an activation, sum |X_i| |X_j| for an interaction term);
  full:    the whole chain from the loss, which on the deep training network
           grows by sum|W| per layer and allowed errors ~1e10 times the
           gradients themselves.

Measured with plain fp32 PyTorch on the CPU (two summation orders), the level-1
bound is exceeded by up to 2.6e-2 on deep layers (rounding carried in from the
operands' own computations), while level 2 holds with a margin of 3x or more
at rtol = 1e-5 on every tensor, except for one effect no level captures: a
ReLU unit whose pre-activation lies within rounding of 0 may take either branch
in fp32, and a flip changes that unit's gradient by its whole value and, through
the rest of that sample's backward pass, everything below it. Those units are
found (|pre-activation| <= kappa x its level-2 size) and the exact effect of
each one flipping is propagated through the sample's backward pass; the bound
adds the sum of |effect| over them. So, element by element,

    |gpu - oracle| <= rtol (|oracle| + S2) + F

with S2 the level-2 size and F the flip allowance. The median S2 / |oracle|
is 2 to 3000 depending on the layer (the old full-chain size: 1e14 to 1e17).

Values here are recomputed in plain fp64 numpy from the same definition as the
oracle (ReLU after every bottom layer and every hidden top layer, the last top
layer linear, Z the strict lower triangle of X X^T in row-major order over
X = [x_dense; e_1..e_K], concat [x_dense, Z], loss the batch mean of
softplus(z) - y z); ``bounds`` cross-checks them against the oracle's
gradients before returning, so a yardstick built on different values fails
loudly. Nothing here feeds the oracle, and no value comes from the GPU.
"""
from __future__ import annotations

import numpy as np

KAPPA = 4e-6        # a pre-activation this close to 0, relative to its level-1 size, may flip in fp32


class _Layer:
    """Forward record of one linear layer: input a (value, s1), pre-activation p, ReLU mask and near set."""

    def __init__(self, W, b, a, a_s1, a_s2, relu):
        aW = np.abs(W)
        self.W, self.a, self.a_s1 = W, a, a_s1
        p = a @ W.T + b
        p_s1 = np.abs(a) @ aW.T + np.abs(b)
        p_s2 = a_s1 @ aW.T + np.abs(b)
        if relu:
            self.mask = p > 0
            self.near = np.abs(p) <= KAPPA * p_s1
        else:
            self.mask = np.ones_like(p, bool)
            self.near = np.zeros_like(p, bool)
        keep = self.mask | self.near
        self.out = np.where(self.mask, p, 0.0)
        self.out_s1 = np.where(keep, p_s1, 0.0)
        self.out_s2 = np.where(keep, p_s2, 0.0)


def _bags(model, B, offsets, indices):
    """(k, b, global row) of every valid occurrence, table-major."""
    K = model.K
    base = np.concatenate([[0], np.cumsum(model.rows)])[:-1].astype(np.int64)
    offs = np.asarray(offsets, np.int64)
    idx = np.asarray(indices, np.int64)
    ks, bs, rs = [], [], []
    nnz = idx.size
    for k in range(K):
        for b in range(B):
            s, e = offs[k * B + b], offs[k * B + b + 1]
            if s < 0 or e < s or e > nnz:
                continue
            r = idx[s:e]
            r = r[(r >= 0) & (r < model.rows[k])]
            ks.append(np.full(r.size, k))
            bs.append(np.full(r.size, b))
            rs.append(r + base[k])
    cat = lambda v: np.concatenate(v) if v else np.zeros(0, np.int64)  # noqa: E731
    return cat(ks).astype(np.int64), cat(bs).astype(np.int64), cat(rs).astype(np.int64)


def _sym(dZ, K):
    """[n][K(K+1)/2] strict-lower-triangle gradients -> symmetric [n][K+1][K+1] with zero diagonal."""
    ii, jj = np.tril_indices(K + 1, -1)
    S = np.zeros((dZ.shape[0], K + 1, K + 1))
    S[:, ii, jj] = dZ
    return S + S.transpose(0, 2, 1)


def bounds(model, dense, offsets, indices, labels, oracle_grads=None):
    """S2 (level-2 size) and F (flip allowance) of every gradient of the training step.

    Returns {key: [per layer arrays]} for bot_dW, bot_db, top_dW, top_db with keys '<key>_S2' and
    '<key>_F', and 'table_grad_S2', 'table_grad_F' over all table rows. When ``oracle_grads`` (the
    oracle's train_grads dict) is given, the fp64 values recomputed here must agree with it to 1e-9 of
    each tensor's largest entry."""
    dense = np.asarray(dense, np.float64)
    labels = np.asarray(labels, np.float64)
    B = dense.shape[0]
    K, d = model.K, model.d
    ii, jj = np.tril_indices(K + 1, -1)

    # ---- forward, keeping each layer's record
    bot = []
    a, a1, a2 = dense, np.abs(dense), np.abs(dense)
    for W, b in zip(model.bot_W, model.bot_b):
        L = _Layer(W, b, a, a1, a2, True)
        bot.append(L)
        a, a1, a2 = L.out, L.out_s1, L.out_s2
    x, x1, x2 = a, a1, a2
    ks, bs, rs = _bags(model, B, offsets, indices)
    E = np.zeros((B, K, d))
    Ea = np.zeros((B, K, d))
    np.add.at(E, (bs, ks), model.tables[rs])
    np.add.at(Ea, (bs, ks), np.abs(model.tables[rs]))
    X = np.concatenate([x[:, None, :], E], 1)                 # [B][K+1][d]
    X1 = np.concatenate([x1[:, None, :], Ea], 1)              # level-1 sizes (a pooled bag: sum |rows|)
    XaT = np.abs(X)
    Z = np.einsum("bid,bjd->bij", X, X)[:, ii, jj]
    Z1 = np.einsum("bid,bjd->bij", XaT, XaT)[:, ii, jj]
    Z2 = np.einsum("bid,bjd->bij", X1, X1)[:, ii, jj]
    h, h1, h2 = (np.concatenate([x, Z], 1), np.concatenate([x1, Z1], 1),
                 np.concatenate([x2, Z2], 1))
    top = []
    n_top = len(model.top_W)
    for l, (W, b) in enumerate(zip(model.top_W, model.top_b)):
        L = _Layer(W, b, h, h1, h2, l < n_top - 1)
        top.append(L)
        h, h1, h2 = L.out, L.out_s1, L.out_s2
    z, z1 = h[:, 0], h1[:, 0]
    sg = 1.0 / (1.0 + np.exp(-z))

    # ---- backward with level-1 sizes of every gradient (level 2 of the sums formed from them)
    dY = ((sg - labels) / B)[:, None]
    dY1 = ((np.abs(sg - labels) + 0.25 * z1) / B)[:, None]    # the sigmoid's slope is at most 1/4
    out = {k: [None] * len(v) for k, v in (("top_dW", top), ("top_db", top), ("top_dW_S2", top),
                                            ("top_db_S2", top), ("bot_dW", bot), ("bot_db", bot),
                                            ("bot_dW_S2", bot), ("bot_db_S2", bot))}
    dYs = {}
    for l in range(n_top - 1, -1, -1):
        L = top[l]
        dYs[("top", l)] = dY
        out["top_dW"][l] = dY.T @ L.a
        out["top_db"][l] = dY.sum(0)
        out["top_dW_S2"][l] = dY1.T @ L.a_s1
        out["top_db_S2"][l] = dY1.sum(0)
        dA = dY @ L.W
        dA1 = np.abs(dY) @ np.abs(L.W)
        if l > 0:
            P = top[l - 1]
            dY = np.where(P.mask, dA, 0.0)
            dY1 = np.where(P.mask | P.near, dA1, 0.0)
        else:
            dc, dc1 = dA, dA1
    S = _sym(dc[:, d:], K)
    dX = np.einsum("bij,bjd->bid", S, X)
    dX[:, 0, :] += dc[:, :d]
    S1 = _sym(dc1[:, d:], K)
    dX1 = np.einsum("bij,bjd->bid", np.abs(S), XaT)
    dX1[:, 0, :] += np.abs(dc[:, :d])
    dX2 = np.einsum("bij,bjd->bid", S1, X1)
    dX2[:, 0, :] += dc1[:, :d]
    n_rows = model.tables.shape[0]
    tg = np.zeros((n_rows, d))
    tg2 = np.zeros((n_rows, d))
    np.add.at(tg, rs, dX[bs, ks + 1])
    np.add.at(tg2, rs, dX1[bs, ks + 1])
    out["table_grad"], out["table_grad_S2"] = tg, tg2
    Lx = bot[-1]
    dY = np.where(Lx.mask, dX[:, 0, :], 0.0)
    dY1 = np.where(Lx.mask | Lx.near, dX1[:, 0, :], 0.0)
    for l in range(len(bot) - 1, -1, -1):
        L = bot[l]
        dYs[("bot", l)] = dY
        out["bot_dW"][l] = dY.T @ L.a
        out["bot_db"][l] = dY.sum(0)
        out["bot_dW_S2"][l] = dY1.T @ L.a_s1
        out["bot_db_S2"][l] = dY1.sum(0)
        if l > 0:
            P = bot[l - 1]
            dA = dY @ L.W
            dY = np.where(P.mask, dA, 0.0)
            dY1 = np.where(P.mask | P.near, np.abs(dYs[("bot", l)]) @ np.abs(L.W), 0.0)
    del dX2

    # ---- flip allowance: every near unit, its gradient toggled, propagated exactly through its sample
    F = {"top_dW_F": [np.zeros_like(w) for w in model.top_W], "top_db_F": [np.zeros(w.shape[0]) for w in model.top_W],
         "bot_dW_F": [np.zeros_like(w) for w in model.bot_W], "bot_db_F": [np.zeros(w.shape[0]) for w in model.bot_W],
         "table_grad_F": np.zeros((n_rows, d))}
    occ_of = [[] for _ in range(B)]
    for q in range(bs.size):
        occ_of[bs[q]].append(q)

    def bottom_effect(delta, samp, start):
        """delta [n][width of bottom layer `start`'s output]: gradient change at that layer's pre-activation."""
        for l in range(start, -1, -1):
            L = bot[l]
            F["bot_dW_F"][l] += np.abs(delta).T @ np.abs(L.a[samp])
            F["bot_db_F"][l] += np.abs(delta).sum(0)
            if l > 0:
                delta = np.where(bot[l - 1].mask[samp], delta @ L.W, 0.0)

    def top_effect(delta, samp, start):
        for l in range(start, -1, -1):
            L = top[l]
            F["top_dW_F"][l] += np.abs(delta).T @ np.abs(L.a[samp])
            F["top_db_F"][l] += np.abs(delta).sum(0)
            delta = delta @ L.W
            if l > 0:
                delta = np.where(top[l - 1].mask[samp], delta, 0.0)
        dXe = np.einsum("nij,njd->nid", _sym(delta[:, d:], K), X[samp])
        dXe[:, 0, :] += delta[:, :d]
        for n, b in enumerate(samp):
            for q in occ_of[b]:
                F["table_grad_F"][rs[q]] += np.abs(dXe[n, ks[q] + 1])
        bottom_effect(np.where(Lx.mask[samp], dXe[:, 0, :], 0.0), samp, len(bot) - 1)

    def flips(layers, grad_key, effect):
        for l, L in enumerate(layers):
            sb, su = np.nonzero(L.near)
            if sb.size == 0:
                continue
            # the gradient reaching this unit from above (before its own mask): dA of layer l+1
            g_above = dYs[(grad_key, l + 1)] @ layers[l + 1].W if l + 1 < len(layers) else None
            if g_above is None:        # the bottom's last layer: its gradient comes from the interaction
                g_above = dX[:, 0, :]
            delta = np.zeros((sb.size, L.out.shape[1]))
            delta[np.arange(sb.size), su] = g_above[sb, su]
            effect(delta, sb, l)

    flips(top, "top", top_effect)
    flips(bot, "bot", bottom_effect)
    out.update(F)

    if oracle_grads is not None:
        for key in ("bot_dW", "bot_db", "top_dW", "top_db"):
            for l, (mine, theirs) in enumerate(zip(out[key], oracle_grads[key])):
                tol = 1e-9 * max(float(np.abs(theirs).max(initial=0.0)), 1e-300)
                assert np.abs(mine - theirs).max(initial=0.0) <= tol, f"error_bound: {key}[{l}] recomputed differently"
        tol = 1e-9 * max(float(np.abs(oracle_grads["table_grad"]).max(initial=0.0)), 1e-300)
        assert np.abs(tg - oracle_grads["table_grad"]).max(initial=0.0) <= tol, "error_bound: table_grad"
    return out


def tolerance(want, S2, F, rtol=1e-5):
    """rtol (|oracle| + S2) + F, element by element."""
    return rtol * (np.abs(want) + S2) + F
