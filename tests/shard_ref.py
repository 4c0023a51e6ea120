"""fp64 numpy values of the training step that the oracle keeps internal, for the sharding tests: the
gradient of the mean loss with respect to every pooled vector (dE [B][K][d]) and every MLP parameter.

Plain definition (ReLU after every bottom layer and every hidden top layer, the last top layer linear,
Z the strict lower triangle of X X^T in row-major order over X = [x_dense; e_1..e_K], concat
[x_dense, Z], loss the batch mean of softplus(z) - y z), computed from given pooled vectors. The tests
check it against the oracle (its gradients, and dE summed over each row's occurrences against the
oracle's table gradients) before relying on it. Test infrastructure only."""
import numpy as np


def step_grads(model, dense, pooled, labels):
    """Returns (loss, {"bot_dW", "bot_db", "top_dW", "top_db": lists, "dE": [B][K][d]}) for pooled vectors
    pooled [B][K][d] (fp64)."""
    dense = np.asarray(dense, np.float64)
    labels = np.asarray(labels, np.float64)
    B = dense.shape[0]
    K, d = model.K, model.d
    ii, jj = np.tril_indices(K + 1, -1)
    acts, x = [dense], dense
    for W, b in zip(model.bot_W, model.bot_b):
        x = np.maximum(x @ W.T + b, 0.0)
        acts.append(x)
    X = np.concatenate([x[:, None, :], pooled], 1)
    h = np.concatenate([x, np.einsum("bid,bjd->bij", X, X)[:, ii, jj]], 1)
    tacts = [h]
    n_top = len(model.top_W)
    for l, (W, b) in enumerate(zip(model.top_W, model.top_b)):
        h = h @ W.T + b
        if l < n_top - 1:
            h = np.maximum(h, 0.0)
        tacts.append(h)
    z = h[:, 0]
    loss = float(np.mean(np.logaddexp(0.0, z) - labels * z))
    dY = ((1.0 / (1.0 + np.exp(-z)) - labels) / B)[:, None]
    g = {"top_dW": [None] * n_top, "top_db": [None] * n_top, "bot_dW": [None] * len(model.bot_W),
         "bot_db": [None] * len(model.bot_W)}
    for l in range(n_top - 1, -1, -1):
        g["top_dW"][l] = dY.T @ tacts[l]
        g["top_db"][l] = dY.sum(0)
        dA = dY @ model.top_W[l]
        dY = np.where(tacts[l] > 0, dA, 0.0) if l > 0 else dA
    dc = dY
    S = np.zeros((B, K + 1, K + 1))
    S[:, ii, jj] = dc[:, d:]
    S = S + S.transpose(0, 2, 1)
    dX = np.einsum("bij,bjd->bid", S, X)
    dX[:, 0, :] += dc[:, :d]
    g["dE"] = dX[:, 1:, :]
    dY = np.where(acts[-1] > 0, dX[:, 0, :], 0.0)
    for l in range(len(model.bot_W) - 1, -1, -1):
        g["bot_dW"][l] = dY.T @ acts[l]
        g["bot_db"][l] = dY.sum(0)
        if l > 0:
            dY = np.where(acts[l] > 0, dY @ model.bot_W[l], 0.0)
    return loss, g


def scatter_rows(dE, model, offsets, indices):
    """Sum of dE[b][k] over the valid occurrences of every table row (occurrence order): [sum rows][d]."""
    B = dE.shape[0]
    K, d = model.K, model.d
    base = np.concatenate([[0], np.cumsum(model.rows)])[:-1]
    out = np.zeros((int(np.sum(model.rows)), d))
    offs = np.asarray(offsets, np.int64)
    for k in range(K):
        for b in range(B):
            for p in range(offs[k * B + b], offs[k * B + b + 1]):
                r = int(indices[p])
                if 0 <= r < model.rows[k]:
                    out[base[k] + r] += dE[b, k]
    return out
