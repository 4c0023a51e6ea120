"""Error budget of fp32 arithmetic for the training step.

The GPU training step runs in fp32; its gradients differ from the fp64 oracle
by rounding, amplified by cancellation in batch sums and by ReLU pre-
activations that rounding moves across 0. How large that difference may be is
measured, not guessed: the same model is run forward and backward in fp32 by
PyTorch on the CPU (torch.nn.functional.embedding_bag, dense matmuls,
autograd), and its distance to the fp64 oracle, per tensor and per quantile,
is the budget (the worse of two summation orders, see budget_refs). This module is a yardstick of fp32 precision only; the values
the GPU is compared with are the oracle's. (The 3xTF32 pair product that the
GPU's GEMMs use is available here too, for study: tf32x3=True.)

Reading of the training step used here (as in the oracle): ReLU after every
bottom layer and every hidden top layer, the last top layer linear, Z = the
strict lower triangle of X X^T in row-major order over X = [x_dense; e_1..e_K],
concat [x_dense, Z], loss = mean(softplus(z) - y z)."""
import numpy as np
import torch


def _tf32_trunc(x):
    return (x.view(torch.int32) & -8192).view(torch.float32)


def _tf32_round(x):
    # nearest TF32 value, ties away from zero (add half a TF32 unit to the magnitude, clear the low 13 bits)
    return ((x.view(torch.int32) + 4096) & -8192).view(torch.float32)


class _MM3(torch.autograd.Function):
    """a @ b.T with every product taken as a_lo b_hi + a_hi b_lo + a_hi b_hi (TF32 pairs, fp32 sums)."""

    @staticmethod
    def forward(ctx, a, b):
        ctx.save_for_backward(a, b)
        return _mm3(a, b.t())

    @staticmethod
    def backward(ctx, g):
        a, b = ctx.saved_tensors
        return _mm3(g, b), _mm3(g.t(), a)


def _mm3(x, y):
    xh, yh = _tf32_round(x), _tf32_round(y)
    xl, yl = _tf32_trunc(x - xh), _tf32_trunc(y - yh)
    return (xl @ yh + xh @ yl) + xh @ yh


class _MM1(torch.autograd.Function):
    """a @ b.T with both operands rounded to TF32 (the precision a single TF32 product keeps)."""

    @staticmethod
    def forward(ctx, a, b):
        ctx.save_for_backward(a, b)
        return _tf32_round(a) @ _tf32_round(b).t()

    @staticmethod
    def backward(ctx, g):
        a, b = ctx.saved_tensors
        return _tf32_round(g) @ _tf32_round(b), _tf32_round(g.t()) @ _tf32_round(a)


def train_grads_f32(model, dense, offsets, indices, labels, tf32x3=False, tf32x1=False, reverse_d=False):
    """Loss, y_hat and every gradient of the fp32 training step (CPU, float32). With tf32x3 the
    matrix products of the MLPs (forward and both gradients) are taken as 3xTF32 pair products,
    with tf32x1 as single TF32 products. reverse_d sums the interaction's dot products over the
    embedding dimension in reverse order (the same values, another fp32 rounding)."""
    f = torch.float32
    if tf32x3:
        mm = lambda a, W: _MM3.apply(a, W)  # noqa: E731
    elif tf32x1:
        mm = lambda a, W: _MM1.apply(a, W)  # noqa: E731
    else:
        mm = lambda a, W: a @ W.t()  # noqa: E731
    K, d = model.K, model.d
    B = dense.shape[0]
    tables = torch.tensor(model.tables, dtype=f, requires_grad=True)
    bW = [torch.tensor(w, dtype=f, requires_grad=True) for w in model.bot_W]
    bb = [torch.tensor(b, dtype=f, requires_grad=True) for b in model.bot_b]
    tW = [torch.tensor(w, dtype=f, requires_grad=True) for w in model.top_W]
    tb = [torch.tensor(b, dtype=f, requires_grad=True) for b in model.top_b]
    x = torch.tensor(np.asarray(dense), dtype=f)
    for W, b in zip(bW, bb):
        x = torch.relu(mm(x, W) + b)
    base = np.concatenate([[0], np.cumsum(model.rows)])[:-1]
    offs = np.asarray(offsets, np.int64)
    idx = np.asarray(indices, np.int64)
    pooled = []
    for k in range(K):
        lo, hi = offs[k * B], offs[(k + 1) * B]
        rows = torch.tensor(idx[lo:hi] + base[k], dtype=torch.int64)
        o = torch.tensor(offs[k * B:(k + 1) * B] - lo, dtype=torch.int64)
        pooled.append(torch.nn.functional.embedding_bag(rows, tables, o, mode="sum"))
    X = torch.stack([x] + pooled, dim=1)                 # [B][K+1][d]
    if reverse_d:
        X = X.flip(2)
    G = X @ X.transpose(1, 2)
    ii, jj = np.tril_indices(K + 1, -1)                 # row-major strict lower triangle: (1,0),(2,0),(2,1),...
    Z = G[:, torch.tensor(ii), torch.tensor(jj)]
    h = torch.cat([x, Z], dim=1)
    for l, (W, b) in enumerate(zip(tW, tb)):
        h = mm(h, W) + b
        if l < len(tW) - 1:
            h = torch.relu(h)
    z = h[:, 0]
    y = torch.tensor(np.asarray(labels), dtype=f)
    loss = (torch.nn.functional.softplus(z) - y * z).mean()
    loss.backward()
    g = lambda ts: [t.grad.double().numpy() for t in ts]  # noqa: E731
    return {"loss": float(loss.detach()), "y_hat": torch.sigmoid(z).detach().double().numpy(), "bot_dW": g(bW),
            "bot_db": g(bb), "top_dW": g(tW), "top_db": g(tb), "table_grad": tables.grad.double().numpy()}


def budget_refs(model, dense, offsets, indices, labels):
    """Two plain-fp32 evaluations of the training step that differ only in summation order. Where
    ReLU pre-activations sit within rounding of 0 (batches with many shared embedding rows), which
    of them flip depends on that order, and so does the shape of the error distribution: the
    budget is the worse of the two."""
    args = (model, dense, offsets, indices, labels)
    return [train_grads_f32(*args), train_grads_f32(*args, reverse_d=True)]


def check_within_budget(got, want, refs, what, factor=16.0, allowance=None):
    """The 50% and 90% quantiles of |got - want| (the 99% one from 1000 entries up) and its maximum
    are at most `factor` times the largest of the same quantiles of |ref - want| over the fp32
    references `refs` (one array or a list), plus 1e-7 of max|want| (one fp32 rounding of the
    largest entry). `allowance` (element-wise, optional) is what a ReLU unit at the kink may move an
    entry by when it takes the other branch (error_bound.py); the maximum is taken over the excess
    max(|got - want| - allowance, 0), since a flip that the fp32 references happened not to take is not
    a loss of precision. Tensors of fewer than 64 entries have no error distribution to compare; the
    element-wise bound covers them."""
    refs = refs if isinstance(refs, (list, tuple)) else [refs]
    got, want = (np.asarray(a, np.float64).ravel() for a in (got, want))
    if want.size < 64:
        return
    floor = 1e-7 * float(np.abs(want).max(initial=0.0))
    e = np.abs(got - want)
    e32 = [np.abs(np.asarray(r, np.float64).ravel() - want) for r in refs]
    for q in (0.5, 0.9) + ((0.99,) if want.size >= 1000 else ()):
        a = float(np.quantile(e, q))
        b = max(float(np.quantile(x, q)) for x in e32)
        assert a <= factor * b + floor, (f"{what}: error quantile {q} = {a:.3g} exceeds {factor} x fp32 budget "
                                         f"{b:.3g} (+{floor:.2g})")
    excess = e if allowance is None else np.maximum(e - np.asarray(allowance, np.float64).ravel(), 0.0)
    a = float(excess.max())
    b = max(float(x.max()) for x in e32)
    assert a <= factor * b + floor, (f"{what}: largest error {a:.3g} (beyond the kink allowance) exceeds {factor} x "
                                     f"the fp32 references' largest {b:.3g} (+{floor:.2g})")
