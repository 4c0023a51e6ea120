"""Pins of the fp64 oracle to facts outside itself.

Each ``pin_*`` function takes a loaded oracle library and raises
AssertionError when the oracle disagrees with:
  - hand-derived worked examples under tests/golden/ (each cites the passage);
  - closed forms and invariants the definition fixes (Z has K(K+1)/2 terms,
    X X^T is symmetric, orthonormal rows give Z = 0, equal rows give |v|^2,
    d = 1 gives products, empty bags pool to 0, zero last layer gives 0.5);
  - independent library routines on the same inputs (torch fp64
    ``embedding_bag``, ``X @ X^T`` + ``numpy.tril_indices``, ``linear``,
    ``binary_cross_entropy_with_logits`` and autograd for every gradient).

The same functions run against deliberately broken copies of the oracle in
test_oracle_mutants.py, to show that plausible mistakes are caught.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch
import torch.nn.functional as F

from oracle import oracle as O
from synth import CONFIGS, gen, shrink

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _close(a, b, rtol=1e-12, atol=1e-12, what=""):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.abs(a - b)
    lim = atol + rtol * np.abs(b)
    assert np.all(err <= lim), f"{what}: max err {err.max()} (worst at {np.unravel_index(np.argmax(err - lim), err.shape)})"


# ----------------------------------------------------------------- torch fp64 reference pieces

def torch_pool(tables64, rows, d, B, offsets, indices):
    """Sum-pooled bags via torch.nn.functional.embedding_bag, one call per table."""
    rows = np.asarray(rows, np.int64)
    base = np.concatenate([[0], np.cumsum(rows)[:-1]])
    K = rows.size
    offs = np.asarray(offsets, np.int64)
    out = torch.zeros(B, K, d, dtype=torch.float64)
    T = torch.from_numpy(np.asarray(tables64, np.float64).reshape(-1, d))
    for k in range(K):
        s, e = offs[k * B], offs[(k + 1) * B]
        inp = torch.from_numpy(np.asarray(indices[s:e], np.int64))
        o = torch.from_numpy(offs[k * B:k * B + B] - s)
        w = T[base[k]:base[k] + rows[k]]
        out[:, k, :] = F.embedding_bag(inp, w, o, mode="sum")
    return out


def torch_interact(x, pooled):
    X = torch.cat([x[:, None, :], pooled], dim=1)
    G = X @ X.transpose(1, 2)
    li, lj = np.tril_indices(X.shape[1], -1)
    return torch.cat([x, G[:, li, lj]], dim=1)


def torch_model_forward(model: O.Model, dense, offsets, indices, params=None):
    """Logits of the whole model from torch library routines (fp64). ``params`` allows autograd leaves."""
    p = params or torch_params(model)
    x = torch.from_numpy(np.asarray(dense, np.float64))
    for W, b in zip(p["bot_W"], p["bot_b"]):
        x = torch.relu(F.linear(x, W, b))
    B = x.shape[0]
    pooled = torch_pool_t(p["tables"], model.rows, model.d, B, offsets, indices)
    c = torch_interact(x, pooled)
    n = len(p["top_W"])
    for l, (W, b) in enumerate(zip(p["top_W"], p["top_b"])):
        c = F.linear(c, W, b)
        if l < n - 1:
            c = torch.relu(c)
    return c[:, 0]


def torch_pool_t(T, rows, d, B, offsets, indices):
    rows = np.asarray(rows, np.int64)
    base = np.concatenate([[0], np.cumsum(rows)[:-1]])
    offs = np.asarray(offsets, np.int64)
    cols = []
    for k in range(rows.size):
        s, e = offs[k * B], offs[(k + 1) * B]
        inp = torch.from_numpy(np.asarray(indices[s:e], np.int64))
        o = torch.from_numpy(offs[k * B:k * B + B] - s)
        cols.append(F.embedding_bag(inp, T[base[k]:base[k] + rows[k]], o, mode="sum"))
    return torch.stack(cols, dim=1)


def torch_params(model: O.Model, grad=False):
    t = lambda a: torch.tensor(np.asarray(a), dtype=torch.float64, requires_grad=grad)  # noqa: E731
    return {"bot_W": [t(w) for w in model.bot_W], "bot_b": [t(b) for b in model.bot_b],
            "top_W": [t(w) for w in model.top_W], "top_b": [t(b) for b in model.top_b],
            "tables": t(model.tables)}


def tiny_case(bag="mix", B=24, seed=3):
    cfg = shrink(CONFIGS["tiny"], B=B, rows_cap=40).with_(bag=bag, seed=seed)
    batch = gen.make_batches(cfg, (0,))[0]
    model = O.model_from_config(cfg)
    return cfg, batch, model


# ----------------------------------------------------------------- pins

def pin_embbag_golden(lib):
    g = _golden("embbag_4x2.json")
    pooled, blen, counts = O.embbag(np.array(g["table"], float), g["rows"], g["d"], g["B"], g["offsets"], g["indices"], lib=lib)
    _close(pooled, g["pooled"], what="golden pooled")
    assert blen.tolist() == g["bag_len"], blen
    assert counts == (0, 0)


def pin_embbag_closed_forms(lib):
    rng = np.random.default_rng(7)
    T = rng.standard_normal((10, 5))
    # one-hot bag = the row; n repeats = n * row; empty = 0
    offsets = [0, 1, 1, 8]
    indices = [4, 6, 6, 6, 6, 6, 6, 6]
    pooled, blen, _ = O.embbag(T, [10], 5, 3, offsets, indices, lib=lib)
    assert np.array_equal(pooled[0, 0], T[4])
    assert np.array_equal(pooled[1, 0], np.zeros(5))
    _close(pooled[2, 0], 7 * T[6], rtol=1e-15, what="7 repeats")
    assert blen.tolist() == [1, 0, 7]


def pin_embbag_vs_library(lib):
    cfg, batch, model = tiny_case(bag="mix")
    pooled, blen, counts = O.embbag(model.tables, cfg.rows, cfg.d, cfg.B, batch.offsets, batch.indices, lib=lib)
    ref = torch_pool(model.tables, cfg.rows, cfg.d, cfg.B, batch.offsets, batch.indices).numpy()
    _close(pooled, ref, rtol=1e-13, atol=1e-15, what="embbag vs torch.embedding_bag")
    assert np.array_equal(blen, np.diff(batch.offsets.astype(np.int64)))
    assert counts == (0, 0)
    # count-matrix route: pooled[b, k] = sum_r C[b, k, r] T_k[r]
    base = gen.row_base(cfg)
    Cm = np.zeros((cfg.B * cfg.K, model.tables.shape[0]))
    offs = batch.offsets.astype(np.int64)
    for k in range(cfg.K):
        for b in range(cfg.B):
            for p in range(offs[k * cfg.B + b], offs[k * cfg.B + b + 1]):
                Cm[b * cfg.K + k, base[k] + batch.indices[p]] += 1
    _close(pooled.reshape(cfg.B * cfg.K, cfg.d), Cm @ model.tables, rtol=1e-13, atol=1e-15, what="count matrix")


def pin_embbag_invalid(lib):
    T = np.arange(12, dtype=float).reshape(6, 2)
    # table 0 has 2 rows, table 1 has 4 rows; B = 2
    offsets = [0, 2, 3, 5, 6]
    indices = [1, 2, -1, 3, 0, 4]   # 2 out of table 0's range, -1 negative, 4 out of table 1's range
    pooled, blen, counts = O.embbag(T, [2, 4], 2, 2, offsets, indices, lib=lib)
    assert counts == (3, 0), counts
    assert np.array_equal(pooled[0, 0], T[1])
    assert np.array_equal(pooled[1, 0], np.zeros(2))
    assert np.array_equal(pooled[0, 1], T[2 + 3] + T[2 + 0])
    assert np.array_equal(pooled[1, 1], np.zeros(2))
    bad = [0, 3, 1, 5, 4]           # bag 1 decreasing, bag 3 beyond nnz? (5 <= 6 ok), bag 2: 1..5 fine
    pooled, blen, counts = O.embbag(T, [2, 4], 2, 2, bad, [0, 1, 0, 1, 2, 3], lib=lib)
    assert counts[1] == 2, counts   # bag (0,1): 3 -> 1 decreasing; bag (1,1): 5 -> 4 decreasing
    assert np.array_equal(pooled[1, 0], np.zeros(2)) and np.array_equal(pooled[1, 1], np.zeros(2))


def pin_interact_golden(lib):
    g = _golden("interaction_3x2.json")
    out = O.interact(np.array(g["x_dense"], float), np.array(g["pooled"], float), lib=lib)
    _close(out, g["concat"], what="golden interaction")


def pin_interact_closed_forms(lib):
    # size: d + K(K+1)/2 for every K
    for K in (1, 2, 5, 26):
        out = O.interact(np.ones((1, 3)), np.ones((1, K, 3)), lib=lib)
        assert out.shape == (1, 3 + K * (K + 1) // 2)
    # orthonormal rows -> Z = 0
    I = np.eye(6)
    out = O.interact(I[None, 0], I[None, 1:], lib=lib)
    assert np.array_equal(out[0, 6:], np.zeros(15)) and np.array_equal(out[0, :6], I[0])
    # all rows equal v -> every term |v|^2
    v = np.array([0.5, -1.25, 2.0])
    out = O.interact(v[None], np.tile(v, (1, 4, 1)), lib=lib)
    _close(out[0, 3:], np.full(10, v @ v), what="equal rows")
    # d = 1 -> Z_ij = x_i x_j in row-major strict-lower order
    x = np.array([2.0, -3.0, 5.0, 7.0])
    out = O.interact(x[None, :1], x[None, 1:, None], lib=lib)
    want = [x[i] * x[j] for i in range(4) for j in range(i)]
    _close(out[0, 1:], want, what="d=1 products")


def pin_interact_vs_library_and_symmetry(lib):
    rng = np.random.default_rng(11)
    B, K, d = 5, 7, 9
    x, e = rng.standard_normal((B, d)), rng.standard_normal((B, K, d))
    out = O.interact(x, e, lib=lib)
    ref = torch_interact(torch.from_numpy(x), torch.from_numpy(e)).numpy()
    _close(out, ref, rtol=1e-13, atol=1e-14, what="interaction vs torch tril(X X^T, -1)")
    # symmetry of X X^T: reversing the row order maps Z_ij to Z_(n-1-j)(n-1-i)
    X = np.concatenate([x[:, None], e], axis=1)
    Xr = X[:, ::-1]
    out_r = O.interact(np.ascontiguousarray(Xr[:, 0]), np.ascontiguousarray(Xr[:, 1:]), lib=lib)
    n = K + 1
    pos = {}
    p = 0
    for i in range(1, n):
        for j in range(i):
            pos[(i, j)] = p
            p += 1
    for (i, j), q in pos.items():
        ii, jj = n - 1 - j, n - 1 - i
        _close(out_r[:, d + pos[(ii, jj)]], out[:, d + q], rtol=1e-13, atol=1e-14, what="symmetry")


def pin_mlp(lib):
    rng = np.random.default_rng(5)
    dims = [13, 20, 7, 3]
    Ws = [rng.standard_normal((dims[l + 1], dims[l])) for l in range(3)]
    bs = [rng.standard_normal(dims[l + 1]) for l in range(3)]
    x = rng.standard_normal((6, 13))
    for relu_last in (False, True):
        out = O.mlp(Ws, bs, x, relu_last, lib=lib)
        t = torch.from_numpy(x)
        for l in range(3):
            t = F.linear(t, torch.from_numpy(Ws[l]), torch.from_numpy(bs[l]))
            if l < 2 or relu_last:
                t = torch.relu(t)
        _close(out, t.numpy(), rtol=1e-13, atol=1e-14, what=f"mlp relu_last={relu_last}")
    # identity weights with zero bias pass non-negative values through
    xi = np.abs(rng.standard_normal((4, 5)))
    out = O.mlp([np.eye(5), np.eye(5)], [np.zeros(5), np.zeros(5)], xi, True, lib=lib)
    assert np.array_equal(out, xi)


def pin_forward_zero_last_layer(lib):
    cfg, batch, model = tiny_case(bag="one", B=16)
    model.top_W[-1][:] = 0.0
    model.top_b[-1][:] = 0.0
    y, z, _ = O.forward(model, batch.dense, batch.offsets, batch.indices, lib=lib)
    assert np.all(y == 0.5) and np.all(z == 0.0)


def pin_forward_golden(lib):
    g = _golden("forward_backward_k1d1.json")
    m = O.Model(np.array([1], np.int64), 1, np.array(g["table"], float),
                [np.array(w, float) for w in g["bot_W"]], [np.array(b, float) for b in g["bot_b"]],
                [np.array(w, float) for w in g["top_W"]], [np.array(b, float) for b in g["top_b"]])
    y, z, counts = O.forward(m, np.array(g["dense"]), g["offsets"], g["indices"], lib=lib)
    _close(y, [g["y_hat"]], what="golden y_hat")
    _close(z, [g["logit"]], what="golden logit")
    r = O.train_grads(m, np.array(g["dense"]), g["offsets"], g["indices"], np.array(g["labels"]), lib=lib)
    _close(r["loss"], g["loss"], what="golden loss")
    _close(r["top_dW"][0], g["top_dW"], what="golden top dW")
    _close(r["top_db"][0], g["top_db"], what="golden top db")
    _close(r["bot_dW"][0], g["bot_dW"], what="golden bottom dW")
    _close(r["bot_db"][0], g["bot_db"], what="golden bottom db")
    _close(r["table_grad"], g["table_grad"], what="golden table grad")


def pin_forward_vs_library(lib):
    for bag in ("one", "mix"):
        cfg, batch, model = tiny_case(bag=bag)
        y, z, counts = O.forward(model, batch.dense, batch.offsets, batch.indices, lib=lib)
        zt = torch_model_forward(model, batch.dense, batch.offsets, batch.indices).numpy()
        _close(z, zt, rtol=1e-12, atol=1e-13, what=f"forward logits vs torch ({bag})")
        _close(y, torch.sigmoid(torch.from_numpy(zt)).numpy(), rtol=1e-12, atol=1e-14, what="sigmoid")
        assert np.all((y > 0) & (y < 1))
        assert counts == (0, 0)


def pin_bce(lib):
    rng = np.random.default_rng(9)
    z = rng.standard_normal(50) * 8
    y = (rng.random(50) < 0.5).astype(float)
    ref = F.binary_cross_entropy_with_logits(torch.from_numpy(z), torch.from_numpy(y)).item()
    _close(O.bce(z, y, lib=lib), ref, rtol=1e-13, what="bce")


def pin_gradients_vs_autograd(lib):
    for bag in ("one", "mix"):
        cfg, batch, model = tiny_case(bag=bag, B=20)
        labels = (np.random.default_rng(2).random(cfg.B) < 0.5).astype(np.float64)
        r = O.train_grads(model, batch.dense, batch.offsets, batch.indices, labels, lib=lib)
        p = torch_params(model, grad=True)
        z = torch_model_forward(model, batch.dense, batch.offsets, batch.indices, params=p)
        loss = F.binary_cross_entropy_with_logits(z, torch.from_numpy(labels))
        loss.backward()
        _close(r["loss"], loss.item(), rtol=1e-13, what="loss")
        for key in ("bot_W", "bot_b", "top_W", "top_b"):
            mine = r[key[:3] + "_d" + key[4:]]
            for l, t in enumerate(p[key]):
                _close(mine[l], t.grad.numpy(), rtol=1e-10, atol=1e-14, what=f"{key}[{l}] grad ({bag})")
        _close(r["table_grad"], p["tables"].grad.numpy(), rtol=1e-10, atol=1e-14, what=f"table grad ({bag})")
        # occurrence counts = histogram of (table base + index)
        keys = np.concatenate([gen.row_base(cfg)[k] + batch.indices[batch.offsets[k * cfg.B]:batch.offsets[(k + 1) * cfg.B]]
                               for k in range(cfg.K)])
        u, c = np.unique(keys, return_counts=True)
        want = np.zeros(model.tables.shape[0], np.int64)
        want[u] = c
        assert np.array_equal(r["row_count"], want)
        assert np.all(r["table_grad"][want == 0] == 0.0)


def pin_gradients_finite_difference(lib):
    cfg, batch, model = tiny_case(bag="one", B=8)
    labels = (np.random.default_rng(4).random(cfg.B) < 0.5).astype(np.float64)
    r = O.train_grads(model, batch.dense, batch.offsets, batch.indices, labels, lib=lib)
    h = 1e-6

    def loss_of():
        _, z, _ = O.forward(model, batch.dense, batch.offsets, batch.indices, lib=lib)
        return O.bce(z, labels, lib=lib)

    probes = [("top_W", 0, (3, 5)), ("top_W", 1, (0, 7)), ("top_b", 0, (2,)), ("bot_W", 0, (4, 6)),
              ("bot_W", 1, (1, 9)), ("bot_b", 1, (3,))]
    row = int(batch.indices[0])
    probes.append(("tables", None, (row, 2)))
    for name, l, idx in probes:
        arr = getattr(model, name) if l is None else getattr(model, name)[l]
        old = arr[idx]
        arr[idx] = old + h
        up = loss_of()
        arr[idx] = old - h
        dn = loss_of()
        arr[idx] = old
        fd = (up - dn) / (2 * h)
        g = r["table_grad"][idx] if name == "tables" else r[name[:3] + "_d" + name[4:]][l][idx]
        assert abs(fd - g) <= 1e-6 * abs(g) + 1e-9, f"{name}[{l}]{idx}: fd {fd} vs {g}"


def pin_sgd(lib):
    w = np.array([1.0, -2.0, 3.5])
    g = np.array([0.5, 0.25, -1.0])
    out = O.sgd(w, g, 0.01, lib=lib)
    assert np.array_equal(out, np.array([1.0 - 0.005, -2.0 - 0.0025, 3.5 + 0.01]))


def pin_quant_golden(lib):
    # hand-worked row (tests/golden/quant_u8_row.json)
    g = _golden("quant_u8_row.json")
    codes, s, m = O.quantize_rows_u8(np.array([g["row"]], np.float32), lib)
    assert codes[0].tolist() == g["codes"], codes
    assert s[0] == np.float32(g["scale"]) and m[0] == np.float32(g["offset"]), (s, m)
    back = O.dequantize_rows_u8(codes, s, m, lib)
    _close(back[0], np.array(g["row"]), rtol=0, atol=1e-6, what="dequantised worked row")


def pin_quant_constant_row(lib):
    codes, s, m = O.quantize_rows_u8(np.full((1, 16), -0.375, np.float32), lib)
    assert s[0] == 0 and np.all(codes == 0) and m[0] == np.float32(-0.375)
    assert np.all(O.dequantize_rows_u8(codes, s, m, lib) == -0.375)


def pin_quant_rounding_bound(lib):
    # nearest code: |s q + m - v| <= s / 2; the row's min and max map to codes 0 and 255
    rng = np.random.default_rng(3)
    v = (rng.standard_normal((200, 64)) * rng.uniform(1e-3, 10, (200, 1))).astype(np.float32)
    codes, s, m = O.quantize_rows_u8(v, lib)
    back = O.dequantize_rows_u8(codes, s, m, lib)
    err = np.abs(back - v.astype(np.float64))
    assert np.all(err <= 0.5 * s[:, None] * (1 + 1e-5) + 1e-6 * np.abs(v).max(axis=1, keepdims=True))
    assert np.all(codes.min(axis=1) == 0) and np.all(codes.max(axis=1) == 255)
    assert np.all(m == v.min(axis=1))


def pin_quant_brute_force(lib):
    # the chosen code is the nearest of all 256 (up to the fp32 division that decides ties)
    rng = np.random.default_rng(4)
    v = rng.uniform(-2, 3, (64, 8)).astype(np.float32)
    codes, s, m = O.quantize_rows_u8(v, lib)
    grid = s[:, None, None].astype(np.float64) * np.arange(256)[None, None, :] + m[:, None, None]
    dist = np.abs(grid - v[:, :, None].astype(np.float64))
    chosen = np.take_along_axis(dist, codes[:, :, None].astype(np.int64), axis=2)[:, :, 0]
    assert np.all(chosen <= dist.min(axis=2) + 1e-6 * s[:, None])


def pin_concat(lib):
    # layout: columns [0, d) are x_dense, [d (k + 1), d (k + 2)) are e_k; against torch.cat
    rng = np.random.default_rng(11)
    B, K, d = 5, 4, 3
    x = rng.standard_normal((B, d))
    p = rng.standard_normal((B, K, d))
    got = O.concat(x, p, lib)
    want = torch.cat([torch.from_numpy(x)] + [torch.from_numpy(p[:, k]) for k in range(K)], dim=1).numpy()
    assert np.array_equal(got, want)
    assert np.array_equal(got[:, :d], x) and np.array_equal(got[:, d * 3:d * 4], p[:, 2])


def pin_forward_cat_vs_library(lib):
    # bottom MLP, pooling, concat, top MLP, sigmoid in torch fp64 (embedding_bag, cat, linear)
    cfg = shrink(CONFIGS["tiny"], B=20).with_(bag="mix", seed=5, interaction="cat", top=(16 * 9, 32, 1))
    batch = gen.make_batches(cfg, (0,))[0]
    model = O.model_from_config(cfg)
    y, z, counts = O.forward_cat(model, batch.dense, batch.offsets, batch.indices, lib)
    x = torch.from_numpy(np.asarray(batch.dense, np.float64))
    for W, b in zip(model.bot_W, model.bot_b):
        x = torch.relu(F.linear(x, torch.from_numpy(W), torch.from_numpy(b)))
    pooled = torch_pool(model.tables, model.rows, model.d, cfg.B, batch.offsets, batch.indices)
    h = torch.cat([x] + [pooled[:, k] for k in range(cfg.K)], dim=1)
    for l, (W, b) in enumerate(zip(model.top_W, model.top_b)):
        h = F.linear(h, torch.from_numpy(W), torch.from_numpy(b))
        if l < len(model.top_W) - 1:
            h = torch.relu(h)
    _close(z, h[:, 0].numpy(), what="concat-only logits")
    _close(y, torch.sigmoid(h[:, 0]).numpy(), what="concat-only y_hat")
    assert counts == (0, 0)


ALL_PINS = [pin_concat, pin_forward_cat_vs_library, pin_quant_golden, pin_quant_constant_row, pin_quant_rounding_bound, pin_quant_brute_force,
            pin_embbag_golden, pin_embbag_closed_forms, pin_embbag_vs_library, pin_embbag_invalid,
            pin_interact_golden, pin_interact_closed_forms, pin_interact_vs_library_and_symmetry,
            pin_mlp, pin_forward_zero_last_layer, pin_forward_golden, pin_forward_vs_library, pin_bce,
            pin_gradients_vs_autograd, pin_gradients_finite_difference, pin_sgd]
