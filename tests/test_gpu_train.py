"""Training step on the GPU (fp32) against the fp64 oracle, through the C ABI:
loss, every MLP gradient, the row-sorted embedding gradients (bit-exact row
set and counts), the SGD update of touched rows only, and bit-reproducibility.

Two checks per gradient tensor (train_checks.py):
  1. element by element, |gpu - oracle| <= 1e-5 (|oracle| + S2) + F, with S2
     the size of the gradient's sum carried two operations back and F what
     ReLU units within rounding of their kink may move it by (error_bound.py);
  2. the fp32 error budget: the 50/90/99 % quantiles and the maximum of
     |gpu - oracle| may be at most 16x those of the same step run in plain fp32
     by PyTorch on the CPU in two summation orders (fp32_budget.py).
The SGD updates are checked as the change of the parameters, against -lr times
the GPU's own gradient to fp32 rounding and against -lr times the oracle's
gradient with the gradient's tolerance; a large learning rate makes every
update far larger than the rounding of the parameters. Planted mistakes in the
oracle's expected values (one gradient column or row 5 % off, one embedding row
5 % off, the learning rate's sign flipped) must fail these checks.
"""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
import error_bound as EB
import train_checks as TC
from fp32_budget import budget_refs, check_within_budget
from gpucase import GpuModel, to_np
from oracle import oracle as O
from synth import CONFIGS, gen, shrink

pytestmark = pytest.mark.gpu

RTOL = 1e-5


def _cases():
    tr = CONFIGS["train"]
    return {
        "train-small": shrink(tr, B=300, rows_cap=3000),
        "train-mix": shrink(tr, B=97, rows_cap=400).with_(bag="mix", seed=2),
        "tiny-train": CONFIGS["tiny"].with_(training=True, B=203),
        "train-hot-rows": shrink(tr, B=2000, rows_cap=50),   # long segments: many occurrences per row
        "train-d64": shrink(tr, B=333, rows_cap=2000).with_(d=64, bottom=(13, 256, 64), top=(415, 256, 1), seed=5),
    }


CASES = _cases()


class Trainer:
    def __init__(self, cfg):
        self.cfg = cfg
        self.g = GpuModel(cfg, training=True)
        self.batch = gen.make_batches(cfg, (0,))[0]
        self.bt = {k: torch.from_numpy(v).cuda() for k, v in
                   (("dense", self.batch.dense), ("offsets", self.batch.offsets), ("indices", self.batch.indices),
                    ("labels", self.batch.labels))}
        self.nnz = self.batch.indices.size
        g = self.g
        self.grads = torch.zeros(E.dlrm_grads_size(g.T, g.bot, g.top, cfg.B, self.nnz), dtype=torch.uint8, device="cuda")
        self.off = E.dlrm_grads_offsets(g.T, g.bot, g.top, cfg.B, self.nnz)

    def backward(self):
        g, cfg = self.g, self.cfg
        loss = torch.zeros(1, device="cuda")
        y = torch.zeros(cfg.B, device="cuda")
        E.dlrm_backward(g.T, g.bot, g.top, cfg.B, self.bt["dense"], self.bt["offsets"], self.bt["indices"],
                        self.bt["labels"], self.grads, g.ws, loss=loss, y_hat=y)
        st = E.dlrm_check_error(g.ws)
        assert st[0] == 0, st
        return float(loss.item()), to_np(y)

    def dense_grads(self):
        g, o = self.g, self.off
        out = {}
        for key, mlp in (("bot", g.bot), ("top", g.top)):
            out[key + "_dW"] = [to_np(E.grads_view(self.grads, o[key + "_dW"][l], (mlp.dims[l + 1], E.dlrm_ld(mlp.dims[l], "f32"))))[:, :mlp.dims[l]]
                                for l in range(len(mlp.Ws))]
            out[key + "_db"] = [to_np(E.grads_view(self.grads, o[key + "_db"][l], (mlp.dims[l + 1],)))
                                for l in range(len(mlp.Ws))]
        return out


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    cfg = CASES[request.param].with_(name=request.param)
    t = Trainer(cfg)
    model = O.model_from_config(cfg)
    args = (model, t.batch.dense, t.batch.offsets, t.batch.indices, t.batch.labels)
    ref = O.train_grads(*args)
    ref["bound"] = EB.bounds(*args, oracle_grads=ref)
    ref["f32"] = budget_refs(*args)
    return cfg, t, model, ref


DENSE_KEYS = ("bot_dW", "bot_db", "top_dW", "top_db")


def _check_dense(cfg, grads, ref, want=None):
    want = want or ref
    bd = ref["bound"]
    for key in DENSE_KEYS:
        for l, gg in enumerate(grads[key]):
            TC.check_grad_and_budget(gg, want[key][l], bd[key + "_S2"][l], bd[key + "_F"][l],
                                     [r[key][l] for r in ref["f32"]], f"{cfg.name} {key}[{l}]")


def _row_grads(t):
    g, cfg = t.g, t.cfg
    rows = torch.full((max(t.nnz, 1),), 0xFFFFFFF, dtype=torch.int32, device="cuda")
    rg = torch.zeros((max(t.nnz, 1), cfg.d), device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    E.dlrm_embedding_row_grads(g.T, g.bot, g.top, cfg.B, t.nnz, t.grads, rows, rg, n)
    torch.cuda.synchronize()
    nr = int(n.item())
    return rows.cpu().numpy()[:nr].astype(np.int64), to_np(rg)[:nr]


def _check_rows(cfg, got_rows, rg, ref, want_tg=None):
    want_tg = ref["table_grad"] if want_tg is None else want_tg
    touched = np.nonzero(ref["row_count"])[0]
    assert got_rows.size == touched.size
    assert np.array_equal(got_rows, touched), "touched rows must match bit-exactly, in increasing order"
    bd = ref["bound"]
    TC.check_grad_and_budget(rg, want_tg[touched], bd["table_grad_S2"][touched], bd["table_grad_F"][touched],
                             [r["table_grad"][touched] for r in ref["f32"]], f"{cfg.name} row grads")


def test_loss_and_dense_gradients(case):
    cfg, t, model, ref = case
    loss, y = t.backward()
    assert abs(loss - ref["loss"]) <= RTOL * abs(ref["loss"]), (loss, ref["loss"])
    assert np.abs(y - ref["y_hat"]).max() <= RTOL * 1.0
    check_within_budget(y, ref["y_hat"], [r["y_hat"] for r in ref["f32"]], f"{cfg.name} y_hat")
    _check_dense(cfg, t.dense_grads(), ref)


def test_embedding_row_gradients_and_bookkeeping(case):
    cfg, t, model, ref = case
    t.backward()
    got_rows, rg = _row_grads(t)
    _check_rows(cfg, got_rows, rg, ref)


def test_planted_gradient_mistakes_fail_the_checks(case):
    """The same GPU gradients against the oracle's, with one mistake planted in the oracle's expected
    values (CPU side): one weight-gradient column 5 % off, one weight-gradient row 5 % off, one touched
    embedding row 5 % off. Each must fail."""
    cfg, t, model, ref = case
    t.backward()
    grads = t.dense_grads()
    got_rows, rg = _row_grads(t)
    key, l = "top_dW", 0
    for bad in (TC.corrupt_column(ref[key][l]), TC.corrupt_row(ref[key][l], int(np.argmax(np.abs(ref[key][l]).sum(1))))):
        want = dict(ref)
        want[key] = list(ref[key])
        want[key][l] = bad
        with pytest.raises(AssertionError):
            _check_dense(cfg, grads, ref, want)
    hot = int(np.argmax(ref["row_count"]))
    with pytest.raises(AssertionError):
        _check_rows(cfg, got_rows, rg, ref, TC.corrupt_row(ref["table_grad"], hot))


LR_LARGE = 1000.0     # every update far above the rounding of the parameters it changes


def _snapshot(g):
    return g.tables.clone(), [w.clone() for w in g.bot.Ws + g.top.Ws], [b.clone() for b in g.bot.bs + g.top.bs]


def _restore(g, snap):
    tables, Ws, bs = snap
    g.tables.copy_(tables)
    for w, w0 in zip(g.bot.Ws + g.top.Ws, Ws):
        w.copy_(w0)
    for b, b0 in zip(g.bot.bs + g.top.bs, bs):
        b.copy_(b0)
    torch.cuda.synchronize()


def _sgd_step(t, lr):
    """backward, the GPU's own gradients, then dlrm_sparse_sgd; returns (before, after, gpu gradients)."""
    g, cfg = t.g, t.cfg
    snap = _snapshot(g)
    t.backward()
    own = t.dense_grads()
    own["rows"], own["row_grads"] = _row_grads(t)
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    E.dlrm_sparse_sgd(g.T, g.bot, g.top, cfg.B, t.nnz, lr, t.grads, n)
    torch.cuda.synchronize()
    own["n_touched"] = int(n.item())
    after = (g.tables.cpu().double().numpy(), [to_np(w) for w in g.bot.Ws + g.top.Ws],
             [to_np(b) for b in g.bot.bs + g.top.bs])
    before = (snap[0].cpu().double().numpy(), [to_np(w) for w in snap[1]], [to_np(b) for b in snap[2]])
    _restore(g, snap)
    return before, after, own


def _check_sgd(cfg, model, ref, before, after, own, lr, lr_oracle=None):
    """Touched rows and every MLP parameter move by -lr g; untouched rows do not move."""
    lr_oracle = lr if lr_oracle is None else lr_oracle
    lr32 = float(np.float32(lr))
    bd = ref["bound"]
    touched = ref["row_count"] > 0
    assert own["n_touched"] == int(touched.sum())
    assert np.array_equal(after[0][~touched], before[0][~touched]), "untouched rows must be bit-identical"
    rows = own["rows"]
    TC.check_update_own(before[0][rows], after[0][rows], own["row_grads"], lr32, f"{cfg.name} rows vs own gradient")
    TC.check_update_oracle(before[0][touched], after[0][touched], ref["table_grad"][touched] * (lr_oracle / lr),
                           bd["table_grad_S2"][touched], bd["table_grad_F"][touched], lr32, f"{cfg.name} rows vs oracle")
    nb = len(model.bot_W)
    for i, (W0, W1) in enumerate(zip(before[1], after[1])):
        key, l = ("bot", i) if i < nb else ("top", i - nb)
        k = (model.bot_W if key == "bot" else model.top_W)[l].shape[1]
        assert np.all(W1[:, k:] == 0), "weight padding untouched"
        TC.check_update_own(W0[:, :k], W1[:, :k], own[key + "_dW"][l], lr32, f"{cfg.name} {key} W[{l}] vs own")
        TC.check_update_oracle(W0[:, :k], W1[:, :k], ref[key + "_dW"][l] * (lr_oracle / lr), bd[key + "_dW_S2"][l],
                               bd[key + "_dW_F"][l], lr32, f"{cfg.name} {key} W[{l}] vs oracle")
        b0, b1 = before[2][i], after[2][i]
        TC.check_update_own(b0, b1, own[key + "_db"][l], lr32, f"{cfg.name} {key} b[{l}] vs own")
        TC.check_update_oracle(b0, b1, ref[key + "_db"][l] * (lr_oracle / lr), bd[key + "_db_S2"][l],
                               bd[key + "_db_F"][l], lr32, f"{cfg.name} {key} b[{l}] vs oracle")


@pytest.mark.parametrize("lr", ["config", "large"])
def test_sparse_and_dense_sgd_updates(case, lr):
    cfg, t, model, ref = case
    lr = cfg.lr if lr == "config" else LR_LARGE
    before, after, own = _sgd_step(t, lr)
    _check_sgd(cfg, model, ref, before, after, own, lr)


def test_planted_sgd_sign_mistake_fails(case):
    """The oracle's update with the learning rate's sign flipped (planted on the CPU side) must fail
    against the GPU's update."""
    cfg, t, model, ref = case
    before, after, own = _sgd_step(t, LR_LARGE)
    with pytest.raises(AssertionError):
        _check_sgd(cfg, model, ref, before, after, own, LR_LARGE, lr_oracle=-LR_LARGE)


def test_training_step_is_bit_reproducible():
    cfg = CASES["train-mix"]
    results = []
    for _ in range(2):
        t = Trainer(cfg)
        for _step in range(2):
            t.backward()
            E.dlrm_sparse_sgd(t.g.T, t.g.bot, t.g.top, cfg.B, t.nnz, cfg.lr, t.grads)
        torch.cuda.synchronize()
        results.append([t.g.tables.cpu()] + [w.cpu() for w in t.g.bot.Ws + t.g.top.Ws + t.g.bot.bs + t.g.top.bs])
    for a, b in zip(*results):
        assert torch.equal(a, b)


def test_training_step_with_skipped_indices():
    """Out-of-range indices in a training batch (the fused interaction's forward validates the bags): they
    are skipped exactly where the oracle skips them, counted once per occurrence by the forward, and the
    loss and y_hat still follow the oracle."""
    cfg = shrink(CONFIGS["train"], B=150, rows_cap=1500).with_(name="train-oob", bag="mix", seed=11)
    t = Trainer(cfg)
    idx = t.batch.indices.copy()
    idx[::9] = 10 ** 7                                  # past the end of every table
    t.bt["indices"] = torch.from_numpy(idx).cuda()
    g = t.g
    loss = torch.zeros(1, device="cuda")
    y = torch.zeros(cfg.B, device="cuda")
    E.dlrm_backward(g.T, g.bot, g.top, cfg.B, t.bt["dense"], t.bt["offsets"], t.bt["indices"], t.bt["labels"],
                    t.grads, g.ws, loss=loss, y_hat=y)
    st = E.dlrm_check_error(g.ws)
    ref = O.train_grads(O.model_from_config(cfg), t.batch.dense, t.batch.offsets, idx, t.batch.labels)
    n_oob = int(ref["counts"][0])
    assert n_oob == idx[::9].size
    assert st[0] == E.ERR_INDEX_OOB and st[2] == n_oob, (st, n_oob)
    assert abs(float(loss.item()) - ref["loss"]) <= RTOL * abs(ref["loss"])
    assert np.abs(to_np(y) - ref["y_hat"]).max() <= RTOL
