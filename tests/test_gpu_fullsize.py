"""Full-size workloads on the GPU, in the launch configuration the benchmark
times, checked on outputs the fp64 oracle can compute one sample at a time
(the forward pass is per-sample independent; an embedding row's gradient only
involves the samples that use it) and on properties that hold at any size
(the touched-row set, bit-exact)."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
import error_bound as EB
import train_checks as TC
from gpucase import GpuModel, assert_close, scale_concat, to_np
from oracle import oracle as O
from synth import CONFIGS, gen

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _dev(batch):
    return {k: torch.from_numpy(v).cuda() for k, v in (("dense", batch.dense), ("offsets", batch.offsets),
                                                       ("indices", batch.indices))
            } | ({"labels": torch.from_numpy(batch.labels).cuda()} if batch.labels is not None else {})


def _sampled_forward(cfg, n_samples, seed):
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    bt = _dev(batch)
    y = to_np(g.forward(bt))
    assert E.dlrm_check_error(g.ws)[0] == 0
    samples = np.sort(np.random.default_rng(seed).choice(cfg.B, n_samples, replace=False))
    Bs, dense, offs, idx, _, rows, used = O.sub_batch(cfg, batch, samples)
    model = O.model_for_rows(cfg, used)
    want, _, counts = O.forward(model, dense, offs, idx)
    assert counts == (0, 0)
    assert_close(y[samples], want, cfg.table_dtype, f"{cfg.name} y_hat (sampled)")
    assert np.all((y >= 0) & (y <= 1))
    return g, batch, bt, samples, model, used


def test_large_forward_and_fused_kernel_full_size():
    cfg = CONFIGS["large"]
    g, batch, bt, samples, model, used = _sampled_forward(cfg, 512, 0)
    # the fused gather + interaction kernel alone, full batch, bf16 concat as the benchmark runs it
    x = np.random.default_rng(1).standard_normal((cfg.B, cfg.d)).astype(np.float32)
    out = torch.full((cfg.B, cfg.concat_ld), float("nan"), dtype=torch.bfloat16, device="cuda")
    E.dlrm_embbag_interact_fwd(g.T, cfg.B, bt["offsets"], bt["indices"], torch.from_numpy(x).cuda(), out,
                               cfg.concat_ld, "bf16", g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    Bs, dense, offs, idx, _, rows, used = O.sub_batch(cfg, batch, samples)
    pooled, _, _ = O.embbag(model.tables, rows, cfg.d, Bs, offs, idx)
    want = O.interact(x[samples], pooled)
    pooled_s = O.embbag(np.abs(model.tables), rows, cfg.d, Bs, offs, idx)[0]
    got = to_np(out[torch.from_numpy(samples).cuda()])
    assert_close(got[:, :cfg.concat_width], want, "bf16", "large fused concat (sampled)",
                 scale_concat(x[samples], pooled_s))
    assert np.all(got[:, cfg.concat_width:] == 0)


def test_medium_forward_full_size():
    _sampled_forward(CONFIGS["medium"], 256, 2)


def test_stress_forward_full_size():
    _sampled_forward(CONFIGS["stress"], 48, 3)


def test_train_step_full_size():
    cfg = CONFIGS["train"]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg, training=True)
    bt = _dev(batch)
    nnz = batch.indices.size
    grads = torch.zeros(E.dlrm_grads_size(g.T, g.bot, g.top, cfg.B, nnz), dtype=torch.uint8, device="cuda")
    loss = torch.zeros(1, device="cuda")
    E.dlrm_backward(g.T, g.bot, g.top, cfg.B, bt["dense"], bt["offsets"], bt["indices"], bt["labels"], grads, g.ws,
                    loss=loss)
    assert E.dlrm_check_error(g.ws)[0] == 0
    rows = torch.zeros(nnz, dtype=torch.int32, device="cuda")
    rg = torch.zeros((nnz, cfg.d), device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    E.dlrm_embedding_row_grads(g.T, g.bot, g.top, cfg.B, nnz, grads, rows, rg, n)
    torch.cuda.synchronize()
    nr = int(n.item())
    got_rows = rows[:nr].cpu().numpy().view(np.uint32).astype(np.int64)
    # touched rows: every (table base + index) of the batch, bit-exact and increasing
    base = gen.row_base(cfg)
    offs = batch.offsets.astype(np.int64)
    keys = np.concatenate([base[k] + batch.indices[offs[k * cfg.B]:offs[(k + 1) * cfg.B]] for k in range(cfg.K)])
    uk, cnt = np.unique(keys, return_counts=True)
    assert np.array_equal(got_rows, uk)
    # loss: mean over the full batch of per-sample BCE from the oracle's forward
    Bs, dense, offs2, idx2, labels, rws, used = O.sub_batch(cfg, batch, np.arange(cfg.B))
    model = O.model_for_rows(cfg, used)
    _, z, _ = O.forward(model, dense, offs2, idx2)
    want_loss = O.bce(z, labels)
    assert abs(loss.item() - want_loss) <= 1e-5 * abs(want_loss), (loss.item(), want_loss)
    # gradients of rows used by few samples: they involve only those samples
    rare = np.nonzero(cnt <= 2)[0]
    pick = np.sort(np.random.default_rng(4).choice(rare, min(64, rare.size), replace=False))
    table_of = np.searchsorted(base, uk[pick], side="right") - 1
    # one-row bags: the key at position k*B + b belongs to sample b
    assert np.all(np.diff(offs) == 1)
    sample_set = set()
    for r in uk[pick]:
        sample_set.update((np.nonzero(keys == r)[0] % cfg.B).tolist())
    S = np.array(sorted(sample_set))
    Bs, dense, offs3, idx3, labels3, rws3, used3 = O.sub_batch(cfg, batch, S)
    m3 = O.model_for_rows(cfg, used3)
    ref = O.train_grads(m3, dense, offs3, idx3, labels3)
    bd = EB.bounds(m3, dense, offs3, idx3, labels3, oracle_grads=ref)
    factor = Bs / cfg.B   # the oracle's mean over |S| samples vs the GPU's mean over B
    got_g = to_np(rg[torch.from_numpy(pick).long().cuda()])
    for q, (r, k) in enumerate(zip(uk[pick], table_of)):
        local_row = np.searchsorted(used3[k], r - base[k])
        ci = int(np.sum([len(u) for u in used3[:k]])) + local_row
        TC.check_grad(got_g[q], ref["table_grad"][ci] * factor, bd["table_grad_S2"][ci] * factor,
                      bd["table_grad_F"][ci] * factor, f"full-size row {r}")
