"""Concat-only interaction (dlrm_embbag_cat_fwd, dlrm_forward_cat) against
the fp64 oracle: every table dtype, vector and element paths, one-hot,
multi-hot and empty bags, fp32 and bf16 concat outputs, skipped indices, and
argument errors."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, assert_close, scale_pooled, to_np
from oracle import oracle as O
from synth import CONFIGS, gen, shrink
from synth import device as sd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    E.lib()
    sd.build_fill()


def _cases():
    t, m, lc = CONFIGS["tiny"], CONFIGS["medium"], CONFIGS["large-cat"]
    return {
        "cat-tiny-f32-mix": shrink(t, B=203).with_(bag="mix", seed=2, interaction="cat", top=(16 * 9, 64, 1)),
        "cat-large-small": shrink(lc, B=301, rows_cap=20000),
        "cat-d64-poisson-bf16mlp": shrink(m, B=97, rows_cap=3000).with_(mlp_dtype="bf16", interaction="cat",
                                                                        top=(64 * 27, 256, 1), seed=3),
        "cat-f16-d5": shrink(t, B=45, rows_cap=50).with_(d=5, table_dtype="f16", mlp_dtype="f16", bag="mix",
                                                         interaction="cat", bottom=(13, 8, 5), top=(45, 16, 1)),
        # f16 tables into an f16 concat (the forward's): rows assembled in shared memory, one bulk store each
        "cat-d64-f16-mix": shrink(m, B=77, rows_cap=2000).with_(table_dtype="f16", mlp_dtype="f16", bag="mix",
                                                                interaction="cat", top=(64 * 27, 256, 1), seed=8),
    }


CASES = _cases()


@pytest.mark.parametrize("name", sorted(CASES))
def test_concat_and_forward(name):
    cfg = CASES[name]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    bt = {k: torch.from_numpy(v).cuda() for k, v in (("dense", batch.dense), ("offsets", batch.offsets),
                                                      ("indices", batch.indices))}
    model = O.model_from_config(cfg)
    rows = np.asarray(cfg.rows, np.int64)
    x = np.random.default_rng(1).standard_normal((cfg.B, cfg.d)).astype(np.float32)
    pooled, _, _ = O.embbag(model.tables, rows, cfg.d, cfg.B, batch.offsets, batch.indices)
    pooled_s = O.embbag(np.abs(model.tables), rows, cfg.d, cfg.B, batch.offsets, batch.indices)[0]
    want = O.concat(x, pooled)
    scale = np.concatenate([np.abs(x).astype(np.float64)] + [pooled_s[:, k] for k in range(cfg.K)], axis=1)
    for out_t in (torch.float32, torch.bfloat16):
        ld = E.dlrm_ld(cfg.concat_width, "f32" if out_t == torch.float32 else "bf16") + 8
        out = torch.full((cfg.B, ld), float("nan"), dtype=out_t, device="cuda")
        E.dlrm_embbag_cat_fwd(g.T, cfg.B, bt["offsets"], bt["indices"], torch.from_numpy(x).cuda(), out, ld, ws=g.ws)
        assert E.dlrm_check_error(g.ws)[0] == 0
        got = to_np(out)
        # one-row bags copy stored values; several rows are summed in fp32: the table's own rule
        assert_close(got[:, :cfg.concat_width], want, "f32" if out_t == torch.float32 else "bf16",
                     f"{name} concat ({out_t})", scale)
        assert np.all(got[:, cfg.concat_width:] == 0), "padding columns are zeroed"
    y = torch.empty(cfg.B, device="cuda")
    E.dlrm_forward_cat(g.T, g.bot, g.top, cfg.B, bt["dense"], bt["offsets"], bt["indices"], y, g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    want_y, _, counts = O.forward_cat(model, batch.dense, batch.offsets, batch.indices)
    assert counts == (0, 0)
    rule = "f32" if cfg.mlp_dtype == "f32" and cfg.table_dtype == "f32" else "bf16"
    assert_close(to_np(y), want_y, rule, f"{name} y_hat")


def test_skipped_indices_and_argument_errors():
    cfg = CASES["cat-tiny-f32-mix"]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    idx = batch.indices.copy()
    idx[::5] = -3
    x = torch.zeros((cfg.B, cfg.d), device="cuda")
    ld = cfg.concat_width
    out = torch.empty((cfg.B, ld), device="cuda")
    offs = torch.from_numpy(batch.offsets).cuda()
    E.dlrm_embbag_cat_fwd(g.T, cfg.B, offs, torch.from_numpy(idx).cuda(), x, out, ld, ws=g.ws)
    assert E.dlrm_check_error(g.ws)[0] == E.ERR_INDEX_OOB
    model = O.model_from_config(cfg)
    pooled, _, counts = O.embbag(model.tables, np.asarray(cfg.rows, np.int64), cfg.d, cfg.B, batch.offsets, idx)
    assert counts[0] > 0
    want = O.concat(np.zeros((cfg.B, cfg.d)), pooled)
    assert_close(to_np(out), want, "f32", "concat with skipped indices",
                 np.concatenate([np.zeros((cfg.B, cfg.d))] + [scale_pooled(model, cfg.B, batch.offsets, idx)[:, k]
                                                              for k in range(cfg.K)], axis=1))
    with pytest.raises(E.DlrmError) as e:
        E.dlrm_embbag_cat_fwd(g.T, cfg.B, offs, torch.from_numpy(batch.indices).cuda(), x, out, ld - 1, ws=g.ws)
    assert e.value.status == E.ERR_INVALID_ARG
    # the dot-interaction forward refuses a concat-width top MLP, and the other way round
    y = torch.empty(cfg.B, device="cuda")
    with pytest.raises(E.DlrmError) as e:
        E.dlrm_forward(g.T, g.bot, g.top, cfg.B, torch.from_numpy(batch.dense).cuda(), offs,
                       torch.from_numpy(batch.indices).cuda(), y, g.ws)
    assert e.value.status == E.ERR_INVALID_ARG


@pytest.mark.slow
def test_large_cat_forward_full_size():
    # the full 65,536-sample batch in the benchmark's launch configuration, checked on sampled outputs
    cfg = CONFIGS["large-cat"]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    bt = {k: torch.from_numpy(v).cuda() for k, v in (("dense", batch.dense), ("offsets", batch.offsets),
                                                      ("indices", batch.indices))}
    y = torch.empty(cfg.B, device="cuda")
    E.dlrm_forward_cat(g.T, g.bot, g.top, cfg.B, bt["dense"], bt["offsets"], bt["indices"], y, g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    samples = np.sort(np.random.default_rng(8).choice(cfg.B, 256, replace=False))
    Bs, dense, offs, idx, _, rows, used = O.sub_batch(cfg, batch, samples)
    want, _, counts = O.forward_cat(O.model_for_rows(cfg, used), dense, offs, idx)
    assert counts == (0, 0)
    assert_close(to_np(y)[samples], want, "bf16", "large-cat y_hat (sampled)")
