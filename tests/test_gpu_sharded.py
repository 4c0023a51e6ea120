"""Table-wise model parallelism on one GPU: the library's side of every rank (its own tables pooled for the
whole batch, dlrm_pooled_assemble, the shard's forward; dlrm_backward_pooled, dlrm_pooled_split,
dlrm_embbag_sgd on the owner, dlrm_mlp_sgd) for 2 and 3 ranks run one after another in one process, with
the all-to-all and the all-reduce done by the test as plain tensor moves (the collectives themselves are
tested over gloo on the CPU). Results against the fp64 oracle of the whole, unsharded batch. A rank that
owns no table takes part too. ShardedDLRM also runs once with a real one-rank NCCL group."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import embedding_bags_dot_b200 as E
import error_bound as EB
import train_checks as TC
from embedding_bags_dot_b200 import sharded as S
from gpucase import GpuModel, assert_close, to_np
from oracle import oracle as O
from synth import CONFIGS, gen, shrink
from synth import device as sd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    E.lib()
    sd.build_fill()


def _rank_tables(g, cfg, plan, r):
    if plan.count[r] == 0:
        return None
    base = np.concatenate([[0], np.cumsum(cfg.rows)])
    lo, hi = int(base[plan.first[r]]), int(base[plan.first[r] + plan.count[r]])
    return E.Tables(g.tables[lo:hi], cfg.rows[plan.first[r]:plan.first[r] + plan.count[r]], cfg.d)


def _own_bags(batch, cfg, plan, r):
    o, i = S.shard_bags(batch.offsets, batch.indices, cfg.B, plan.first[r], plan.count[r])
    return torch.from_numpy(o).cuda(), torch.from_numpy(np.ascontiguousarray(i)).cuda()


def _pool_all(g, cfg, batch, plan, ws):
    """Every rank pools its own tables for the whole batch; returns pooled_own per rank."""
    out = []
    for r in range(plan.world):
        p = torch.empty((cfg.B, plan.count[r], cfg.d), device="cuda")
        if plan.count[r]:
            offs, idx = _own_bags(batch, cfg, plan, r)
            E.dlrm_embbag_fwd(_rank_tables(g, cfg, plan, r), cfg.B, offs, idx, p, None, ws)
        out.append(p)
    return out


CASES = {
    "large-bf16": shrink(CONFIGS["large"], B=192, rows_cap=3000),
    "medium-f32-mix": shrink(CONFIGS["medium"], B=96, rows_cap=2000).with_(bag="mix", seed=5),
}


@pytest.mark.parametrize("world", [2, 3, 27])
@pytest.mark.parametrize("name", sorted(CASES))
def test_sharded_forward(name, world):
    cfg = CASES[name]
    if cfg.B % world:
        cfg = cfg.with_(B=cfg.B // world * world)
    g = GpuModel(cfg)
    batch = gen.make_batches(cfg, (0,))[0]
    plan = S.plan_tables([r * cfg.d for r in cfg.rows], world)
    assert world < cfg.K + 2 or 0 in plan.count
    own = _pool_all(g, cfg, batch, plan, g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    B_l, K, d = cfg.B // world, cfg.K, cfg.d
    ld = cfg.concat_ld
    want, _, _ = O.forward(O.model_from_config(cfg), batch.dense, batch.offsets, batch.indices)
    dense = torch.from_numpy(batch.dense).cuda()
    for s in range(world):
        parts = [own[r][s * B_l:(s + 1) * B_l] for r in range(world)]          # the all-to-all, emulated
        pooled = torch.full((B_l, K, d), float("nan"), device="cuda")
        E.dlrm_pooled_assemble(B_l, K, d, plan.first, plan.count, parts, pooled)
        x = torch.empty((B_l, d), device="cuda")
        E.dlrm_mlp_fwd(g.bot, B_l, dense[s * B_l:(s + 1) * B_l].contiguous(), cfg.n_dense, x, d, E.ACT_RELU, g.ws)
        concat = torch.zeros((B_l, ld), dtype=sd.TORCH_DT[cfg.mlp_dtype], device="cuda")
        E.dlrm_interact_fwd(B_l, K, d, x, pooled, concat, ld)
        y = torch.empty(B_l, device="cuda")
        E.dlrm_mlp_fwd(g.top, B_l, concat, ld, y, 1, E.ACT_SIGMOID, g.ws)
        assert_close(to_np(y), want[s * B_l:(s + 1) * B_l], cfg.table_dtype, f"{name} shard {s} of {world}")


def test_pooled_assemble_and_split_are_inverse_placements():
    B, K, d = 37, 9, 12
    plan = S.ShardPlan(4, (0, 2, 2, 7), (2, 0, 5, 2))
    full = torch.randn(B, K, d, device="cuda")
    parts = [torch.full((B, c, d), float("nan"), device="cuda") for c in plan.count]
    E.dlrm_pooled_split(B, K, d, plan.first, plan.count, full, parts)
    for r, p in enumerate(parts):
        assert torch.equal(p, full[:, plan.first[r]:plan.first[r] + plan.count[r]])
    back = torch.full((B, K, d), float("nan"), device="cuda")
    E.dlrm_pooled_assemble(B, K, d, plan.first, plan.count, parts, back)
    assert torch.equal(back, full)
    with pytest.raises(E.DlrmError):   # parts that do not tile the tables
        E.dlrm_pooled_assemble(B, K, d, (0, 3), (2, 7), parts[:2], back)


TRAIN = shrink(CONFIGS["train"], B=240, rows_cap=2000).with_(bag="mix", seed=9)


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_training_step(world):
    cfg = TRAIN
    lr = 1000.0                              # every update well above the parameters' rounding
    g = GpuModel(cfg, training=True)
    batch = gen.make_batches(cfg, (0,))[0]
    plan = S.plan_tables([r * cfg.d * 4 for r in cfg.rows], world)
    B_l, K, d = cfg.B // world, cfg.K, cfg.d
    model = O.model_from_config(cfg)
    tables0 = g.tables.clone()
    W0 = [w.clone() for w in g.bot.Ws + g.top.Ws]
    b0 = [b.clone() for b in g.bot.bs + g.top.bs]

    own = _pool_all(g, cfg, batch, plan, g.ws)
    gsize = E.dlrm_grads_pooled_size(K, d, g.bot, g.top, B_l)
    gofs = E.dlrm_grads_pooled_offsets(K, d, g.bot, g.top, B_l)
    tws = E.alloc_workspace(E.dlrm_backward_pooled_workspace_size(K, d, g.bot, g.top, B_l))
    grads = [torch.zeros(gsize, dtype=torch.uint8, device="cuda") for _ in range(world)]
    dE_parts = []
    losses = []
    dense = torch.from_numpy(batch.dense).cuda()
    labels = torch.from_numpy(batch.labels).cuda()
    for s in range(world):
        pooled = torch.empty((B_l, K, d), device="cuda")
        E.dlrm_pooled_assemble(B_l, K, d, plan.first, plan.count, [own[r][s * B_l:(s + 1) * B_l] for r in range(world)],
                               pooled)
        loss = torch.zeros(1, device="cuda")
        E.dlrm_backward_pooled(K, d, g.bot, g.top, B_l, dense[s * B_l:(s + 1) * B_l].contiguous(), pooled,
                               labels[s * B_l:(s + 1) * B_l].contiguous(), grads[s], tws, loss=loss)
        losses.append(float(loss.item()))
        dE = E.grads_view(grads[s], gofs["dE"], (B_l, K, d))
        parts = [torch.empty((B_l, c, d), device="cuda") for c in plan.count]
        E.dlrm_pooled_split(B_l, K, d, plan.first, plan.count, dE, parts)
        dE_parts.append(parts)
    assert E.dlrm_check_error(tws)[0] == 0
    # owners: their tables' gradients for the whole batch (the reverse all-to-all, emulated), then the update
    for r in range(world):
        if not plan.count[r]:
            continue
        dE_own = torch.cat([dE_parts[s][r] for s in range(world)], 0).contiguous()
        offs, idx = _own_bags(batch, cfg, plan, r)
        T = _rank_tables(g, cfg, plan, r)
        scratch = E.alloc_workspace(E.dlrm_embbag_sgd_scratch_size(T, cfg.B, idx.numel()))
        E.dlrm_embbag_sgd(T, cfg.B, offs, idx, dE_own, lr / world, scratch)
    # the all-reduce of the MLP gradients, emulated: sum of the dense parts
    dense_end = gofs["dense_end"]
    for s in range(1, world):
        grads[0][:dense_end].view(torch.float32).add_(grads[s][:dense_end].view(torch.float32))
    E.dlrm_mlp_sgd(K, d, g.bot, g.top, B_l, lr / world, grads[0])
    torch.cuda.synchronize()

    args = (model, batch.dense, batch.offsets, batch.indices, batch.labels)
    ref = O.train_grads(*args)
    bd = EB.bounds(*args, oracle_grads=ref)
    assert abs(np.mean(losses) - ref["loss"]) <= 1e-5 * abs(ref["loss"])
    touched = ref["row_count"] > 0
    after = g.tables.cpu().double().numpy()
    before = tables0.cpu().double().numpy()
    assert np.array_equal(after[~touched], before[~touched]), "untouched rows must be bit-identical"
    TC.check_update_oracle(before[touched], after[touched], ref["table_grad"][touched], bd["table_grad_S2"][touched],
                           bd["table_grad_F"][touched], lr, "sharded rows")
    nb = len(model.bot_W)
    for i, (w0, w1) in enumerate(zip(W0, g.bot.Ws + g.top.Ws)):
        key, l = ("bot", i) if i < nb else ("top", i - nb)
        k = (model.bot_W if key == "bot" else model.top_W)[l].shape[1]
        TC.check_update_oracle(to_np(w0)[:, :k], to_np(w1)[:, :k], ref[key + "_dW"][l], bd[key + "_dW_S2"][l],
                               bd[key + "_dW_F"][l], lr, f"sharded {key} W[{l}]")
    for i, (c0, c1) in enumerate(zip(b0, g.bot.bs + g.top.bs)):
        key, l = ("bot", i) if i < nb else ("top", i - nb)
        TC.check_update_oracle(to_np(c0), to_np(c1), ref[key + "_db"][l], bd[key + "_db_S2"][l], bd[key + "_db_F"][l],
                               lr, f"sharded {key} b[{l}]")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_sharded_dlrm_on_a_one_rank_nccl_group():
    """The composed ShardedDLRM (exchanges through torch.distributed) with world = 1: forward and one
    training step against the oracle."""
    cfg = TRAIN.with_(B=128)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        g = GpuModel(cfg, training=True)
        batch = gen.make_batches(cfg, (0,))[0]
        plan = S.plan_tables([r * cfg.d * 4 for r in cfg.rows], 1)
        m = S.ShardedDLRM(plan, 0, g.T, g.bot, g.top, cfg.d, cfg.B)
        offs, idx = _own_bags(batch, cfg, plan, 0)
        dense = torch.from_numpy(batch.dense).cuda()
        y = torch.empty(cfg.B, device="cuda")
        m.forward(dense, offs, idx, y)
        model = O.model_from_config(cfg)
        want, _, _ = O.forward(model, batch.dense, batch.offsets, batch.indices)
        assert_close(to_np(y), want, "f32", "ShardedDLRM forward")
        before = g.tables.clone()
        loss = m.train_step(dense, offs, idx, torch.from_numpy(batch.labels).cuda(), cfg.lr)
        ref = O.train_grads(model, batch.dense, batch.offsets, batch.indices, batch.labels)
        assert abs(float(loss.item()) - ref["loss"]) <= 1e-5 * abs(ref["loss"])
        touched = ref["row_count"] > 0
        assert torch.equal(g.tables.cpu()[torch.from_numpy(~touched)], before.cpu()[torch.from_numpy(~touched)])
        assert not torch.equal(g.tables.cpu()[torch.from_numpy(touched)], before.cpu()[torch.from_numpy(touched)])
    finally:
        dist.destroy_process_group()
