"""Table-wise model parallelism over 2 and 3 gloo ranks on the CPU: the shard plan, the input cut, and both
exchanges (pooled vectors forward, their gradients back to the owners) plus the all-reduce of the MLP
gradients, with the arithmetic done by the fp64 oracle (each rank pools only its own tables).

The sharded forward must give bit for bit the single-rank oracle's y_hat for every shard (the same fp64
operations on the same values); the owners' row gradients and the all-reduced MLP gradients must equal the
single-rank full-batch oracle's to fp64 rounding (only the order of the batch sums differs)."""
import itertools
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import shard_ref as R
from embedding_bags_dot_b200 import sharded as S
from oracle import oracle as O
from synth import CONFIGS, gen, shrink

CFG = shrink(CONFIGS["tiny"], B=96).with_(rows=(300, 40, 120, 300, 7, 90, 300, 5), bag="mix", seed=3, training=True)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_plan_tiles_the_tables_and_minimises_the_largest_rank():
    rng = np.random.default_rng(0)
    for K, world in itertools.product((1, 3, 7), (1, 2, 3, 5)):
        sizes = rng.integers(1, 100, K)
        p = S.plan_tables(sizes, world)
        assert p.first[0] == 0 and p.K == K and len(p.first) == world
        assert all(p.first[r + 1] == p.first[r] + p.count[r] for r in range(world - 1))
        got = max(sum(sizes[k] for k in p.tables_of(r)) for r in range(world))
        # brute force over every placement of world - 1 cut points
        best = min(max(sum(sizes[a:b]) for a, b in zip((0,) + c, c + (K,)))
                   for c in itertools.combinations_with_replacement(range(K + 1), world - 1))
        assert got == best
        assert [p.owner(k) for k in range(K)] == sorted(p.owner(k) for k in range(K))


def test_shard_bags_cuts_the_table_major_csr():
    b = gen.make_batches(CFG, (0,))[0]
    B = CFG.B
    offs = b.offsets.astype(np.int64)
    for first, count in ((0, 8), (2, 3), (7, 1), (4, 0)):
        o, idx = S.shard_bags(b.offsets, b.indices, B, first, count)
        assert o.dtype == np.int32 and o.size == count * B + 1 and o[0] == 0
        assert np.array_equal(o.astype(np.int64), offs[first * B:(first + count) * B + 1] - offs[first * B])
        assert np.array_equal(idx, b.indices[offs[first * B]:offs[(first + count) * B]])


def _own_model(model, plan, r):
    base = np.concatenate([[0], np.cumsum(model.rows)])
    lo, hi = base[plan.first[r]], base[plan.first[r] + plan.count[r]]
    return model.rows[plan.first[r]:plan.first[r] + plan.count[r]], model.tables[lo:hi], lo, hi


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CFG
        B, K, d = cfg.B, cfg.K, cfg.d
        B_l = B // world
        sl = slice(rank * B_l, (rank + 1) * B_l)
        batch = gen.make_batches(cfg, (0,))[0]
        model = O.model_from_config(cfg)
        plan = S.plan_tables([r * d * 4 for r in cfg.rows], world)
        f, c = plan.first[rank], plan.count[rank]
        offs_own, idx_own = S.shard_bags(batch.offsets, batch.indices, B, f, c)
        rows_own, tab_own, lo, hi = _own_model(model, plan, rank)
        # forward: own tables pooled for the whole batch, exchanged, placed
        if c:
            pooled_own, _, _ = O.embbag(tab_own, rows_own, d, B, offs_own, idx_own)
        else:
            pooled_own = np.zeros((B, 0, d))
        parts = S.exchange_pooled(torch.from_numpy(np.ascontiguousarray(pooled_own)), plan, rank)
        pooled = np.zeros((B_l, K, d))
        for s, p in enumerate(parts):
            pooled[:, plan.first[s]:plan.first[s] + plan.count[s]] = p.numpy()
        x = O.mlp(model.bot_W, model.bot_b, batch.dense[sl], relu_last=True)
        z = O.mlp(model.top_W, model.top_b, O.interact(x, pooled), relu_last=False)[:, 0]
        y_shard = 1.0 / (1.0 + np.exp(-z))
        y_full, _, _ = O.forward(model, batch.dense, batch.offsets, batch.indices)
        fwd_exact = bool(np.array_equal(y_shard, y_full[sl]))
        # training: shard-mean gradients, dE back to the owners, MLP gradients all-reduced
        _, g = R.step_grads(model, batch.dense[sl], pooled, batch.labels[sl])
        dE_parts = [torch.from_numpy(np.ascontiguousarray(g["dE"][:, plan.first[s]:plan.first[s] + plan.count[s]]))
                    for s in range(world)]
        dE_own = S.exchange_grads(dE_parts, plan, rank).numpy() / world
        ref = O.train_grads(model, batch.dense, batch.offsets, batch.indices, batch.labels)
        errs = {}
        if c:
            own = O.Model(np.asarray(rows_own, np.int64), d, tab_own, model.bot_W, model.bot_b, model.top_W,
                          model.top_b)
            rg = R.scatter_rows(dE_own, own, offs_own, idx_own)
            want = ref["table_grad"][lo:hi]
            errs["rows"] = float(np.abs(rg - want).max() / (np.abs(want).max() + 1e-300))
        for key in ("bot_dW", "bot_db", "top_dW", "top_db"):
            for l, t in enumerate(g[key]):
                tt = torch.from_numpy(np.ascontiguousarray(t))
                dist.all_reduce(tt)
                want = ref[key][l]
                errs[f"{key}[{l}]"] = float(np.abs(tt.numpy() / world - want).max() / (np.abs(want).max() + 1e-300))
        # every table row the batch touches is owned by exactly one rank
        out[rank] = (fwd_exact, errs, (lo, hi))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_step_over_gloo_matches_the_single_rank_oracle(world):
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    spans = []
    for r in range(world):
        fwd_exact, errs, span = out[r]
        assert fwd_exact, f"rank {r}: sharded y_hat differs from the oracle"
        for what, e in errs.items():
            assert e <= 1e-12, f"rank {r} {what}: relative error {e:.3g}"
        spans.append(span)
    assert spans[0][0] == 0 and all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] == sum(CFG.rows)
