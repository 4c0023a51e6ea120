"""GPU forward path against the fp64 oracle, through the C ABI (cuda:0)."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import (GpuModel, assert_close, batch_dev, concat_width, random_pooled, scale_concat,
                     scale_mlp, scale_pooled, to_np)
from oracle import oracle as O
from synth import CONFIGS, gen, shrink
from synth import device as sd

pytestmark = pytest.mark.gpu

# (name, config) cases sized for the oracle; each spans several kernel tiles and ends in a ragged tail.
def _cases():
    t, m, l, s = CONFIGS["tiny"], CONFIGS["medium"], CONFIGS["large"], CONFIGS["stress"]
    return {
        "tiny": t,
        "tiny-ragged-mix": shrink(t, B=203).with_(bag="mix", seed=1),
        "medium-small": shrink(m, B=197, rows_cap=5000),
        # a batch large enough for the fp32 MLP layers to run on the tensor cores (3xTF32 pairs)
        "medium-b4200": shrink(m, B=4200, rows_cap=300).with_(seed=4, bag="fixed:3"),
        "large-small": shrink(l, B=261, rows_cap=20000),
        "large-batch3": shrink(l, B=3, rows_cap=2000),          # serving-size batch: small-batch layer kernel
        "stress-small": shrink(s, B=37, rows_cap=3000).with_(bag="uniform100"),
        "f16-d64-mix": shrink(m, B=77, rows_cap=700).with_(table_dtype="f16", mlp_dtype="f16", bag="mix"),
        "f32-d3-mix": shrink(t, B=45, rows_cap=50).with_(d=3, bag="mix", bottom=(13, 8, 3), top=(3 + 36, 16, 1)),
        "bf16-d5": shrink(t, B=45, rows_cap=50).with_(d=5, table_dtype="bf16", mlp_dtype="bf16",
                                                         bottom=(13, 8, 5), top=(5 + 36, 16, 1)),
        "f32-d256": shrink(t, B=40, rows_cap=300).with_(d=256, bag="mix", bottom=(13, 32, 256), top=(256 + 36, 32, 1)),
        "f32-d512-K3": shrink(t, B=19, rows_cap=300).with_(rows=(300, 17, 5), d=512, bag="poisson20",
                                                           bottom=(13, 32, 512), top=(512 + 6, 16, 1)),
        "bf16-K1": shrink(l, B=33, rows_cap=100).with_(rows=(100,), bottom=(13, 16, 128), top=(129, 8, 1)),
        # tensor-core fused path: multi-hot and empty bags, every supported width and tile count
        "bf16-d64-K40-mix": shrink(m, B=83).with_(rows=(2000,) * 40, table_dtype="bf16", mlp_dtype="bf16", bag="mix",
                                                   bottom=(13, 32, 64), top=(64 + 820, 32, 1)),
        "bf16-d256-K8-mix": shrink(t, B=51, rows_cap=400).with_(d=256, table_dtype="bf16", mlp_dtype="bf16",
                                                                bag="mix", bottom=(13, 32, 256), top=(256 + 36, 32, 1)),
        "bf16-d32-K62": shrink(t, B=35).with_(rows=(300,) * 62, d=32, table_dtype="bf16", mlp_dtype="bf16",
                                               bottom=(13, 16, 32), top=(32 + 1953, 16, 1)),
        # many tables (K + 2 > 64): row gather U deep and the Gram on mma.sync, m-tile counts 4..8
        "bf16-d64-K63-mix": shrink(s, B=29, rows_cap=500).with_(rows=(500,) * 63, bag="mix", seed=6,
                                                                 top=(64 + 2016, 64, 1)),
        "bf16-d128-K70-u100": shrink(s, B=13, rows_cap=900).with_(rows=(900,) * 70, d=128, seed=7,
                                                                   bottom=(13, 64, 128), top=(128 + 2485, 64, 1)),
        "bf16-d64-K128-mix": shrink(s, B=9, rows_cap=300).with_(rows=(300,) * 128, bag="mix", seed=8,
                                                                 top=(64 + 8256, 32, 1)),
        "bf16-d64-K100-batch1": shrink(s, B=1, rows_cap=1000),
    }


CASES = _cases()


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    E.lib()
    sd.build_fill()


@pytest.mark.parametrize("dt", ["f32", "bf16", "f16"])
def test_device_fill_matches_host_generator(dt):
    cfg = shrink(CONFIGS["tiny"], rows_cap=777).with_(table_dtype=dt, rows=(777, 5, 1000), d=24)
    dev = sd.tables_on_device(cfg, on_device_fill=True).cpu()
    host = sd.host_to_torch(gen.full_tables(cfg), dt)
    assert torch.equal(dev.view(torch.int16 if dt != "f32" else torch.int32),
                       host.view(torch.int16 if dt != "f32" else torch.int32))


def _oracle_pool(cfg, batch):
    model = O.model_from_config(cfg)
    return O.embbag(model.tables, cfg.rows, cfg.d, cfg.B, batch.offsets, batch.indices)


@pytest.mark.parametrize("name", sorted(CASES))
def test_embbag_fwd(name):
    cfg = CASES[name]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    bt = batch_dev(batch)
    pooled = torch.full((cfg.B, cfg.K, cfg.d), float("nan"), device="cuda")
    blen = torch.full((cfg.K * cfg.B,), -7, dtype=torch.int32, device="cuda")
    E.dlrm_embbag_fwd(g.T, cfg.B, bt["offsets"], bt["indices"], pooled, blen, g.ws)
    st = E.dlrm_check_error(g.ws)
    want, wlen, counts = _oracle_pool(cfg, batch)
    assert st == (0, 0, counts[0], counts[1])
    assert np.array_equal(blen.cpu().numpy(), wlen)
    model = O.model_from_config(cfg)
    sc = scale_pooled(model, cfg.B, batch.offsets, batch.indices)
    assert_close(to_np(pooled), want, cfg.table_dtype, f"pooled {name}", sc)


@pytest.mark.parametrize("K,d,dt", [(8, 16, "f32"), (26, 64, "f32"), (26, 128, "bf16"), (100, 64, "bf16"),
                                    (3, 5, "f32"), (1, 1, "f32"), (26, 128, "f16"), (40, 256, "f32")])
def test_interact_fwd(K, d, dt):
    B = 131
    x, p = random_pooled(B, K, d, seed=K * 1000 + d, scale=0.5)
    ld = E.dlrm_ld(concat_width(K, d), dt) + 8
    out = torch.full((B, ld), float("nan"), dtype=sd.TORCH_DT[dt], device="cuda")
    E.dlrm_interact_fwd(B, K, d, torch.from_numpy(x).cuda(), torch.from_numpy(p).cuda(), out, ld)
    torch.cuda.synchronize()
    want = O.interact(x, p)
    got = to_np(out)
    assert_close(got[:, :want.shape[1]], want, dt, f"interaction K={K} d={d} {dt}", scale_concat(x, np.abs(p)))
    assert np.all(got[:, want.shape[1]:] == 0.0), "padding columns must be zero"


@pytest.mark.parametrize("name", sorted(CASES))
def test_embbag_interact_fwd(name):
    cfg = CASES[name]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    bt = batch_dev(batch)
    x = np.random.default_rng(5).standard_normal((cfg.B, cfg.d)).astype(np.float32)
    ld = cfg.concat_ld
    out_t = sd.TORCH_DT[cfg.mlp_dtype]
    out = torch.full((cfg.B, ld), float("nan"), dtype=out_t, device="cuda")
    E.dlrm_embbag_interact_fwd(g.T, cfg.B, bt["offsets"], bt["indices"], torch.from_numpy(x).cuda(), out, ld,
                               cfg.mlp_dtype, g.ws)
    st = E.dlrm_check_error(g.ws)
    pooled, _, counts = _oracle_pool(cfg, batch)
    assert st == (0, 0, counts[0], counts[1])
    want = O.interact(x, pooled)
    got = to_np(out)
    tol_dt = "f32" if (cfg.table_dtype == "f32" and cfg.mlp_dtype == "f32") else "bf16"
    model = O.model_from_config(cfg)
    sc = scale_concat(x, scale_pooled(model, cfg.B, batch.offsets, batch.indices))
    assert_close(got[:, :want.shape[1]], want, tol_dt, f"fused concat {name}", sc)
    assert np.all(got[:, want.shape[1]:] == 0.0)


@pytest.mark.parametrize("name", ["tiny", "medium-small", "medium-b4200", "large-small", "stress-small", "f16-d64-mix"])
def test_mlp_fwd(name):
    cfg = CASES[name]
    g = GpuModel(cfg)
    rng = np.random.default_rng(1)
    for which, mlp in (("bottom", g.bot), ("top", g.top)):
        n_in = mlp.dims[0]
        x = rng.standard_normal((cfg.B, n_in)).astype(np.float32)
        in_dt = "f32" if which == "bottom" else cfg.mlp_dtype
        ld_in = E.dlrm_ld(n_in, in_dt)
        xin = torch.zeros((cfg.B, ld_in), dtype=sd.TORCH_DT[in_dt])
        xin[:, :n_in] = torch.from_numpy(x)
        x_used = to_np(xin)[:, :n_in]          # the values the GPU sees after storage rounding
        n_out = mlp.dims[-1]
        out = torch.full((cfg.B, n_out), float("nan"), device="cuda")
        act = E.ACT_RELU if which == "bottom" else E.ACT_SIGMOID
        E.dlrm_mlp_fwd(mlp, cfg.B, xin.cuda(), ld_in, out, n_out, act, g.ws)
        layers = gen.mlp_layers(cfg, which)
        Ws, bs = O.layers_f64(layers, cfg.mlp_dtype)
        want = O.mlp(Ws, bs, x_used, relu_last=(which == "bottom"))
        if which == "top":
            want = 1.0 / (1.0 + np.exp(-want))
        sc = scale_mlp(Ws, bs, x_used, sigmoid=(which == "top"))
        assert_close(to_np(out), want, cfg.mlp_dtype, f"{which} MLP {name}", sc)


@pytest.mark.parametrize("name", sorted(CASES))
def test_forward(name):
    cfg = CASES[name]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    y = g.forward(batch_dev(batch))
    st = E.dlrm_check_error(g.ws)
    model = O.model_from_config(cfg)
    want, _, counts = O.forward(model, batch.dense, batch.offsets, batch.indices)
    assert st == (0, 0, counts[0], counts[1])
    got = to_np(y)
    assert np.all((got >= 0) & (got <= 1))
    assert_close(got, want, cfg.table_dtype, f"y_hat {name}")


def test_two_batches_back_to_back_are_independent():
    cfg = CASES["tiny-ragged-mix"]
    b0, b1 = gen.make_batches(cfg, (0, 1))
    g = GpuModel(cfg)
    y0 = to_np(g.forward(batch_dev(b0)))
    y1 = to_np(g.forward(batch_dev(b1)))
    y0b = to_np(g.forward(batch_dev(b0)))
    assert np.array_equal(y0, y0b), "same inputs must give bit-identical outputs"
    model = O.model_from_config(cfg)
    assert_close(y1, O.forward(model, b1.dense, b1.offsets, b1.indices)[0], "f32", "second batch")


@pytest.mark.parametrize("name", ["large-small", "bf16-K1", "bf16-d32-K62"])
def test_fused_bf16_one_hot_keeps_fp32_precision(name):
    """One-row bags of bf16 tables are exact in bf16 and x_dense is split into
    two bf16 halves, so the tensor-core Gram with an fp32 output is accurate to
    about 2^-16 of the terms' magnitude (checked at 1e-4)."""
    cfg = CASES[name]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    bt = batch_dev(batch)
    x = np.random.default_rng(9).standard_normal((cfg.B, cfg.d)).astype(np.float32)
    ld = E.dlrm_ld(cfg.concat_width, "f32")
    out = torch.full((cfg.B, ld), float("nan"), device="cuda")
    E.dlrm_embbag_interact_fwd(g.T, cfg.B, bt["offsets"], bt["indices"], torch.from_numpy(x).cuda(), out, ld, "f32",
                               g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    model = O.model_from_config(cfg)
    pooled, _, _ = O.embbag(model.tables, cfg.rows, cfg.d, cfg.B, batch.offsets, batch.indices)
    want = O.interact(x, pooled)
    got = to_np(out)
    sc = scale_concat(x, scale_pooled(model, cfg.B, batch.offsets, batch.indices))
    err = np.abs(got[:, :want.shape[1]] - want)
    assert np.all(err <= 1e-4 * (np.abs(want) + sc)), float((err / (np.abs(want) + sc)).max())
    assert np.all(got[:, want.shape[1]:] == 0)
