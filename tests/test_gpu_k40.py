"""Fused gather + interaction with K = 40 tables (three 16-row tiles): bf16 tables and row-wise 8-bit
tables (integer route for one-row bags, dequantising route for mixed bags) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, assert_close, scale_concat, to_np
from oracle import oracle as O
from synth import CONFIGS, gen, shrink
from synth import device as sd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    E.lib()
    sd.build_fill()


def _cfg(dt, bag):
    K, d = 40, 64
    P = K * (K + 1) // 2
    return shrink(CONFIGS["medium"], B=150, rows_cap=800).with_(
        rows=(800,) * K, d=d, table_dtype=dt, mlp_dtype="bf16", bag=bag, bottom=(13, 64, d), top=(d + P, 64, 1),
        seed=12, name=f"k40-{dt}-{bag}")


@pytest.mark.parametrize("dt,bag", [("bf16", "one"), ("bf16", "mix"), ("u8row", "one"), ("u8row", "mix")])
def test_forty_tables(dt, bag):
    cfg = _cfg(dt, bag)
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    x = np.random.default_rng(3).standard_normal((cfg.B, cfg.d)).astype(np.float32)
    ld = E.dlrm_ld(cfg.concat_width, "bf16")
    out = torch.full((cfg.B, ld), float("nan"), dtype=torch.bfloat16, device="cuda")
    E.dlrm_embbag_interact_fwd(g.T, cfg.B, torch.from_numpy(batch.offsets).cuda(),
                               torch.from_numpy(batch.indices).cuda(), torch.from_numpy(x).cuda(), out, ld, "bf16", g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    model = O.model_from_config(cfg)
    rows = np.asarray(cfg.rows, np.int64)
    pooled = O.embbag(model.tables, rows, cfg.d, cfg.B, batch.offsets, batch.indices)[0]
    pooled_s = O.embbag(np.abs(model.tables), rows, cfg.d, cfg.B, batch.offsets, batch.indices)[0]
    got = to_np(out)
    assert_close(got[:, :cfg.concat_width], O.interact(x, pooled), "bf16" if dt == "bf16" else "u8row",
                 f"{cfg.name} concat", scale_concat(x, pooled_s))
    assert np.all(got[:, cfg.concat_width:] == 0)
