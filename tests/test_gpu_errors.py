"""Error paths of the C ABI on the GPU: invalid indices and offsets are
skipped and recorded by the kernels' own bounds checks (never trapped), and
host-detectable argument errors return a status before any launch."""
import ctypes as C

import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, assert_close, scale_concat, scale_pooled, to_np
from oracle import oracle as O
from synth import CONFIGS, gen, shrink
from synth import device as sd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["f32", "bf16", "bf16-many"])
def tiny(request):
    # bf16 with d = 16 x 8 = 128 takes the tensor-core fused path; f32 the CUDA-core one; 70 bf16 tables of
    # d = 64 the many-table fused path
    if request.param == "f32":
        cfg = shrink(CONFIGS["tiny"], B=70).with_(bag="mix", seed=4)
    elif request.param == "bf16-many":
        cfg = shrink(CONFIGS["stress"], B=70, rows_cap=1000).with_(rows=(1000,) * 70, bag="mix", seed=4,
                                                                   top=(64 + 2485, 64, 1))
    else:
        cfg = shrink(CONFIGS["large"], B=70, rows_cap=1000).with_(rows=(1000,) * 8, bag="mix", seed=4,
                                                                  top=(128 + 36, 64, 1))
    return cfg, gen.make_batches(cfg, (0,))[0], GpuModel(cfg)


def _run_pool(cfg, g, offsets, indices):
    pooled = torch.full((cfg.B, cfg.K, cfg.d), float("nan"), device="cuda")
    blen = torch.zeros(cfg.K * cfg.B, dtype=torch.int32, device="cuda")
    E.dlrm_embbag_fwd(g.T, cfg.B, torch.from_numpy(offsets).cuda(), torch.from_numpy(indices).cuda(), pooled, blen,
                      g.ws)
    return pooled, blen, E.dlrm_check_error(g.ws)


def test_out_of_range_indices_are_skipped_and_counted(tiny):
    cfg, batch, g = tiny
    idx = batch.indices.copy()
    rng = np.random.default_rng(0)
    pos = rng.choice(idx.size, 25, replace=False)
    idx[pos[:10]] = -1
    idx[pos[10:20]] = cfg.rows[0]     # == m_k: one past the end
    idx[pos[20:]] = 2 ** 31 - 1
    pooled, blen, st = _run_pool(cfg, g, batch.offsets, idx)
    model = O.model_from_config(cfg)
    want, wlen, counts = O.embbag(model.tables, cfg.rows, cfg.d, cfg.B, batch.offsets, idx)
    assert counts == (25, 0)
    assert st == (E.ERR_INDEX_OOB, 1, 25, 0)
    assert np.array_equal(blen.cpu().numpy(), wlen)
    assert_close(to_np(pooled), want, cfg.table_dtype, "pooled with skipped indices",
                 scale_pooled(model, cfg.B, batch.offsets, idx))
    # the record was cleared by the read
    assert E.dlrm_check_error(g.ws) == (0, 0, 0, 0)


def test_bad_offsets_pool_to_zero_and_are_counted(tiny):
    cfg, batch, g = tiny
    offs = batch.offsets.copy()
    nnz = batch.indices.size
    # bag (0, 5): decreasing end; bag (3, 17): start below zero; last bag: end beyond nnz
    offs[6] = offs[5] - 1
    offs[3 * cfg.B + 17] = -3
    offs[-1] = nnz + 5
    pooled, blen, st = _run_pool(cfg, g, offs, batch.indices)
    model = O.model_from_config(cfg)
    want, wlen, counts = O.embbag(model.tables, cfg.rows, cfg.d, cfg.B, offs, batch.indices)
    assert counts[1] >= 3
    assert st == (E.ERR_BAD_OFFSETS, 2 | (1 if counts[0] else 0), counts[0], counts[1])
    assert np.array_equal(blen.cpu().numpy(), wlen)
    assert_close(to_np(pooled), want, cfg.table_dtype, "pooled with bad bags",
                 scale_pooled(model, cfg.B, offs, batch.indices))


def test_forward_records_errors_and_completes(tiny):
    cfg, batch, g = tiny
    idx = batch.indices.copy()
    idx[::7] = 50000
    bt = sd.batch_on_device(batch)
    bt["indices"] = torch.from_numpy(idx).cuda()
    y = g.forward(bt)
    st = E.dlrm_check_error(g.ws)
    model = O.model_from_config(cfg)
    want, _, counts = O.forward(model, batch.dense, batch.offsets, idx)
    assert st == (E.ERR_INDEX_OOB, 1, counts[0], 0)
    assert_close(to_np(y), want, cfg.table_dtype, "forward with skipped indices")


def test_fused_interaction_with_bad_bags(tiny):
    """The fused gather + interaction skips out-of-range indices and pools bags with bad offsets to zero,
    as the oracle does, and counts both."""
    cfg, batch, g = tiny
    offs = batch.offsets.copy()
    idx = batch.indices.copy()
    idx[::11] = cfg.rows[0] + 3
    offs[7] = offs[6] - 1
    offs[2 * cfg.B + 33] = -1
    bt = sd.batch_on_device(batch)
    x = np.random.default_rng(9).standard_normal((cfg.B, cfg.d)).astype(np.float32)
    out = torch.full((cfg.B, cfg.concat_ld), float("nan"), dtype=sd.TORCH_DT[cfg.mlp_dtype], device="cuda")
    E.dlrm_embbag_interact_fwd(g.T, cfg.B, torch.from_numpy(offs).cuda(), torch.from_numpy(idx).cuda(),
                               torch.from_numpy(x).cuda(), out, cfg.concat_ld, cfg.mlp_dtype, g.ws)
    st = E.dlrm_check_error(g.ws)
    model = O.model_from_config(cfg)
    pooled, _, counts = O.embbag(model.tables, cfg.rows, cfg.d, cfg.B, offs, idx)
    assert counts[0] > 0 and counts[1] >= 2
    assert st == (E.ERR_BAD_OFFSETS, 3, counts[0], counts[1])
    want = O.interact(x, pooled)
    sc = scale_concat(x, scale_pooled(model, cfg.B, offs, idx))
    tol = "f32" if cfg.table_dtype == "f32" else "bf16"
    assert_close(to_np(out)[:, :want.shape[1]], want, tol, "fused concat with bad bags", sc)


def test_host_argument_errors(tiny):
    cfg, batch, g = tiny
    L = E.lib()
    bt = sd.batch_on_device(batch)
    pooled = torch.empty((cfg.B, cfg.K, cfg.d), device="cuda")
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    nnz = batch.indices.size
    P = lambda t: t.data_ptr()  # noqa: E731
    # null tables
    nws = g.ws.numel()
    assert L.dlrm_embbag_fwd(None, cfg.B, P(bt["offsets"]), P(bt["indices"]), nnz, P(pooled), None, P(g.ws), nws, s) == E.ERR_INVALID_ARG
    # nnz out of range
    assert L.dlrm_embbag_fwd(g.T.ref(), cfg.B, P(bt["offsets"]), P(bt["indices"]), 2 ** 31, P(pooled), None, P(g.ws), nws, s) == E.ERR_INVALID_ARG
    # missing or short workspace, misaligned output
    assert L.dlrm_embbag_fwd(g.T.ref(), cfg.B, P(bt["offsets"]), P(bt["indices"]), nnz, P(pooled), None, None, 0, s) == E.ERR_WORKSPACE
    assert L.dlrm_embbag_fwd(g.T.ref(), cfg.B, P(bt["offsets"]), P(bt["indices"]), nnz, P(pooled), None, P(g.ws), 255, s) == E.ERR_WORKSPACE
    assert L.dlrm_embbag_fwd(g.T.ref(), cfg.B, P(bt["offsets"]), P(bt["indices"]), nnz, P(pooled) + 4, None, P(g.ws), nws, s) == E.ERR_INVALID_ARG
    # concat leading dimension too small
    x = torch.zeros((cfg.B, cfg.d), device="cuda")
    out = torch.zeros((cfg.B, 64), device="cuda")
    assert L.dlrm_interact_fwd(cfg.B, cfg.K, cfg.d, P(x), P(pooled), P(out), cfg.concat_width - 1, 0, s) == E.ERR_INVALID_ARG
    # too many tables
    assert L.dlrm_interact_fwd(cfg.B, 257, cfg.d, P(x), P(pooled), P(out), 10 ** 6, 0, s) == E.ERR_UNSUPPORTED
    # a table with zero rows
    bad = E.Tables(g.tables, [0] + list(cfg.rows[1:]), cfg.d)
    assert L.dlrm_embbag_fwd(bad.ref(), cfg.B, P(bt["offsets"]), P(bt["indices"]), nnz, P(pooled), None, P(g.ws), nws, s) == E.ERR_INVALID_ARG
    # unsupported row width: d = 301 fp32 is neither a 16-byte multiple <= 2 KB nor <= 256
    t300 = torch.zeros((10, 301), device="cuda")
    T300 = E.Tables(t300, [10], 301)
    assert L.dlrm_embbag_fwd(T300.ref(), 1, P(bt["offsets"]), P(bt["indices"]), 0, P(pooled), None, P(g.ws), nws, s) == E.ERR_UNSUPPORTED
    # forward with a top MLP whose input width does not match d + K(K+1)/2
    y = torch.empty(cfg.B, device="cuda")
    assert L.dlrm_forward(g.T.ref(), g.bot.ref(), g.bot.ref(), cfg.B, P(bt["dense"]), P(bt["offsets"]), P(bt["indices"]), nnz, P(y), P(g.ws), nws, s) == E.ERR_INVALID_ARG
    # B = 0 is a valid no-op
    assert L.dlrm_forward(g.T.ref(), g.bot.ref(), g.top.ref(), 0, None, None, None, 0, None, P(g.ws), nws, s) == E.OK
    torch.cuda.synchronize()
    assert E.dlrm_check_error(g.ws) == (0, 0, 0, 0)


def test_all_bags_empty(tiny):
    cfg, batch, g = tiny
    offs = np.zeros(cfg.K * cfg.B + 1, np.int32)
    idx = np.zeros(0, np.int32)
    pooled = torch.full((cfg.B, cfg.K, cfg.d), float("nan"), device="cuda")
    E.dlrm_embbag_fwd(g.T, cfg.B, torch.from_numpy(offs).cuda(), torch.zeros(1, dtype=torch.int32, device="cuda")[:0],
                      pooled, None, g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    assert torch.all(pooled == 0)
    y = g.forward({"dense": torch.from_numpy(batch.dense).cuda(), "offsets": torch.from_numpy(offs).cuda(),
                   "indices": torch.zeros(0, dtype=torch.int32, device="cuda")})
    model = O.model_from_config(cfg)
    want, _, _ = O.forward(model, batch.dense, offs, idx)
    assert_close(to_np(y), want, cfg.table_dtype, "forward with empty bags")
