"""Bounded device waits that run out (failure detection without a GPU fault).

dlrm_set_wait_polls(0) makes the first bounded wait of the row-gathering
kernels and the ordinary waits of the single-CTA tensor-core layer and of the
one-kernel three-layer MLP give up at once. Each call below must still return, report DLRM_ERR_TIMEOUT through
dlrm_check_error (the kernel drained its own copies and MMAs, freed its tensor
memory and returned), and, after the default is restored, the same call on
the same stream must give exactly the result of a call that never timed out.
Nothing here faults or hangs the GPU: every wait stays bounded, and the drain
after giving up waits with the full bound for copies that were issued."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, batch_dev
from synth import CONFIGS, gen, shrink
from synth import device as sd

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _restore_polls():
    E.lib()
    sd.build_fill()
    yield
    torch.cuda.synchronize()
    E.dlrm_set_wait_polls(-1)
    torch.cuda.synchronize()


def _timed_out_then_recovers(run, ws, out):
    """run() launches the call; out is its output tensor. Returns nothing; asserts the protocol."""
    torch.cuda.synchronize()
    run()
    assert E.dlrm_check_error(ws)[0] == E.OK
    want = out.clone()
    E.dlrm_set_wait_polls(0)
    torch.cuda.synchronize()
    out.fill_(float("nan")) if out.is_floating_point() else out.zero_()
    run()
    st = E.dlrm_check_error(ws)            # synchronises: the call returned and its kernels finished
    assert st[0] == E.ERR_TIMEOUT and st[1] & 4, st
    E.dlrm_set_wait_polls(-1)
    torch.cuda.synchronize()
    out.fill_(float("nan")) if out.is_floating_point() else out.zero_()
    run()
    assert E.dlrm_check_error(ws)[0] == E.OK
    assert torch.equal(out, want), "the call after a timeout must match a call that never timed out"


def test_tensor_core_layer_wait_runs_out():
    """A bf16 MLP at 256 rows: single-CTA tcgen05 layers (TMA ring, TMEM accumulators)."""
    torch.manual_seed(0)
    dims = [64, 256, 128]
    Ws = [(torch.randn(dims[l + 1], dims[l], device="cuda") * 0.1).to(torch.bfloat16) for l in range(2)]
    bs = [torch.randn(dims[l + 1], device="cuda") * 0.1 for l in range(2)]
    mlp = E.MLP(Ws, bs, dims)
    B = 256
    x = torch.randn(B, dims[0], device="cuda").to(torch.bfloat16)
    out = torch.empty(B, dims[-1], device="cuda")
    ws = E.alloc_workspace(E.dlrm_mlp_workspace_size(mlp, B, torch.bfloat16))
    _timed_out_then_recovers(lambda: E.dlrm_mlp_fwd(mlp, B, x, dims[0], out, dims[-1], E.ACT_RELU, ws), ws, out)


@pytest.mark.parametrize("B", [100, 1000])    # one CTA per 128-row tile; SM pairs from 256 rows on
def test_one_kernel_mlp_wait_runs_out(B):
    """Three bf16 layers in one kernel (weight ring, layer-1 chunks and h2 staged on chip, three accumulators)."""
    torch.manual_seed(1)
    dims = [13, 512, 256, 128]
    Ws = [torch.zeros(dims[l + 1], E.dlrm_ld(dims[l], "bf16"), device="cuda", dtype=torch.bfloat16) for l in range(3)]
    for l in range(3):
        Ws[l][:, :dims[l]] = (torch.randn(dims[l + 1], dims[l], device="cuda") * 0.1).bfloat16()
    bs = [torch.randn(dims[l + 1], device="cuda") * 0.1 for l in range(3)]
    mlp = E.MLP(Ws, bs, dims)
    x = torch.randn(B, dims[0], device="cuda")
    out = torch.empty(B, dims[-1], device="cuda")
    ws = E.alloc_workspace(E.dlrm_mlp_workspace_size(mlp, B, torch.float32))
    _timed_out_then_recovers(lambda: E.dlrm_mlp_fwd(mlp, B, x, dims[0], out, dims[-1], E.ACT_RELU, ws), ws, out)


def test_fused_gather_interaction_wait_runs_out():
    """The bulk-copy gather + tensor-core interaction on bf16 tables (one-hot and multi-row bags)."""
    cfg = shrink(CONFIGS["large"], B=96, rows_cap=2000).with_(bag="mix", seed=4)
    g = GpuModel(cfg)
    bt = batch_dev(gen.make_batches(cfg, (0,))[0])
    x = torch.randn(cfg.B, cfg.d, device="cuda")
    ld = cfg.concat_ld
    out = torch.empty(cfg.B, ld, dtype=torch.bfloat16, device="cuda")
    _timed_out_then_recovers(lambda: E.dlrm_embbag_interact_fwd(g.T, cfg.B, bt["offsets"], bt["indices"], x, out, ld,
                                                                ws=g.ws), g.ws, out)


def test_concat_only_bulk_wait_runs_out():
    cfg = shrink(CONFIGS["large-cat"], B=64, rows_cap=2000)
    g = GpuModel(cfg)
    bt = batch_dev(gen.make_batches(cfg, (0,))[0])
    x = torch.randn(cfg.B, cfg.d, device="cuda")
    ld = cfg.concat_ld
    out = torch.empty(cfg.B, ld, dtype=torch.bfloat16, device="cuda")
    _timed_out_then_recovers(lambda: E.dlrm_embbag_cat_fwd(g.T, cfg.B, bt["offsets"], bt["indices"], x, out, ld,
                                                           ws=g.ws), g.ws, out)


def test_whole_forward_wait_runs_out():
    """dlrm_forward at 512 samples: bottom layers, fused gather, top layers all on the single-CTA path."""
    cfg = shrink(CONFIGS["large"], B=512, rows_cap=4096)
    g = GpuModel(cfg)
    bt = batch_dev(gen.make_batches(cfg, (0,))[0])
    y = torch.empty(cfg.B, device="cuda")
    _timed_out_then_recovers(lambda: E.dlrm_forward(g.T, g.bot, g.top, cfg.B, bt["dense"], bt["offsets"],
                                                    bt["indices"], y, g.ws), g.ws, y)
    assert np.isfinite(y.cpu().numpy()).all()
