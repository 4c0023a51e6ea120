"""dlrm_forward_noalloc: the forward pass for callers that cannot allocate
device memory (a plugin inside a runtime that owns all device memory, a
request path where cudaMalloc and its implicit synchronisation are not
allowed, a C caller with no device allocator). It uses a fixed scratch array
compiled into the library instead of a caller workspace.

Checked through the C ABI against dlrm_forward on two calls in a row (the
array keeps the previous call's contents, so the second call shows that
nothing stale leaks through), with the same tolerance as the other forward
tests. This file sorts last so that a run stopping at the first failure has
run every other test already; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, assert_close, batch_dev, to_np
from synth import CONFIGS, gen, shrink

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [shrink(CONFIGS["medium"], B=300, rows_cap=4000).with_(bag="mix"),
                                 shrink(CONFIGS["large"], B=1000, rows_cap=30000)],
                         ids=["medium-mix", "large"])
def test_noalloc_forward_matches_forward_on_two_calls(cfg):
    g = GpuModel(cfg)
    assert E.dlrm_workspace_size(g.T, g.bot, g.top, cfg.B, 0) <= E.NOALLOC_SCRATCH_BYTES
    b0, b1 = gen.make_batches(cfg, (0, 1))
    flags = torch.full((1,), 77, dtype=torch.int32, device="cuda")
    for batch in (b0, b1):
        bt = batch_dev(batch)
        want = g.forward(bt)
        assert E.dlrm_check_error(g.ws)[0] == E.OK
        got = torch.full((cfg.B,), float("nan"), device="cuda")
        E.dlrm_forward_noalloc(g.T, g.bot, g.top, cfg.B, bt["dense"], bt["offsets"], bt["indices"], got, flags)
        torch.cuda.synchronize()
        assert int(flags.item()) == 0
        assert_close(to_np(got), to_np(want), cfg.table_dtype, f"noalloc vs forward ({cfg.name})")


def test_noalloc_reports_errors_and_rejects_oversize():
    cfg = shrink(CONFIGS["tiny"], B=64)
    g = GpuModel(cfg)
    batch = gen.make_batches(cfg, (0,))[0]
    bt = batch_dev(batch)
    idx = bt["indices"].clone()
    idx[3] = 10 ** 6                       # out of range: skipped and flagged
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.empty(cfg.B, device="cuda")
    E.dlrm_forward_noalloc(g.T, g.bot, g.top, cfg.B, bt["dense"], bt["offsets"], idx, y, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & 1
    # the next call starts from a cleared record
    E.dlrm_forward_noalloc(g.T, g.bot, g.top, cfg.B, bt["dense"], bt["offsets"], bt["indices"], y, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    # a batch whose scratch need exceeds the array is refused before any launch
    big = 1 << 22
    assert E.dlrm_workspace_size(g.T, g.bot, g.top, big, 0) > E.NOALLOC_SCRATCH_BYTES
    n0 = E.dlrm_launch_count()
    with pytest.raises(E.DlrmError) as ei:
        E.dlrm_forward_noalloc(g.T, g.bot, g.top, big, bt["dense"], bt["offsets"], bt["indices"], y, flags)
    assert ei.value.status == E.ERR_WORKSPACE
    assert E.dlrm_launch_count() == n0
    assert np.isfinite(to_np(y)).all()
