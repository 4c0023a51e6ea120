"""dlrm_forward_noalloc: the forward pass for callers that cannot allocate
device memory (a plugin inside a runtime that owns all device memory, a
request path where cudaMalloc and its implicit synchronisation are not
allowed, a C caller with no device allocator). It uses a fixed scratch array
compiled into the library instead of a caller workspace.

Checked through the C ABI against dlrm_forward on two calls in a row (the
array keeps the previous call's contents, so the second call shows that
nothing stale leaks through). Both entry points run the same kernels in the
same order on the same inputs, so the outputs must be bit-identical. A call
that dlrm_forward would refuse is refused with the same status, before
anything is queued, and leaves err_flags alone. This file sorts last so that
a run stopping at the first failure has run every other test already; it also
passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, batch_dev, to_np
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
        assert torch.equal(got, want), f"noalloc vs forward ({cfg.name}): not bit-identical"


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


def test_noalloc_refuses_what_forward_refuses_with_the_same_status():
    """Too many tables (DLRM_ERR_UNSUPPORTED), a bottom MLP that does not end at d and a null y_hat
    (DLRM_ERR_INVALID_ARG): the status equals dlrm_forward's, nothing is launched, err_flags keeps its
    value."""
    import ctypes as C
    cfg = shrink(CONFIGS["tiny"], B=64)
    g = GpuModel(cfg)
    bt = batch_dev(gen.make_batches(cfg, (0,))[0])
    L = E.lib()
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    flags = torch.full((1,), 77, dtype=torch.int32, device="cuda")
    y = torch.empty(cfg.B, device="cuda")
    P = lambda t: t.data_ptr()  # noqa: E731
    many = (C.c_int64 * (E.MAX_TABLES + 1))(*([1000] * (E.MAX_TABLES + 1)))
    T_many = E._abi.dlrm_tables(g.T.data.data_ptr(), many, E.MAX_TABLES + 1, cfg.d, E.F32)
    bad_dims = (C.c_int * (len(g.bot.dims)))(*(g.bot.dims[:-1] + [g.bot.dims[-1] + 4]))
    bot_bad = E._abi.dlrm_mlp(len(g.bot.Ws), bad_dims, g.bot._W, g.bot._b, g.bot.dt)
    cases = [(C.byref(T_many), g.bot.ref(), P(y)), (g.T.ref(), C.byref(bot_bad), P(y)), (g.T.ref(), g.bot.ref(), None)]
    n0 = E.dlrm_launch_count()
    for T, bot, yp in cases:
        args = (T, bot, g.top.ref(), cfg.B, P(bt["dense"]), P(bt["offsets"]), P(bt["indices"]), bt["indices"].numel(), yp)
        want = L.dlrm_forward(*args, P(g.ws), g.ws.numel(), s)
        got = L.dlrm_forward_noalloc(*args, P(flags), s)
        assert want != E.OK and got == want, (got, want)
    assert E.dlrm_launch_count() == n0
    torch.cuda.synchronize()
    assert int(flags.item()) == 77
