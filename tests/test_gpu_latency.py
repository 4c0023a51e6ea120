"""The latency-bounded serving paths (bench.py --latency) compute what the plain forward computes:
dlrm_forward captured once in a CUDA graph and replayed gives bit for bit the eager call's y_hat at
serving-size batches, and four streams each serving their own batches side by side (own workspaces,
launches interleaved) give bit for bit what each batch gives alone, and the oracle's values."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, assert_close, batch_dev, to_np
from oracle import oracle as O
from synth import CONFIGS, gen, shrink
from synth import device as sd

pytestmark = pytest.mark.gpu

CFG = shrink(CONFIGS["large"], B=256, rows_cap=5000)


@pytest.fixture(scope="module")
def model():
    E.lib()
    sd.build_fill()
    return GpuModel(CFG)


@pytest.mark.parametrize("B", [1, 8, 64])
def test_graph_replay_equals_the_eager_forward(model, B):
    g = model
    c = CFG.with_(B=B)
    batch = gen.make_batches(c, (3,))[0]
    bt = batch_dev(batch)
    ws = E.alloc_workspace(E.dlrm_workspace_size(g.T, g.bot, g.top, B, 0))
    y = torch.empty(B, device="cuda")
    E.dlrm_forward(g.T, g.bot, g.top, B, bt["dense"], bt["offsets"], bt["indices"], y, ws)
    assert E.dlrm_check_error(ws)[0] == 0
    want = y.clone()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):    # warm-up on a side stream before capture
        E.dlrm_forward(g.T, g.bot, g.top, B, bt["dense"], bt["offsets"], bt["indices"], y, ws, side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        E.dlrm_forward(g.T, g.bot, g.top, B, bt["dense"], bt["offsets"], bt["indices"], y, ws,
                       torch.cuda.current_stream())
    for _ in range(3):
        y.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, want)
    del graph
    ref, _, _ = O.forward(O.model_from_config(c), batch.dense, batch.offsets, batch.indices)
    assert_close(to_np(want), ref, c.table_dtype, f"forward at batch {B}")


def test_colocated_streams_equal_their_batches_alone(model):
    g = model
    S, Bc = 4, 64
    c = CFG.with_(B=Bc)
    batches = gen.make_batches(c, tuple(10 + j for j in range(S)))
    bts = [batch_dev(b) for b in batches]
    wss = [E.alloc_workspace(E.dlrm_workspace_size(g.T, g.bot, g.top, Bc, 0)) for _ in range(S)]
    alone = []
    for j in range(S):
        y = torch.empty(Bc, device="cuda")
        E.dlrm_forward(g.T, g.bot, g.top, Bc, bts[j]["dense"], bts[j]["offsets"], bts[j]["indices"], y, wss[j])
        torch.cuda.synchronize()
        alone.append(y.clone())
    streams = [torch.cuda.Stream() for _ in range(S)]
    ys = [torch.full((Bc,), float("nan"), device="cuda") for _ in range(S)]
    for _ in range(5):                              # several rounds, launches interleaved across streams
        for j in range(S):
            E.dlrm_forward(g.T, g.bot, g.top, Bc, bts[j]["dense"], bts[j]["offsets"], bts[j]["indices"], ys[j], wss[j],
                           streams[j])
    torch.cuda.synchronize()
    model_f64 = O.model_from_config(c)
    for j in range(S):
        assert E.dlrm_check_error(wss[j], streams[j])[0] == 0
        assert torch.equal(ys[j], alone[j]), f"stream {j}"
        ref, _, _ = O.forward(model_f64, batches[j].dense, batches[j].offsets, batches[j].indices)
        assert_close(to_np(ys[j]), ref, c.table_dtype, f"co-located stream {j}")
