"""Every kernel of the library is a programmatic dependent of the kernel before it on the stream: it may be
scheduled while that kernel finishes and must wait (griddepcontrol.wait) before touching global memory.
A kernel that read or wrote too early would show up when calls follow one another with no host
synchronisation and share one workspace: each forward overwrites the bottom-MLP output, the concat and
the hidden activations that the previous forward's kernels read. Back-to-back forwards (alternating
batches, small-batch 64-wide GEMM tiles and the SM-pair path) and back-to-back training steps must give
bit for bit what the same calls give one at a time."""
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, batch_dev
from synth import CONFIGS, gen, shrink

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B", [1, 200, 5000])
def test_back_to_back_forwards_equal_separate_calls(B):
    cfg = shrink(CONFIGS["large"], B=B, rows_cap=20000)
    g = GpuModel(cfg)
    bts = [batch_dev(b) for b in gen.make_batches(cfg, (11, 12))]
    want = []
    for bt in bts:
        want.append(g.forward(bt).clone())
        torch.cuda.synchronize()
        assert E.dlrm_check_error(g.ws)[0] == 0
    assert not torch.equal(want[0], want[1])
    n = 8
    ys = [torch.full((B,), float("nan"), device="cuda") for _ in range(n)]
    for i in range(n):                       # one stream, one workspace, no synchronisation in between
        bt = bts[i & 1]
        E.dlrm_forward(g.T, g.bot, g.top, B, bt["dense"], bt["offsets"], bt["indices"], ys[i], g.ws)
    torch.cuda.synchronize()
    assert E.dlrm_check_error(g.ws)[0] == 0
    for i in range(n):
        assert torch.equal(ys[i], want[i & 1]), f"forward {i} of {n} differs from its separate call"


def test_back_to_back_training_steps_equal_stepwise_calls():
    cfg = shrink(CONFIGS["train"], B=512, rows_cap=3000)
    batches = gen.make_batches(cfg, (21, 22, 23))
    runs = []
    for sync_each in (True, False):
        g = GpuModel(cfg, training=True)
        bts = [{k: torch.from_numpy(v).cuda() for k, v in (("dense", b.dense), ("offsets", b.offsets),
                                                          ("indices", b.indices), ("labels", b.labels))}
               for b in batches]
        nnz = max(b.indices.size for b in batches)
        grads = torch.zeros(E.dlrm_grads_size(g.T, g.bot, g.top, cfg.B, nnz), dtype=torch.uint8, device="cuda")
        losses = torch.zeros(len(bts), device="cuda")
        for i, bt in enumerate(bts):
            E.dlrm_backward(g.T, g.bot, g.top, cfg.B, bt["dense"], bt["offsets"], bt["indices"], bt["labels"],
                            grads, g.ws, loss=losses[i:i + 1])
            E.dlrm_sparse_sgd(g.T, g.bot, g.top, cfg.B, bt["indices"].numel(), cfg.lr, grads)
            if sync_each:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        assert E.dlrm_check_error(g.ws)[0] == 0
        runs.append((g.tables.clone(), [w.clone() for w in g.bot.Ws + g.top.Ws] + [b.clone() for b in g.bot.bs + g.top.bs],
                     losses.clone()))
    (t0, w0, l0), (t1, w1, l1) = runs
    assert torch.equal(l0, l1)
    assert torch.equal(t0, t1)
    assert all(torch.equal(a, b) for a, b in zip(w0, w1))
