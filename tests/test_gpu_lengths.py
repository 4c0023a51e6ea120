"""Bags given by uint8 lengths: the device prefix sum against numpy's, bit for
bit (chunk boundaries, ragged tails, zero and 255 lengths, an input that does
not start on a 16-byte boundary), and dlrm_forward_lengths against
dlrm_forward on the same bags, bit for bit; lengths that add up to more than
the index count are reported as bad bags."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import GpuModel, to_np
from synth import CONFIGS, gen, shrink
from synth import device as sd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    E.lib()
    sd.build_fill()


@pytest.mark.parametrize("n", [0, 1, 31, 8191, 8192, 8193, 100003, 3000001])
@pytest.mark.parametrize("shift", [0, 1])
def test_offsets_from_lengths_match_numpy(n, shift):
    rng = np.random.default_rng(n + shift)
    lens = rng.integers(0, 256, n + shift, dtype=np.uint8)
    lens[shift::7] = 0
    lens[shift + 3::11] = 255
    dev = torch.from_numpy(lens).cuda()[shift:]          # shift = 1: not on a 16-byte boundary
    out = torch.full((n + 1,), -7, dtype=torch.int32, device="cuda")
    ws = E.alloc_workspace(E.dlrm_offsets_from_lengths_workspace_size(n))
    E.dlrm_offsets_from_lengths(dev, out, ws)
    want = np.concatenate([[0], np.cumsum(lens[shift:].astype(np.int64))]).astype(np.int32)
    assert np.array_equal(out.cpu().numpy(), want)


def _cases():
    lg, lu = CONFIGS["large"], CONFIGS["large-u8"]
    return {
        "large-onehot": shrink(lg, B=1000, rows_cap=30000),
        "large-mix": shrink(lg, B=333, rows_cap=2000).with_(bag="mix", seed=4),
        "u8-onehot": shrink(lu, B=257, rows_cap=5000),
    }


@pytest.mark.parametrize("name", sorted(_cases()))
def test_forward_lengths_equals_forward(name):
    cfg = _cases()[name]
    batch = gen.make_batches(cfg, (0,))[0]
    lens = np.diff(batch.offsets.astype(np.int64))
    assert lens.max() <= 255
    g = GpuModel(cfg)
    dense = torch.from_numpy(batch.dense).cuda()
    offs = torch.from_numpy(batch.offsets).cuda()
    idx = torch.from_numpy(batch.indices).cuda()
    y1 = torch.full((cfg.B,), float("nan"), device="cuda")
    y2 = torch.full((cfg.B,), float("nan"), device="cuda")
    E.dlrm_forward(g.T, g.bot, g.top, cfg.B, dense, offs, idx, y1, g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    E.dlrm_forward_lengths(g.T, g.bot, g.top, cfg.B, dense, torch.from_numpy(lens.astype(np.uint8)).cuda(), idx, y2,
                           g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    assert np.array_equal(to_np(y1), to_np(y2))


def test_lengths_past_the_indices_are_bad_bags():
    cfg = shrink(CONFIGS["large"], B=200, rows_cap=3000)
    batch = gen.make_batches(cfg, (0,))[0]
    lens = np.diff(batch.offsets.astype(np.int64)).astype(np.uint8)
    lens[-5:] = 200                                    # the last bags claim indices that do not exist
    g = GpuModel(cfg)
    y = torch.empty(cfg.B, device="cuda")
    E.dlrm_forward_lengths(g.T, g.bot, g.top, cfg.B, torch.from_numpy(batch.dense).cuda(),
                           torch.from_numpy(lens).cuda(), torch.from_numpy(batch.indices).cuda(), y, g.ws)
    st = E.dlrm_check_error(g.ws)
    assert st[0] == E.ERR_BAD_OFFSETS and st[3] == 5
