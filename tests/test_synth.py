"""Seeded input generators (CPU only)."""
import numpy as np
import torch

from synth import CONFIGS, gen, shrink


def test_splitmix64_reference_sequence():
    # First three outputs of SplitMix64 from state 0 (Steele, Lea & Flood 2014 reference generator).
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert [int(v) for v in gen.splitmix64_at(0, np.arange(3))] == want


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0], np.float32)])
    mine = gen.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_table_values_range_and_determinism():
    for m in (1000, 40_000_000):
        v = gen.table_rows_f32(0, 3, m, np.array([0, 1, m - 1]), 128)
        s = gen.table_scale(m)
        assert np.all(np.abs(v) <= s) and v.dtype == np.float32
        assert np.array_equal(v, gen.table_rows_f32(0, 3, m, np.array([0, 1, m - 1]), 128))
        assert abs(float(v.mean())) < 0.2 * s
    full = gen.table_rows(0, 1, 50, np.arange(50), 16, "bf16")
    part = gen.table_rows(0, 1, 50, np.array([7, 49]), 16, "bf16")
    assert np.array_equal(full[[7, 49]], part)


def test_batches_structure():
    for name in ("tiny", "medium"):
        cfg = shrink(CONFIGS[name], B=64, rows_cap=1000)
        b = gen.make_batches(cfg, (0, 1))
        for bt in b:
            offs = bt.offsets.astype(np.int64)
            assert offs[0] == 0 and offs[-1] == bt.indices.size and np.all(np.diff(offs) >= 0)
            lens = np.diff(offs)
            if cfg.bag == "one":
                assert np.all(lens == 1)
            else:
                assert lens.min() >= 1 and lens.max() <= 64
            for k in range(cfg.K):
                idx = bt.indices[offs[k * cfg.B]:offs[(k + 1) * cfg.B]]
                assert idx.min() >= 0 and idx.max() < cfg.rows[k]
        assert not np.array_equal(b[0].indices, b[1].indices)


def test_zipf_ranks_truncated():
    rng = np.random.default_rng(0)
    r = gen.zipf_ranks(rng, 1.05, 1000, 200000)
    assert r.min() >= 1 and r.max() <= 1000
    # P(1)/P(2) = 2^alpha for the truncated law
    ratio = np.sum(r == 1) / np.sum(r == 2)
    assert abs(ratio - 2 ** 1.05) < 0.1


def test_configs_shapes():
    c = CONFIGS["large"]
    assert c.K == 26 and c.P == 351 and c.concat_width == 479 and c.concat_ld == 480
    assert sum(c.rows) == 115_776_360
    assert CONFIGS["stress"].concat_width == 5114 and CONFIGS["tiny"].concat_width == 52
    assert CONFIGS["medium"].concat_width == 415
