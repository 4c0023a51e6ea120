"""Row-wise 8-bit tables (DLRM_U8ROW) on the GPU: the library's quantiser
against the oracle's, byte for byte; the fused gather + interaction and the
whole forward against the fp64 oracle on the dequantised tables (one-hot and
multi-hot bags, empty and out-of-range bags, both supported widths); entry
points without uint8 support refuse it."""
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


@pytest.mark.parametrize("d", [16, 64, 128, 100])
@pytest.mark.parametrize("src_dt", ["f32", "bf16"])
def test_quantiser_matches_oracle_byte_for_byte(d, src_dt):
    rng = np.random.default_rng(d)
    v = (rng.standard_normal((777, d)) * rng.uniform(1e-4, 30, (777, 1))).astype(np.float32)
    v[5] = 0.25                       # constant row: scale 0
    v[6, ::2] = -3.0                  # ties and repeated extremes
    if src_dt == "bf16":
        src = torch.from_numpy(v).to(torch.bfloat16)
        v = src.float().numpy()       # the values the quantiser sees
    else:
        src = torch.from_numpy(v)
    rb = E.dlrm_row_bytes(d, E.U8ROW)
    assert rb == (d + 8 + 15) // 16 * 16
    dst = torch.full((777, rb), 0xAB, dtype=torch.uint8, device="cuda")
    E.dlrm_quantize_rows_u8(src.cuda(), dst)
    torch.cuda.synchronize()
    want = O.u8_records(*O.quantize_rows_u8(v))
    assert np.array_equal(dst.cpu().numpy(), want)


def _cases():
    lu, m = CONFIGS["large-u8"], CONFIGS["medium"]
    return {
        "u8-d128-onehot": shrink(lu, B=301, rows_cap=20000),
        "u8-d128-mix": shrink(lu, B=97, rows_cap=500).with_(bag="mix", seed=3),
        "u8-d64-poisson": shrink(m, B=133, rows_cap=3000).with_(table_dtype="u8row", mlp_dtype="bf16", seed=5),
        "u8-d64-f32mlp": shrink(m, B=70, rows_cap=900).with_(table_dtype="u8row", bag="mix", seed=6),
    }


CASES = _cases()


@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_and_fused_concat(name):
    cfg = CASES[name]
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    bt = {k: torch.from_numpy(v).cuda() for k, v in (("dense", batch.dense), ("offsets", batch.offsets),
                                                      ("indices", batch.indices))}
    y = to_np(g.forward(bt))
    assert E.dlrm_check_error(g.ws)[0] == 0
    model = O.model_from_config(cfg)
    want, _, counts = O.forward(model, batch.dense, batch.offsets, batch.indices)
    assert counts == (0, 0)
    assert_close(y, want, "u8row", f"{name} y_hat")
    # the fused kernel alone, bf16 concat
    x = _dense_with_edge_rows(cfg.B, cfg.d, 1)
    ld = E.dlrm_ld(cfg.concat_width, "bf16")
    out = torch.full((cfg.B, ld), float("nan"), dtype=torch.bfloat16, device="cuda")
    E.dlrm_embbag_interact_fwd(g.T, cfg.B, bt["offsets"], bt["indices"], torch.from_numpy(x).cuda(), out, ld, "bf16",
                               g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    base = gen.row_base(cfg)
    rows = [np.arange(m) for m in cfg.rows]
    pooled, _, _ = O.embbag(model.tables, np.asarray(cfg.rows, np.int64), cfg.d, cfg.B, batch.offsets, batch.indices)
    pooled_s = O.embbag(np.abs(model.tables), np.asarray(cfg.rows, np.int64), cfg.d, cfg.B, batch.offsets,
                        batch.indices)[0]
    want_c = O.interact(x, pooled)
    got = to_np(out)
    assert_close(got[:, :cfg.concat_width], want_c, "u8row", f"{name} concat", scale_concat(x, pooled_s))
    assert np.all(got[:, cfg.concat_width:] == 0)
    del base, rows


def _dense_with_edge_rows(B, d, seed):
    """Normal x_dense plus rows the per-sample 24-bit quantisation of x_dense must handle:
    constant rows (range 0), all-zero rows and rows with one large outlier."""
    x = np.random.default_rng(seed).standard_normal((B, d)).astype(np.float32)
    x[::5] = 0.5
    x[1::7] = 0.0
    x[2::11, 3] = 1.0e4
    x[3::13] = np.abs(x[3::13]) + 100.0
    return x


def _empty_bags(offsets, indices, K, B, pred):
    """The CSR batch with every bag (k, b) for which pred(k, b) holds emptied."""
    lens = np.diff(offsets.astype(np.int64))
    keep = np.ones(len(indices), bool)
    for k in range(K):
        for b in range(B):
            if pred(k, b):
                q = k * B + b
                keep[offsets[q]:offsets[q + 1]] = False
                lens[q] = 0
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), indices[keep].copy()


@pytest.mark.parametrize("name", ["u8-d128-onehot", "u8-d64-onehot"])
def test_integer_route_fp32_concat_is_tight(name):
    """One-row bags take the integer route: exact u8 x u8 Gram, fp32 affine terms, 24-bit x_dense. With an
    fp32 concat (no bf16 rounding of the output) the error has two sources: x_dense quantised to 24 bits of
    its per-sample range (at most ~1.5 range 2^-24 per element) and the fp32 rounding of the affine terms,
    which are as large as sum |e - m| |x - min x|. On ordinary rows both stay below 1e-5 of the magnitude
    scale sum |e_i| |x_j|; a row with one x_dense element 1e4 times the rest, met by an embedding element
    near zero, reaches a few 1e-5, so those rows get 1e-4. The dequantising route (bf16 rows) is at ~2e-3."""
    cfg = CASES["u8-d128-onehot"] if name == "u8-d128-onehot" else shrink(
        CONFIGS["medium"], B=211, rows_cap=3000).with_(table_dtype="u8row", mlp_dtype="bf16", bag="one", seed=8)
    batch = gen.make_batches(cfg, (0,))[0]
    # some bags emptied: tables 0, 5, 10, ... for every third sample
    offs, idx = _empty_bags(batch.offsets, batch.indices, cfg.K, cfg.B, lambda k, b: k % 5 == 0 and b % 3 == 0)
    g = GpuModel(cfg)
    x = _dense_with_edge_rows(cfg.B, cfg.d, 2)
    ld = E.dlrm_ld(cfg.concat_width, "f32")
    out = torch.full((cfg.B, ld), float("nan"), dtype=torch.float32, device="cuda")
    E.dlrm_embbag_interact_fwd(g.T, cfg.B, torch.from_numpy(offs).cuda(), torch.from_numpy(idx).cuda(),
                               torch.from_numpy(x).cuda(), out, ld, "f32", g.ws)
    assert E.dlrm_check_error(g.ws)[0] == 0
    model = O.model_from_config(cfg)
    pooled, _, _ = O.embbag(model.tables, np.asarray(cfg.rows, np.int64), cfg.d, cfg.B, offs, idx)
    pooled_s = O.embbag(np.abs(model.tables), np.asarray(cfg.rows, np.int64), cfg.d, cfg.B, offs, idx)[0]
    want = O.interact(x, pooled)
    scale = scale_concat(x, pooled_s)
    got = to_np(out)[:, :cfg.concat_width]
    rel = np.abs(got - want) / (scale + 1e-300)
    outlier = np.zeros(cfg.B, bool)
    outlier[2::11] = True
    worst = (float(rel[~outlier].max()), float(rel[outlier].max()))
    assert worst[0] <= 1e-5 and worst[1] <= 1e-4, f"{name}: worst of scale, ordinary/outlier rows {worst}"
    assert np.all(to_np(out)[:, cfg.concat_width:] == 0)


def test_invalid_bags_and_unsupported_entry_points():
    cfg = shrink(CONFIGS["large-u8"], B=64, rows_cap=300).with_(bag="mix", seed=9)
    batch = gen.make_batches(cfg, (0,))[0]
    g = GpuModel(cfg)
    idx = batch.indices.copy()
    idx[::7] = 10 ** 6                # out of range for every table
    offs = batch.offsets.copy()
    x = torch.zeros((cfg.B, cfg.d), device="cuda")
    ld = E.dlrm_ld(cfg.concat_width, "bf16")
    out = torch.empty((cfg.B, ld), dtype=torch.bfloat16, device="cuda")
    E.dlrm_embbag_interact_fwd(g.T, cfg.B, torch.from_numpy(offs).cuda(), torch.from_numpy(idx).cuda(), x, out, ld,
                               "bf16", g.ws)
    st = E.dlrm_check_error(g.ws)
    assert st[0] == E.ERR_INDEX_OOB
    model = O.model_from_config(cfg)
    pooled, _, counts = O.embbag(model.tables, np.asarray(cfg.rows, np.int64), cfg.d, cfg.B, offs, idx)
    assert counts[0] > 0
    want = O.interact(np.zeros((cfg.B, cfg.d), np.float32), pooled)
    pooled_s = O.embbag(np.abs(model.tables), np.asarray(cfg.rows, np.int64), cfg.d, cfg.B, offs, idx)[0]
    assert_close(to_np(out)[:, :cfg.concat_width], want, "u8row", "u8 concat with skipped indices",
                 scale_concat(np.zeros((cfg.B, cfg.d), np.float32), pooled_s))
    # the pooled-output entry point has no uint8 path
    pooled_t = torch.empty((cfg.B, cfg.K, cfg.d), device="cuda")
    with pytest.raises(E.DlrmError) as e:
        E.dlrm_embbag_fwd(g.T, cfg.B, torch.from_numpy(batch.offsets).cuda(), torch.from_numpy(batch.indices).cuda(),
                          pooled_t, None, g.ws)
    assert e.value.status == E.ERR_UNSUPPORTED


@pytest.mark.slow
def test_large_u8_forward_full_size():
    from test_gpu_fullsize import _sampled_forward
    _sampled_forward(CONFIGS["large-u8"], 512, 7)
