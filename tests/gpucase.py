"""Helpers for the GPU parity tests: seeded models on the device and the
element-wise tolerance rule.

Tolerance (the same rule everywhere, applied element by element against the
fp64 oracle):

    |gpu - oracle| <= rtol * (|oracle| + scale) + atol

with rtol = 1e-5, atol = 0 for fp32 tables and rtol = 2e-2, atol = 1e-3 for
bf16 / fp16 tables. ``scale`` is the magnitude of the element's last sum:
the same oracle computation on absolute values (sum of |rows| for a pooled
bag; sum_t |X_it||X_jt| for an interaction term, with pooled rows replaced by
their sums of |rows|; |W_L| |a_(L-1)| + |b_L| for the last layer of an MLP,
with the oracle's own penultimate activations, times 1/4 under a sigmoid,
whose slope is at most 1/4). This is the usual forward-error yardstick for a
floating-point sum: a sum that cancels to nearly zero keeps the absolute error
of its terms, so its error is judged against the terms, not against the small
result. Where no scale is given (the model output y_hat, which lies in (0, 1))
the floor is 1e-3 * max|oracle| over the tensor.
"""
from __future__ import annotations

import numpy as np
import torch

import embedding_bags_dot_b200 as E
from oracle import oracle as O
from synth import device as sd
from synth import gen

# u8row: the fused path dequantises row-wise 8-bit tables into bf16 and follows the bf16 rule
TOL = {"f32": (1e-5, 0.0), "bf16": (2e-2, 1e-3), "f16": (2e-2, 1e-3), "u8row": (2e-2, 1e-3)}


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype != torch.float64 else t.cpu().numpy()


def assert_close(got, want, dtype: str, what: str, scale=None):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, f"{what}: shape {got.shape} vs {want.shape}"
    if want.size == 0:
        return
    rtol, atol = TOL[dtype]
    mx = float(np.abs(want).max())
    floor = 1e-3 * mx if scale is None else np.asarray(scale, np.float64)
    lim = rtol * (np.abs(want) + floor) + atol
    err = np.abs(got - want)
    bad = ~(err <= lim)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - lim, -np.inf)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance ({dtype}); "
                             f"worst at {i}: gpu {got[i]!r} oracle {want[i]!r} (max |oracle| {mx:.3g})")


def max_rel(got, want) -> float:
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    den = np.abs(want) + 1e-3 * (np.abs(want).max() if want.size else 0) + 1e-300
    return float((np.abs(got - want) / den).max()) if want.size else 0.0


# ----------------------------------------------------------------- magnitude scales (oracle on |inputs|)

def abs_model(model: O.Model) -> O.Model:
    a = lambda v: [np.abs(x) for x in v]  # noqa: E731
    return O.Model(model.rows, model.d, np.abs(model.tables), a(model.bot_W), a(model.bot_b), a(model.top_W),
                   a(model.top_b))


def scale_pooled(model: O.Model, B, offsets, indices):
    return O.embbag(np.abs(model.tables), model.rows, model.d, B, offsets, indices)[0]


def scale_concat(x, pooled_scale):
    return O.interact(np.abs(x), pooled_scale)


def scale_mlp(Ws, bs, x, sigmoid=False):
    a = O.mlp(Ws[:-1], bs[:-1], x, relu_last=True) if len(Ws) > 1 else np.asarray(x, np.float64)
    s = np.abs(a) @ np.abs(Ws[-1]).T + np.abs(bs[-1])
    return 0.25 * s if sigmoid else s


class GpuModel:
    """A seeded model on cuda:0 wrapped for the C ABI."""

    def __init__(self, cfg, on_device_fill=None, training=None):
        self.cfg = cfg
        self.tables = sd.tables_on_device(cfg, on_device_fill=on_device_fill,
                                          quantize=lambda src, dst: E.dlrm_quantize_rows_u8(src, dst))
        self.T = E.Tables(self.tables, cfg.rows, cfg.d)
        bW, bb, bd = sd.mlp_on_device(cfg, "bottom")
        tW, tb, td = sd.mlp_on_device(cfg, "top")
        self.bot = E.MLP(bW, bb, bd)
        self.top = E.MLP(tW, tb, td)
        tr = cfg.training if training is None else training
        self.ws = E.alloc_workspace(E.dlrm_workspace_size(self.T, self.bot, self.top, cfg.B, int(tr)))

    def forward(self, bt: dict, B=None):
        B = self.cfg.B if B is None else B
        y = torch.empty(B, dtype=torch.float32, device="cuda")
        E.dlrm_forward(self.T, self.bot, self.top, B, bt["dense"], bt["offsets"], bt["indices"], y, self.ws)
        return y


def random_pooled(B, K, d, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((B, d)) * scale).astype(np.float32)
    p = (rng.standard_normal((B, K, d)) * scale).astype(np.float32)
    return x, p


def concat_width(K, d):
    return d + K * (K + 1) // 2


def batch_dev(batch: gen.Batch):
    return sd.batch_on_device(batch)
