"""The fp32 error budget used by the GPU training tests can tell fp32-quality
gradients from TF32-quality ones: run on the CPU against the fp64 oracle, a
training step whose MLP products keep only TF32 precision fails it, and one
that takes them as 3xTF32 pair products (the GPU's method) passes."""
import numpy as np
import pytest

from fp32_budget import budget_refs, check_within_budget, train_grads_f32
from oracle import oracle as O
from synth import CONFIGS, gen, shrink

CASES = {"tiny-train": CONFIGS["tiny"].with_(training=True, B=203),
         "train-mix": shrink(CONFIGS["train"], B=97, rows_cap=400).with_(bag="mix", seed=2)}


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    cfg = CASES[request.param]
    b = gen.make_batches(cfg, (0,))[0]
    m = O.model_from_config(cfg)
    ref = O.train_grads(m, b.dense, b.offsets, b.indices, b.labels)
    args = (m, b.dense, b.offsets, b.indices, b.labels)
    return cfg, ref, budget_refs(*args), train_grads_f32(*args, tf32x3=True), train_grads_f32(*args, tf32x1=True)


KEYS = ("bot_dW", "bot_db", "top_dW", "top_db")


def _budget_failures(ref, r32, got):
    fails = 0
    for key in KEYS:
        for l, (g, o) in enumerate(zip(got[key], ref[key])):
            try:
                check_within_budget(g, o, [r[key][l] for r in r32], f"{key}[{l}]")
            except AssertionError:
                fails += 1
    return fails


def test_tf32x3_products_are_within_the_fp32_budget(case):
    cfg, ref, r32, x3, x1 = case
    assert _budget_failures(ref, r32, x3) == 0


def test_tf32_width_products_fail_the_fp32_budget(case):
    cfg, ref, r32, x3, x1 = case
    checked = sum(np.asarray(o).size >= 64 for key in KEYS for o in ref[key])
    assert _budget_failures(ref, r32, x1) >= checked // 2
