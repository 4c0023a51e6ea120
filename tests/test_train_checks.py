"""The training-step checks have teeth, shown on the CPU.

A correct fp32 program (the training step in plain fp32 PyTorch, standing in
for the GPU) must pass the element-wise gradient bound of error_bound.py and
the SGD update checks of train_checks.py; the same program against an oracle
with one planted mistake (a weight-gradient column or row 5 % off, one touched
embedding row 5 % off, the learning rate's sign flipped) must fail them, and
so must an update taken with the wrong sign or rate."""
import numpy as np
import pytest

import error_bound as EB
import train_checks as TC
from fp32_budget import train_grads_f32
from oracle import oracle as O
from synth import CONFIGS, gen, shrink

CASES = {"tiny-train": CONFIGS["tiny"].with_(training=True, B=203),
         "train-mix": shrink(CONFIGS["train"], B=97, rows_cap=400).with_(bag="mix", seed=2)}
KEYS = ("bot_dW", "bot_db", "top_dW", "top_db")


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    cfg = CASES[request.param]
    b = gen.make_batches(cfg, (0,))[0]
    m = O.model_from_config(cfg)
    args = (m, b.dense, b.offsets, b.indices, b.labels)
    ref = O.train_grads(*args)
    return cfg, m, ref, EB.bounds(*args, oracle_grads=ref), train_grads_f32(*args)


def test_fp32_program_is_within_the_bound(case):
    cfg, m, ref, bd, f32 = case
    for key in KEYS:
        for l in range(len(ref[key])):
            TC.check_grad(f32[key][l], ref[key][l], bd[key + "_S2"][l], bd[key + "_F"][l], f"{key}[{l}]")
    touched = ref["row_count"] > 0
    TC.check_grad(f32["table_grad"][touched], ref["table_grad"][touched], bd["table_grad_S2"][touched],
                  bd["table_grad_F"][touched], "row grads")


def test_bound_is_far_below_the_full_chain_size(case):
    """The bound is a few per cent of the gradient at most on its typical entry, not a multiple of it."""
    cfg, m, ref, bd, f32 = case
    for key in KEYS:
        for l in range(len(ref[key])):
            o = ref[key][l]
            nz = np.abs(o) > 1e-3 * np.abs(o).max()
            lim = EB.tolerance(o, bd[key + "_S2"][l], bd[key + "_F"][l])
            assert np.median(lim[nz] / np.abs(o[nz])) < 0.05, (key, l)


@pytest.mark.parametrize("what", ["column", "row"])
def test_corrupted_weight_gradient_fails(case, what):
    cfg, m, ref, bd, f32 = case
    for key in ("bot_dW", "top_dW"):
        for l in range(len(ref[key])):
            o = ref[key][l]
            bad = TC.corrupt_column(o) if what == "column" else TC.corrupt_row(o, int(np.argmax(np.abs(o).sum(1))))
            with pytest.raises(AssertionError):
                TC.check_grad(f32[key][l], bad, bd[key + "_S2"][l], bd[key + "_F"][l], f"{key}[{l}]")


def test_corrupted_embedding_row_fails(case):
    cfg, m, ref, bd, f32 = case
    touched = np.nonzero(ref["row_count"])[0]
    for r in (int(np.argmax(ref["row_count"])), int(touched[len(touched) // 2])):
        bad = TC.corrupt_row(ref["table_grad"], r)
        with pytest.raises(AssertionError):
            TC.check_grad(f32["table_grad"][touched], bad[touched], bd["table_grad_S2"][touched],
                          bd["table_grad_F"][touched], "row grads")


def _fp32_update(w, g, lr):
    """w - lr g in fp32 with two roundings (product, then difference)."""
    w32, g32 = np.float32(w), np.float32(g)
    return (w32 - np.float32(lr) * g32).astype(np.float64)


@pytest.mark.parametrize("lr", [0.01, 1000.0])
def test_sgd_checks(case, lr):
    cfg, m, ref, bd, f32 = case
    touched = ref["row_count"] > 0
    T0 = np.float32(m.tables[touched]).astype(np.float64)
    g = f32["table_grad"][touched]
    lr32 = float(np.float32(lr))
    T1 = _fp32_update(T0, g, lr)
    S2, F = bd["table_grad_S2"][touched], bd["table_grad_F"][touched]
    TC.check_update_own(T0, T1, g, lr32, "rows")
    TC.check_update_oracle(T0, T1, ref["table_grad"][touched], S2, F, lr32, "rows")
    W0 = np.float32(m.top_W[0]).astype(np.float64)
    W1 = _fp32_update(W0, f32["top_dW"][0], lr)
    TC.check_update_own(W0, W1, f32["top_dW"][0], lr32, "W")
    TC.check_update_oracle(W0, W1, ref["top_dW"][0], bd["top_dW_S2"][0], bd["top_dW_F"][0], lr32, "W")
    if lr < 1.0:
        return
    # at a learning rate that lifts every update above the parameters' rounding, mistakes fail:
    with pytest.raises(AssertionError):                      # the oracle's update with the sign flipped
        TC.check_update_oracle(T0, T1, -ref["table_grad"][touched], S2, F, lr32, "rows")
    with pytest.raises(AssertionError):
        TC.check_update_oracle(W0, W1, -ref["top_dW"][0], bd["top_dW_S2"][0], bd["top_dW_F"][0], lr32, "W")
    with pytest.raises(AssertionError):                      # an update taken with the wrong sign
        TC.check_update_own(T0, _fp32_update(T0, -g, lr), g, lr32, "rows")
    with pytest.raises(AssertionError):                      # ... or at twice the rate
        TC.check_update_own(W0, _fp32_update(W0, f32["top_dW"][0], 2 * lr), f32["top_dW"][0], lr32, "W")
