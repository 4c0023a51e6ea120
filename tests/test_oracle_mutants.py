"""Planted mistakes in the oracle must be caught by its pins.

Each case copies ``oracle/dlrm_oracle.c``, applies one plausible slip (a
dropped term, a wrong sign or index, a transposed operand, a missing
activation or scale), builds it on the CPU and runs the pin suite against it.
A mutant that passes every pin would mean the pins do not constrain that part
of the oracle. All mutations keep memory accesses in bounds.
"""
import os

import pytest

from oracle import oracle as O
from pins import ALL_PINS

SRC = os.path.join(os.path.dirname(O.__file__), "dlrm_oracle.c")

MUTANTS = {
    "dot_uses_xi_twice": ("s += xi[t] * xj[t];", "s += xi[t] * xi[t];"),
    "interaction_row_off_by_one": ("const double* xj = (j == 0) ? x_dense : e + (int64_t)(j - 1) * d;",
                                   "const double* xj = (j == 0) ? x_dense : e + (int64_t)(j) * d;"),
    "relu_on_logit": ("M->top_W[l], M->top_b[l], a, c, l < M->n_top - 1);", "M->top_W[l], M->top_b[l], a, c, 1);"),
    "no_relu_bottom": ("M->bot_W[l], M->bot_b[l], a, c, 1);", "M->bot_W[l], M->bot_b[l], a, c, 0);"),
    "pool_overwrites": ("for (int t = 0; t < d; ++t) out[t] += row[t];", "for (int t = 0; t < d; ++t) out[t] = row[t];"),
    "bias_dropped": ("double s = bias[o];", "double s = 0.0;"),
    "weight_transposed": ("for (int i = 0; i < n_in; ++i) s += w[i] * x[i];",
                          "for (int i = 0; i < n_in; ++i) s += W[((int64_t)i * n_out + o) % ((int64_t)n_in * n_out)] * x[i]; (void)w;"),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    "grad_missing_mean": ("dY[b] = (sigmoid(z[b]) - labels[b]) / B;", "dY[b] = (sigmoid(z[b]) - labels[b]);"),
    "interaction_grad_one_side": ("g[(int64_t)j * d + t] += dz * xi[t];", "(void)0;"),
    "bce_sign": ("s += sp - y[b] * z[b];", "s += sp + y[b] * z[b];"),
    "relu_grad_at_zero": ("if (!(Y[q] > 0.0)) dY[q] = 0.0;", "if (!(Y[q] >= 0.0)) dY[q] = 0.0;"),
    "table_grad_wrong_row": ("double* tg = table_grad + (base[k] + r) * d;", "double* tg = table_grad + (base[k]) * d;"),
    "bias_grad_dropped": ("db[o] = sb;", "db[o] = 0.0;"),
    "sgd_sign": ("w[q] -= lr * g[q];", "w[q] += lr * g[q];"),
    "dense_grad_direct_part_dropped": ("for (int t = 0; t < d; ++t) g[t] += dc[t];", "(void)0;"),
    "oob_not_counted": ("if (r < 0 || r >= rows[k]) { ++oob; continue; }", "if (r < 0 || r >= rows[k]) { continue; }"),
    "concat_dense_last": ("for (int t = 0; t < d; ++t) o[t] = x_dense[(int64_t)b * d + t];",
                          "for (int t = 0; t < d; ++t) o[(int64_t)K * d + t] = x_dense[(int64_t)b * d + t];"),
    "quant_floor": ("if (s > 0.0f) q = rintf((v[c] - lo) / s);", "if (s > 0.0f) q = floorf((v[c] - lo) / s);"),
    "quant_scale_256": ("const float s = (hi - lo) / 255.0f;", "const float s = (hi - lo) / 256.0f;"),
    "quant_offset_hi": ("        offset[r] = lo;", "        offset[r] = hi;"),
    "dequant_no_offset": ("(double)codes[r * d + c] + (double)offset[r];", "(double)codes[r * d + c];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} must be unique"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = O.load(O.build(str(path), str(tmp_path / "libmutant.so"), extra=("-DMUTANT",)))
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            return
    pytest.fail(f"no pin caught mutant {name}")
