"""ctypes front end of the fp64 CPU oracle (``dlrm_oracle.c``).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. It shares no code
with the CUDA library: it compiles its own C file with gcc and takes its
inputs from ``synth`` (seeded input generation only).

The pages' definition of each step is cited in ``dlrm_oracle.c``. This file
only marshals arrays: it widens stored table and weight values to fp64
(exact), drops weight padding, and, for batches whose tables are too large
for host RAM, builds a sub-batch over chosen samples whose tables hold just
the rows those samples reference (indices remapped; no arithmetic of the
method involved).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

from synth import gen
from synth.configs import Config

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dlrm_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-ffp-contract=off"]


def build(src: str = _SRC, out: str = _LIB, extra=()) -> str:
    """Compile the oracle with gcc (fp64, no fast-math, no FMA contraction)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src) or extra:
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, *extra, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


class _Model(C.Structure):
    _fields_ = [
        ("K", C.c_int), ("d", C.c_int), ("n_bot", C.c_int), ("n_top", C.c_int),
        ("bot_dims", C.POINTER(C.c_int)), ("top_dims", C.POINTER(C.c_int)),
        ("bot_W", C.POINTER(C.c_void_p)), ("bot_b", C.POINTER(C.c_void_p)),
        ("top_W", C.POINTER(C.c_void_p)), ("top_b", C.POINTER(C.c_void_p)),
        ("rows", C.POINTER(C.c_int64)), ("tables", C.c_void_p),
    ]


def _declare(lib):
    vp, i, l, d = C.c_void_p, C.c_int, C.c_long, C.c_double
    lib.oracle_threads.restype = i
    lib.oracle_set_threads.argtypes = [i]
    lib.oracle_embbag.argtypes = [i, i, i, l, vp, vp, vp, vp, vp, vp, vp]
    lib.oracle_interact.argtypes = [i, i, i, vp, vp, vp]
    lib.oracle_mlp.argtypes = [i, vp, vp, vp, i, vp, vp, i]
    lib.oracle_forward.argtypes = [vp, i, l, vp, vp, vp, vp, vp, vp]
    lib.oracle_bce.argtypes = [i, vp, vp]
    lib.oracle_bce.restype = d
    lib.oracle_train_grads.argtypes = [vp, i, l, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.oracle_sgd.argtypes = [C.c_int64, d, vp, vp]
    lib.oracle_quantize_rows_u8.argtypes = [C.c_int64, i, vp, vp, vp, vp]
    lib.oracle_concat.argtypes = [i, i, i, vp, vp, vp]
    lib.oracle_dequantize_rows_u8.argtypes = [C.c_int64, i, vp, vp, vp, vp]
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library. A path loads a specific build (mutation tests)."""
    global _lib
    if path is not None:
        return _declare(C.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(C.CDLL(build()))
    return _lib


def _p(a: np.ndarray):
    return C.c_void_p(a.ctypes.data) if a.size else C.c_void_p(0)


def _c64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def threads(lib=None) -> int:
    return (lib or load()).oracle_threads()


# ----------------------------------------------------------------- primitive calls

def embbag(tables: np.ndarray, rows, d: int, B: int, offsets, indices, lib=None):
    """Sum-pooled bags. tables: fp64 [sum rows][d]. Returns (pooled [B][K][d], bag_len [K*B], (n_oob, n_bad))."""
    lib = lib or load()
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    K = rows.size
    tables, offsets, indices = _c64(tables), _i32(offsets), _i32(indices)
    pooled = np.zeros((B, K, d), np.float64)
    blen = np.zeros(K * B, np.int32)
    counts = np.zeros(2, np.int64)
    lib.oracle_embbag(K, B, d, indices.size, _p(rows), _p(tables), _p(offsets), _p(indices),
                      _p(pooled), _p(blen), _p(counts))
    return pooled, blen, (int(counts[0]), int(counts[1]))


def interact(x_dense: np.ndarray, pooled: np.ndarray, lib=None) -> np.ndarray:
    """[B][d] and [B][K][d] -> concat [B][d + K(K+1)/2]."""
    lib = lib or load()
    x_dense, pooled = _c64(x_dense), _c64(pooled)
    B, K, d = pooled.shape
    out = np.zeros((B, d + K * (K + 1) // 2), np.float64)
    lib.oracle_interact(B, K, d, _p(x_dense), _p(pooled), _p(out))
    return out


def mlp(Ws, bs, x: np.ndarray, relu_last: bool, lib=None) -> np.ndarray:
    """Ws[l]: fp64 [out][in]; relu after every hidden layer, and after the last iff relu_last."""
    lib = lib or load()
    Ws = [_c64(w) for w in Ws]
    bs = [_c64(b) for b in bs]
    x = _c64(x)
    dims = np.array([Ws[0].shape[1]] + [w.shape[0] for w in Ws], np.int32)
    Wp = (C.c_void_p * len(Ws))(*[w.ctypes.data for w in Ws])
    bp = (C.c_void_p * len(bs))(*[b.ctypes.data for b in bs])
    out = np.zeros((x.shape[0], dims[-1]), np.float64)
    lib.oracle_mlp(len(Ws), _p(dims), Wp, bp, x.shape[0], _p(x), _p(out), int(relu_last))
    return out


# ----------------------------------------------------------------- model assembly

@dataclass
class Model:
    """fp64 copy of a model's parameters, kept alive alongside the ctypes view."""
    rows: np.ndarray           # int64 [K]
    d: int
    tables: np.ndarray         # fp64 [sum rows][d]
    bot_W: list
    bot_b: list
    top_W: list
    top_b: list

    @property
    def K(self):
        return int(self.rows.size)

    def struct(self):
        self._bd = np.array([self.bot_W[0].shape[1]] + [w.shape[0] for w in self.bot_W], np.int32)
        self._td = np.array([self.top_W[0].shape[1]] + [w.shape[0] for w in self.top_W], np.int32)
        keep = [self.bot_W, self.bot_b, self.top_W, self.top_b]
        self._ptrs = [(C.c_void_p * len(v))(*[a.ctypes.data for a in v]) for v in keep]
        m = _Model(self.K, self.d, len(self.bot_W), len(self.top_W),
                   self._bd.ctypes.data_as(C.POINTER(C.c_int)), self._td.ctypes.data_as(C.POINTER(C.c_int)),
                   self._ptrs[0], self._ptrs[1], self._ptrs[2], self._ptrs[3],
                   self.rows.ctypes.data_as(C.POINTER(C.c_int64)),
                   C.c_void_p(self.tables.ctypes.data if self.tables.size else 0))
        self._struct = m
        return m


def layers_f64(layers, dtype: str):
    """Exact fp64 copies of synth layers, padding columns dropped."""
    Ws = [np.ascontiguousarray(gen.to_f64(L.W, dtype)[:, :L.n_in]) for L in layers]
    bs = [L.b.astype(np.float64) for L in layers]
    return Ws, bs


def model_from_config(cfg: Config, tables_stored: np.ndarray | None = None, rows=None,
                      bot=None, top=None) -> Model:
    """fp64 model from the seeded config (full tables: only for tables that fit in host RAM)."""
    if tables_stored is None:
        tables_stored = gen.full_tables(cfg)
    bot = bot if bot is not None else gen.mlp_layers(cfg, "bottom")
    top = top if top is not None else gen.mlp_layers(cfg, "top")
    bW, bb = layers_f64(bot, cfg.mlp_dtype)
    tW, tb = layers_f64(top, cfg.mlp_dtype)
    rows = np.asarray(cfg.rows if rows is None else rows, np.int64)
    return Model(rows, cfg.d, table_values(tables_stored, cfg.table_dtype).reshape(-1, cfg.d), bW, bb, tW, tb)


def sub_batch(cfg: Config, batch: gen.Batch, samples: np.ndarray):
    """Restrict a batch to ``samples`` and compact each table to the rows they use.

    Returns (B', dense', offsets', indices', labels', rows', table_ids_of_rows) where
    ``table_ids_of_rows[k]`` lists the original row id behind each compacted row.
    Only for batches with valid offsets and indices."""
    samples = np.asarray(samples, np.int64)
    K, B = cfg.K, cfg.B
    offs = batch.offsets.astype(np.int64)
    new_len, new_idx, used = [], [], []
    for k in range(K):
        starts, ends = offs[k * B + samples], offs[k * B + samples + 1]
        parts = [batch.indices[s:e] for s, e in zip(starts, ends)]
        flat = np.concatenate(parts) if parts else np.zeros(0, np.int32)
        uniq, inv = np.unique(flat, return_inverse=True)
        used.append(uniq.astype(np.int64))
        new_idx.append(inv.astype(np.int32))
        new_len.append(ends - starts)
    lens = np.stack(new_len).reshape(-1)
    offsets = np.zeros(lens.size + 1, np.int64)
    np.cumsum(lens, out=offsets[1:])
    labels = None if batch.labels is None else batch.labels[samples]
    return (samples.size, batch.dense[samples], offsets.astype(np.int32), np.concatenate(new_idx),
            labels, np.array([max(u.size, 0) for u in used], np.int64), used)


def model_for_rows(cfg: Config, used_rows: list, bot=None, top=None) -> Model:
    """fp64 model whose table k holds only rows ``used_rows[k]`` (generated on demand)."""
    parts = [gen.table_rows(gen.table_seed(cfg), k, cfg.rows[k], u, cfg.d, cfg.table_dtype)
             for k, u in enumerate(used_rows)]
    stored = np.concatenate(parts, axis=0) if parts else np.zeros((0, cfg.d))
    return model_from_config(cfg, stored, rows=[u.size for u in used_rows], bot=bot, top=top)


# ----------------------------------------------------------------- whole-model calls

def forward(model: Model, dense, offsets, indices, lib=None):
    """Returns (y_hat [B], logits [B], (n_oob, n_bad))."""
    lib = lib or load()
    dense, offsets, indices = _c64(dense), _i32(offsets), _i32(indices)
    B = dense.shape[0]
    y = np.zeros(B, np.float64)
    z = np.zeros(B, np.float64)
    counts = np.zeros(2, np.int64)
    s = model.struct()
    lib.oracle_forward(C.byref(s), B, indices.size, _p(dense), _p(offsets), _p(indices), _p(y), _p(z), _p(counts))
    return y, z, (int(counts[0]), int(counts[1]))


def concat(x_dense: np.ndarray, pooled: np.ndarray, lib=None) -> np.ndarray:
    """Concat-only interaction: [B][d] and [B][K][d] -> [B][d (K + 1)] = [x_dense, e_1 .. e_K]."""
    lib = lib or load()
    x_dense, pooled = _c64(x_dense), _c64(pooled)
    B, K, d = pooled.shape
    out = np.zeros((B, d * (K + 1)), np.float64)
    lib.oracle_concat(B, K, d, _p(x_dense), _p(pooled), _p(out))
    return out


def forward_cat(model: Model, dense, offsets, indices, lib=None):
    """The forward pass with the concat-only interaction: bottom MLP (ReLU after every layer), pooled
    bags, [x_dense, e_1 .. e_K], top MLP (last layer linear), sigmoid. Returns (y_hat, logits, counts)."""
    lib = lib or load()
    dense = _c64(dense)
    B = dense.shape[0]
    x = mlp(model.bot_W, model.bot_b, dense, relu_last=True, lib=lib)
    pooled, _, counts = embbag(model.tables, model.rows, model.d, B, offsets, indices, lib=lib)
    z = mlp(model.top_W, model.top_b, concat(x, pooled, lib=lib), relu_last=False, lib=lib)[:, 0]
    return 1.0 / (1.0 + np.exp(-z)), z, counts


def bce(z, y, lib=None) -> float:
    lib = lib or load()
    z, y = _c64(z), _c64(y)
    return float(lib.oracle_bce(z.size, _p(z), _p(y)))


def train_grads(model: Model, dense, offsets, indices, labels, lib=None) -> dict:
    """Loss, y_hat, all MLP gradients, per-row table gradients and occurrence counts."""
    lib = lib or load()
    dense, offsets, indices, labels = _c64(dense), _i32(offsets), _i32(indices), _c64(labels)
    B = dense.shape[0]
    bdW = [np.zeros_like(w) for w in model.bot_W]
    bdb = [np.zeros_like(b) for b in model.bot_b]
    tdW = [np.zeros_like(w) for w in model.top_W]
    tdb = [np.zeros_like(b) for b in model.top_b]
    ptr = lambda v: (C.c_void_p * len(v))(*[a.ctypes.data for a in v])  # noqa: E731
    tg = np.zeros_like(model.tables)
    cnt = np.zeros(model.tables.shape[0], np.int64)
    loss = np.zeros(1, np.float64)
    y = np.zeros(B, np.float64)
    counts = np.zeros(2, np.int64)
    out = {}
    s = model.struct()
    lib.oracle_train_grads(C.byref(s), B, indices.size, _p(dense), _p(offsets), _p(indices), _p(labels),
                           _p(loss), _p(y), ptr(bdW), ptr(bdb), ptr(tdW), ptr(tdb), _p(tg), _p(cnt), _p(counts))
    out.update({"loss": float(loss[0]), "y_hat": y, "bot_dW": bdW, "bot_db": bdb, "top_dW": tdW, "top_db": tdb,
                "table_grad": tg, "row_count": cnt, "counts": (int(counts[0]), int(counts[1]))})
    return out


def quantize_rows_u8(rows_f32: np.ndarray, lib=None):
    """Row-wise 8-bit quantisation of fp32 rows [n][d]: (codes uint8 [n][d], scale fp32 [n], offset fp32 [n])."""
    lib = lib or load()
    v = np.ascontiguousarray(rows_f32, dtype=np.float32)
    n, d = v.shape
    codes = np.zeros((n, d), np.uint8)
    scale = np.zeros(n, np.float32)
    offset = np.zeros(n, np.float32)
    if n:
        lib.oracle_quantize_rows_u8(n, d, _p(v), _p(codes), _p(scale), _p(offset))
    return codes, scale, offset


def dequantize_rows_u8(codes: np.ndarray, scale: np.ndarray, offset: np.ndarray, lib=None) -> np.ndarray:
    """fp64 values s * q + m of row-wise 8-bit rows."""
    lib = lib or load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    n, d = codes.shape
    out = np.zeros((n, d), np.float64)
    if n:
        lib.oracle_dequantize_rows_u8(n, d, _p(codes), _p(np.ascontiguousarray(scale, np.float32)),
                                      _p(np.ascontiguousarray(offset, np.float32)), _p(out))
    return out


def u8_records(codes: np.ndarray, scale: np.ndarray, offset: np.ndarray) -> np.ndarray:
    """The DLRM_U8ROW byte records [n][round_up(d + 8, 16)]: codes, fp32 scale, fp32 offset, zero padding."""
    n, d = codes.shape
    rb = (d + 8 + 15) // 16 * 16
    rec = np.zeros((n, rb), np.uint8)
    rec[:, :d] = codes
    rec[:, d:d + 4] = np.ascontiguousarray(scale, np.float32).view(np.uint8).reshape(n, 4)
    rec[:, d + 4:d + 8] = np.ascontiguousarray(offset, np.float32).view(np.uint8).reshape(n, 4)
    return rec


def table_values(stored: np.ndarray, dtype: str) -> np.ndarray:
    """fp64 values of stored table rows; row-wise 8-bit tables are stored as their fp32 source rows
    and quantised here."""
    if dtype == "u8row":
        return dequantize_rows_u8(*quantize_rows_u8(np.asarray(stored, np.float32)))
    return gen.to_f64(stored, dtype)


def sgd(w: np.ndarray, g: np.ndarray, lr: float, lib=None) -> np.ndarray:
    """Returns w - lr * g (fp64), leaving the input unchanged."""
    lib = lib or load()
    out = _c64(w).copy()
    g = _c64(g)
    lib.oracle_sgd(out.size, float(lr), _p(out), _p(g))
    return out
