"""Seeded synthetic inputs for the DLRM hot path (shared by the oracle and the CUDA side).

Everything here is input generation: table contents, dense features, CSR bags,
MLP parameters and labels. None of the method's arithmetic (pooling,
interaction, MLP, loss, gradients) lives here.

Embedding-table contents come from a counter-based generator so that any row
can be produced on demand, on the host (this file) or on the device
(``synth/fill.cu``), without materialising tables that do not fit in host RAM.
The generator is SplitMix64 as published by Steele, Lea and Flood,
"Fast splittable pseudorandom number generators" (OOPSLA 2014): output n of the
stream whose state starts at ``seed`` is ``mix(seed + (n + 1) * GAMMA)``.

Element (table k, row r, column c) uses counter ``(k << 40) + r * d + c`` and
becomes ``fp32(fp32((2u - 2^24) * 2^-24) * fp32(1/sqrt(m_k)))`` with ``u`` the
top 24 bits of the 64-bit output, i.e. U(-1/sqrt(m_k), 1/sqrt(m_k)) as the
workloads ask; 16-bit tables take that fp32 value rounded to nearest-even.
All other streams use numpy's PCG64 seeded by ``SeedSequence([seed, stream, ...])``.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .configs import Config, ld_pad

GAMMA = np.uint64(0x9E3779B97F4A7C15)
MIX1 = np.uint64(0xBF58476D1CE4E5B9)
MIX2 = np.uint64(0x94D049BB133111EB)

# numpy PCG64 stream ids (first word after the seed in the SeedSequence entropy)
S_DENSE, S_BAGLEN, S_INDEX, S_PERM, S_WEIGHT, S_LABEL = 1, 2, 3, 4, 5, 6


def splitmix64_at(seed: int, n: np.ndarray) -> np.ndarray:
    """Output number ``n`` (0-based, uint64 array) of the SplitMix64 stream starting at ``seed``."""
    n = np.asarray(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (n + np.uint64(1)) * GAMMA
        z = (z ^ (z >> np.uint64(30))) * MIX1
        z = (z ^ (z >> np.uint64(27))) * MIX2
        return z ^ (z >> np.uint64(31))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, nearest-even, returning the 16-bit patterns (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def table_scale(m: int) -> np.float32:
    """fp32(1/sqrt(m)), computed once in fp64."""
    return np.float32(1.0 / np.sqrt(float(m)))


def table_rows_f32(seed: int, table_id: int, m: int, row_ids: np.ndarray, d: int) -> np.ndarray:
    """fp32 values of the given rows of table ``table_id`` (m rows of width d)."""
    row_ids = np.asarray(row_ids, dtype=np.uint64).reshape(-1)
    n = (np.uint64(table_id) << np.uint64(40)) + row_ids[:, None] * np.uint64(d) + np.arange(d, dtype=np.uint64)[None, :]
    z = splitmix64_at(seed, n)
    u = (z >> np.uint64(40)).astype(np.int64)
    t = (2 * u - (1 << 24)).astype(np.float32)              # exact: |t| <= 2^24
    v = (t * np.float32(2.0 ** -24)) * table_scale(m)        # one fp32 rounding
    return v.astype(np.float32)


def table_rows(seed: int, table_id: int, m: int, row_ids: np.ndarray, d: int, dtype: str) -> np.ndarray:
    """Rows in storage form: float32, float16, or uint16 bf16 bit patterns."""
    v = table_rows_f32(seed, table_id, m, row_ids, d)
    if dtype == "f32":
        return v
    if dtype == "f16":
        return v.astype(np.float16)
    if dtype == "bf16":
        return f32_to_bf16_bits(v)
    if dtype == "u8row":
        return v   # row-wise 8-bit tables: the fp32 source rows; quantisation belongs to the consumers
    raise ValueError(dtype)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to fp64."""
    if dtype == "bf16":
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a).astype(np.float64)


def table_seed(cfg: Config) -> int:
    return int(cfg.seed)


def full_tables(cfg: Config) -> np.ndarray:
    """All tables in one contiguous row-major buffer (only for tables that fit in host RAM)."""
    parts = [table_rows(table_seed(cfg), k, m, np.arange(m), cfg.d, cfg.table_dtype) for k, m in enumerate(cfg.rows)]
    return np.concatenate(parts, axis=0)


def row_base(cfg: Config) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(cfg.rows, dtype=np.int64))[:-1]]).astype(np.int64)


# --------------------------------------------------------------------------- batches

def _rng(*words) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(w) for w in words])))


def dense_features(cfg: Config, batch: int) -> np.ndarray:
    rng = _rng(cfg.seed, S_DENSE, batch)
    shape = (cfg.B, cfg.n_dense)
    if cfg.dense == "normal":
        return rng.standard_normal(shape).astype(np.float32)
    if cfg.dense == "log1p_poisson3":
        return np.log1p(rng.poisson(3.0, shape).astype(np.float64)).astype(np.float32)
    raise ValueError(cfg.dense)


def bag_lengths(cfg: Config, batch: int) -> np.ndarray:
    """int64 [K][B] bag lengths (table-major, as the CSR offsets are laid out)."""
    rng = _rng(cfg.seed, S_BAGLEN, batch)
    K, B = cfg.K, cfg.B
    if cfg.bag == "one":
        return np.ones((K, B), np.int64)
    if cfg.bag == "poisson20":
        return np.clip(rng.poisson(20.0, (K, B)), 1, 64).astype(np.int64)
    if cfg.bag == "uniform100":
        return rng.integers(1, 101, (K, B)).astype(np.int64)
    if cfg.bag == "mix":          # 0..4 rows per bag: exercises empty and multi-row bags
        return rng.integers(0, 5, (K, B)).astype(np.int64)
    if cfg.bag.startswith("fixed:"):
        return np.full((K, B), int(cfg.bag.split(":")[1]), np.int64)
    raise ValueError(cfg.bag)


def zipf_ranks(rng: np.random.Generator, alpha: float, m: int, n: int) -> np.ndarray:
    """n ranks in 1..m with P(r) proportional to r^-alpha, by rejection from numpy's unbounded Zipf."""
    out = np.empty(n, np.int64)
    filled = 0
    while filled < n:
        need = n - filled
        draw = rng.zipf(alpha, size=2 * need + 1024)
        ok = draw[draw <= m]
        take = min(ok.size, need)
        out[filled:filled + take] = ok[:take]
        filled += take
    return out


def table_permutation(cfg: Config, k: int) -> np.ndarray:
    """Per-table random permutation of rows; Zipf rank r maps to row perm[r - 1]."""
    return _rng(cfg.seed, S_PERM, k).permutation(cfg.rows[k])


@dataclass
class Batch:
    dense: np.ndarray            # float32 [B][13]
    offsets: np.ndarray          # int32 [K*B + 1], bag (k, b) is offsets[k*B + b] .. offsets[k*B + b + 1]
    indices: np.ndarray          # int32 [nnz], row ids local to their table
    labels: np.ndarray | None    # float32 [B] of 0/1, training only


def make_batches(cfg: Config, batch_ids=(0,), perms: dict | None = None) -> list:
    """Seeded batches; the Zipf permutation of each table is shared by all batches."""
    K, B = cfg.K, cfg.B
    lens = {j: bag_lengths(cfg, j) for j in batch_ids}
    idx = {j: [] for j in batch_ids}
    for k in range(K):
        m = cfg.rows[k]
        perm = None
        for j in batch_ids:
            n = int(lens[j][k].sum())
            rng = _rng(cfg.seed, S_INDEX, j, k)
            if cfg.index == "uniform":
                r = rng.integers(0, m, n)
            elif cfg.index.startswith("zipf:"):
                if perm is None:
                    perm = perms[k] if perms is not None and k in perms else table_permutation(cfg, k)
                r = perm[zipf_ranks(rng, float(cfg.index.split(":")[1]), m, n) - 1]
            else:
                raise ValueError(cfg.index)
            idx[j].append(r.astype(np.int32))
    out = []
    for j in batch_ids:
        flat = lens[j].reshape(-1)
        offs = np.zeros(K * B + 1, np.int64)
        np.cumsum(flat, out=offs[1:])
        if offs[-1] >= 2 ** 31:
            raise ValueError("nnz must stay below 2^31")
        dense = dense_features(cfg, j)
        labels = make_labels(cfg, j, dense) if cfg.training else None
        out.append(Batch(dense, offs.astype(np.int32), np.concatenate(idx[j]) if K else np.zeros(0, np.int32), labels))
    return out


def make_labels(cfg: Config, batch: int, dense: np.ndarray) -> np.ndarray:
    """Bernoulli(sigmoid(w . dense)) click labels, w ~ N(0, 1/13), seeded."""
    rng = _rng(cfg.seed, S_LABEL, batch)
    w = rng.normal(0.0, np.sqrt(1.0 / cfg.n_dense), cfg.n_dense)
    s = dense.astype(np.float64) @ w
    p = 1.0 / (1.0 + np.exp(-s))
    return (rng.random(cfg.B) < p).astype(np.float32)


# --------------------------------------------------------------------------- MLP parameters

@dataclass
class Layer:
    W: np.ndarray   # [out][ld] in storage form (float32, float16 or bf16 bits); columns >= in are 0
    b: np.ndarray   # float32 [out]
    n_in: int
    n_out: int
    ld: int


def mlp_layers(cfg: Config, which: str) -> list:
    """Xavier-uniform weights U(+-sqrt(6/(in+out))) and biases U(+-1/sqrt(in))."""
    dims = cfg.bottom if which == "bottom" else cfg.top
    tag = 0 if which == "bottom" else 1
    layers = []
    for l in range(len(dims) - 1):
        n_in, n_out = dims[l], dims[l + 1]
        rng = _rng(cfg.seed, S_WEIGHT, tag, l)
        a = np.sqrt(6.0 / (n_in + n_out))
        w32 = rng.uniform(-a, a, (n_out, n_in)).astype(np.float32)
        b32 = rng.uniform(-1.0 / np.sqrt(n_in), 1.0 / np.sqrt(n_in), n_out).astype(np.float32)
        ld = ld_pad(n_in, cfg.mlp_dtype)
        if cfg.mlp_dtype == "f32":
            W = np.zeros((n_out, ld), np.float32)
            W[:, :n_in] = w32
        elif cfg.mlp_dtype == "bf16":
            W = np.zeros((n_out, ld), np.uint16)
            W[:, :n_in] = f32_to_bf16_bits(w32)
        elif cfg.mlp_dtype == "f16":
            W = np.zeros((n_out, ld), np.float16)
            W[:, :n_in] = w32.astype(np.float16)
        else:
            raise ValueError(cfg.mlp_dtype)
        layers.append(Layer(W, b32, n_in, n_out, ld))
    return layers
