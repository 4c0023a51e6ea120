"""Workload shapes for the DLRM hot path, as plain data.

The five workloads follow the DLRM architecture of "Deep Learning
Recommendation Model (DLRM)" (nadeemcite summary, Key Method Details) and
"DLRM" (briansu.co, section 4 Key equations): K embedding tables of width d,
a bottom MLP mapping the 13 dense features to d, the pairwise interaction over
K+1 vectors and a top MLP ending in one logit. Sizes, dtypes and input
distributions are the synthetic stand-ins for the Criteo click-log workload
the pages train on; no item of that dataset is used.

This module holds no arithmetic of the method. It is shared by the oracle
side and the CUDA side only as a description of the inputs.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

ESIZE = {"f32": 4, "f16": 2, "bf16": 2}


def ld_pad(n: int, dtype: str) -> int:
    """Smallest leading dimension >= n whose row is a multiple of 16 bytes."""
    per = 16 // ESIZE[dtype]
    return (n + per - 1) // per * per


@dataclass(frozen=True)
class Config:
    name: str
    B: int                      # batch size (samples)
    rows: tuple                 # m_k, one per table
    d: int                      # shared embedding width
    table_dtype: str            # "f32" | "f16" | "bf16" | "u8row" (row-wise 8-bit: fp32 source rows, quantised by the user)
    mlp_dtype: str              # dtype of MLP weights and hidden activations
    bag: str                    # "one" | "poisson20" | "uniform100" | "fixed:<n>" | "mix"
    index: str                  # "uniform" | "zipf:<alpha>"
    dense: str                  # "normal" | "log1p_poisson3"
    bottom: tuple               # layer widths, first is 13, last is d
    top: tuple                  # layer widths, first is the concat width, last is 1
    training: bool = False
    lr: float = 0.01
    seed: int = 0
    interaction: str = "dot"    # "dot": [x_dense, Z] (the pages' DLRM); "cat": [x_dense, e_1..e_K] (concat-only)

    @property
    def K(self) -> int:
        return len(self.rows)

    @property
    def P(self) -> int:
        """Number of interaction terms: the strict lower triangle of (K+1)x(K+1)."""
        return self.K * (self.K + 1) // 2

    @property
    def concat_width(self) -> int:
        return self.d + self.P if self.interaction == "dot" else self.d * (self.K + 1)

    @property
    def concat_ld(self) -> int:
        return ld_pad(self.concat_width, self.mlp_dtype)

    @property
    def n_dense(self) -> int:
        return self.bottom[0]

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)

    def check(self) -> None:
        assert self.bottom[-1] == self.d, "bottom MLP must end at d"
        assert self.interaction in ("dot", "cat")
        assert self.top[0] == self.concat_width, "top MLP must start at the concat width"
        assert self.top[-1] == 1, "top MLP must end in one logit"


def _logspaced_rows(lo: float, hi: float, n: int) -> tuple:
    return tuple(int(v) for v in np.round(np.logspace(np.log10(lo), np.log10(hi), n)).astype(np.int64))


LARGE_ROWS = _logspaced_rows(1e3, 4e7, 26)

CONFIGS = {
    # Tiny forward, fp32: 8 tables of 1000 x 16, one uniform index per bag.
    "tiny": Config("tiny", B=128, rows=(1000,) * 8, d=16, table_dtype="f32", mlp_dtype="f32",
                   bag="one", index="uniform", dense="normal",
                   bottom=(13, 64, 16), top=(52, 64, 1)),
    # Medium forward, fp32: 26 tables of 100k x 64, multi-hot Poisson(20) bags.
    "medium": Config("medium", B=2048, rows=(100_000,) * 26, d=64, table_dtype="f32", mlp_dtype="f32",
                     bag="poisson20", index="uniform", dense="normal",
                     bottom=(13, 512, 256, 64), top=(415, 512, 256, 1)),
    # Large memory-bound forward, bf16 tables: 26 log-spaced tables, one-hot Zipf(1.05).
    "large": Config("large", B=65536, rows=LARGE_ROWS, d=128, table_dtype="bf16", mlp_dtype="bf16",
                    bag="one", index="zipf:1.05", dense="log1p_poisson3",
                    bottom=(13, 512, 256, 128), top=(479, 1024, 1024, 512, 256, 1)),
    # EmbeddingBag-heavy stress, bf16: 100 tables of 1M x 64, U[1,100] bags, Zipf(1.2).
    "stress": Config("stress", B=16384, rows=(1_000_000,) * 100, d=64, table_dtype="bf16", mlp_dtype="bf16",
                     bag="uniform100", index="zipf:1.2", dense="normal",
                     bottom=(13, 256, 64), top=(5114, 1024, 1)),
    # Training step on the large shapes with fp32 tables at a quarter of the rows.
    "train": Config("train", B=65536, rows=tuple(r // 4 for r in LARGE_ROWS), d=128, table_dtype="f32",
                    mlp_dtype="f32", bag="one", index="zipf:1.05", dense="log1p_poisson3",
                    bottom=(13, 512, 256, 128), top=(479, 1024, 1024, 512, 256, 1), training=True),
    # The large forward with the concat-only interaction (top MLP input [x_dense, e_1..e_26] = 3456 wide).
    "large-cat": Config("large-cat", B=65536, rows=LARGE_ROWS, d=128, table_dtype="bf16", mlp_dtype="bf16",
                        bag="one", index="zipf:1.05", dense="log1p_poisson3",
                        bottom=(13, 512, 256, 128), top=(3456, 1024, 1024, 512, 256, 1), interaction="cat"),
    # The large forward with row-wise 8-bit tables (d uint8 codes + fp32 scale and offset per row).
    "large-u8": Config("large-u8", B=65536, rows=LARGE_ROWS, d=128, table_dtype="u8row", mlp_dtype="bf16",
                       bag="one", index="zipf:1.05", dense="log1p_poisson3",
                       bottom=(13, 512, 256, 128), top=(479, 1024, 1024, 512, 256, 1)),
}

for _c in CONFIGS.values():
    _c.check()


def shrink(cfg: Config, B: int | None = None, rows_cap: int | None = None, name: str | None = None) -> Config:
    """Same structure, smaller batch and/or tables (for oracle-sized parity cases)."""
    rows = cfg.rows if rows_cap is None else tuple(min(r, rows_cap) for r in cfg.rows)
    return cfg.with_(B=cfg.B if B is None else B, rows=rows, name=name or f"{cfg.name}-small")
