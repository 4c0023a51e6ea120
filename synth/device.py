"""Place seeded inputs on the GPU (input generation only; torch for memory).

Small tables are generated on the host by ``synth.gen`` and copied; tables
too large for that are filled on the device by ``synth/fill.cu``, the
device twin of the same counter-based generator (checked bit-exact against
the host version by the GPU tests).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np
import torch

from . import gen
from .configs import Config

_HERE = os.path.dirname(os.path.abspath(__file__))
_FILL_SRC = os.path.join(_HERE, "fill.cu")
_FILL_LIB = os.path.join(_HERE, "libsynthfill.so")
_fill = None

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
DT_CODE = {"f32": 0, "f16": 1, "bf16": 2}


def build_fill() -> str:
    if not os.path.exists(_FILL_LIB) or os.path.getmtime(_FILL_LIB) < os.path.getmtime(_FILL_SRC):
        tmp = _FILL_LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-o", tmp, _FILL_SRC])
        os.replace(tmp, _FILL_LIB)
    return _FILL_LIB


def _fill_lib():
    global _fill
    if _fill is None:
        if not os.path.exists(_FILL_LIB):
            raise RuntimeError(f"{_FILL_LIB} is not built; call synth.device.build_fill()")
        L = C.CDLL(_FILL_LIB)
        L.synth_fill_table.restype = C.c_int
        L.synth_fill_table.argtypes = [C.c_void_p, C.c_int, C.c_longlong, C.c_int, C.c_int, C.c_ulonglong, C.c_float,
                                       C.c_void_p]
        _fill = L
    return _fill


def host_to_torch(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Storage-form numpy array (bf16 as uint16 bits) to a CPU torch tensor of the right dtype."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a))


def tables_on_device(cfg: Config, device="cuda", on_device_fill: bool | None = None, quantize=None) -> torch.Tensor:
    """All tables as one [sum rows][d] device tensor of the table dtype. Row-wise 8-bit tables
    ("u8row") come back as uint8 records [sum rows][record bytes]: each table's fp32 source rows are
    made on the device and handed to quantize(src_f32 [m][d], dst_records [m][rb]) (the caller's
    quantiser, e.g. the library's dlrm_quantize_rows_u8)."""
    total = int(sum(cfg.rows))
    if cfg.table_dtype == "u8row":
        if quantize is None:
            raise ValueError("row-wise 8-bit tables need a quantize callback")
        rb = (cfg.d + 8 + 15) // 16 * 16
        out = torch.empty((total, rb), dtype=torch.uint8, device=device)
        base = 0
        for k, m in enumerate(cfg.rows):
            src = _fill_table_f32(cfg, k, m, device)
            quantize(src, out[base:base + m])
            del src
            base += m
        return out
    if on_device_fill is None:
        on_device_fill = total * cfg.d > (1 << 26)
    if not on_device_fill:
        return host_to_torch(gen.full_tables(cfg), cfg.table_dtype).to(device)
    out = torch.empty((total, cfg.d), dtype=TORCH_DT[cfg.table_dtype], device=device)
    L = _fill_lib()
    stream = torch.cuda.current_stream(device).cuda_stream
    base = 0
    es = out.element_size()
    for k, m in enumerate(cfg.rows):
        ptr = out.data_ptr() + base * cfg.d * es
        r = L.synth_fill_table(ptr, DT_CODE[cfg.table_dtype], m, cfg.d, k, gen.table_seed(cfg),
                               float(gen.table_scale(m)), stream)
        if r != 0:
            raise RuntimeError(f"synth_fill_table failed: cudaError {r}")
        base += m
    return out


def _fill_table_f32(cfg: Config, k: int, m: int, device) -> torch.Tensor:
    """fp32 source rows of table k on the device (the same values as gen.table_rows_f32)."""
    src = torch.empty((m, cfg.d), dtype=torch.float32, device=device)
    if m * cfg.d <= (1 << 24):
        src.copy_(torch.from_numpy(gen.table_rows_f32(gen.table_seed(cfg), k, m, np.arange(m), cfg.d)))
        return src
    L = _fill_lib()
    r = L.synth_fill_table(src.data_ptr(), DT_CODE["f32"], m, cfg.d, k, gen.table_seed(cfg),
                           float(gen.table_scale(m)), torch.cuda.current_stream(device).cuda_stream)
    if r != 0:
        raise RuntimeError(f"synth_fill_table failed: cudaError {r}")
    return src


def mlp_on_device(cfg: Config, which: str, device="cuda"):
    """(Ws, bs, dims): device weights [out][ld] in the MLP dtype and fp32 biases."""
    layers = gen.mlp_layers(cfg, which)
    Ws = [host_to_torch(L.W, cfg.mlp_dtype).to(device) for L in layers]
    bs = [torch.from_numpy(L.b).to(device) for L in layers]
    dims = [layers[0].n_in] + [L.n_out for L in layers]
    return Ws, bs, dims


def batch_on_device(batch: gen.Batch, device="cuda", pin: bool = False):
    """dict of device tensors (or pinned host tensors if pin) for one batch."""
    t = {"dense": torch.from_numpy(batch.dense), "offsets": torch.from_numpy(batch.offsets),
         "indices": torch.from_numpy(batch.indices)}
    if batch.labels is not None:
        t["labels"] = torch.from_numpy(batch.labels)
    if pin:
        return {k: v.pin_memory() for k, v in t.items()}
    return {k: v.to(device) for k, v in t.items()}
