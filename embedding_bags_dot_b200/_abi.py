"""ctypes binding of libdlrm.so.

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of libdlrm.so. PyTorch provides device memory and streams. The
functions keep the C names (``dlrm_forward`` ...) and take torch tensors;
a non-OK status raises ``DlrmError`` carrying the status code.

There is no CPU fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdlrm.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_INDEX_OOB, ERR_BAD_OFFSETS, ERR_TIMEOUT, ERR_CUDA, ERR_WORKSPACE = range(8)
F32, F16, BF16 = 0, 1, 2
ACT_NONE, ACT_RELU, ACT_SIGMOID = 0, 1, 2
MAX_TABLES = 256
MAX_LAYERS = 16
ERR_RECORD_BYTES = 256
NOALLOC_SCRATCH_BYTES = 32 << 20

U8ROW = 3   # row-wise 8-bit table records (tables only)
DT_CODE = {"f32": F32, "f16": F16, "bf16": BF16, "u8row": U8ROW, torch.float32: F32, torch.float16: F16,
           torch.bfloat16: BF16, torch.uint8: U8ROW}
DT_TORCH = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


class DlrmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: status {status} ({status_str(status)})")


class dlrm_tables(C.Structure):
    _fields_ = [("data", C.c_void_p), ("rows", C.POINTER(C.c_int64)), ("K", C.c_int), ("d", C.c_int), ("dt", C.c_int)]


class dlrm_mlp(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("dims", C.POINTER(C.c_int)), ("W", C.POINTER(C.c_void_p)),
                ("b", C.POINTER(C.c_void_p)), ("dt", C.c_int)]


_lib = None
_lock = threading.Lock()

_SIGS = {
    "dlrm_launch_count": (C.c_uint64, []),
    "dlrm_set_wait_polls": (C.c_int, [C.c_int64]),
    "dlrm_pooled_assemble": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                                       C.c_void_p, C.c_void_p]),
    "dlrm_pooled_split": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                                    C.c_void_p, C.c_void_p]),
    "dlrm_embbag_sgd_scratch_size": (C.c_size_t, [C.c_void_p, C.c_int, C.c_int64]),
    "dlrm_backward_pooled_workspace_size": (C.c_size_t, [C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_int]),
    "dlrm_grads_pooled_size": (C.c_size_t, [C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_int]),
    "dlrm_grads_pooled_offsets": (C.c_int, [C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                            C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dlrm_backward_pooled": (C.c_int, [C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                       C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p,
                                       C.c_size_t, C.c_void_p]),
    "dlrm_mlp_sgd": (C.c_int, [C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_float, C.c_void_p, C.c_size_t,
                               C.c_void_p]),
    "dlrm_embbag_sgd": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_float,
                                  C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p]),
    "dlrm_ld": (C.c_int, [C.c_int, C.c_int]),
    "dlrm_status_str": (C.c_char_p, [C.c_int]),
    "dlrm_workspace_size": (C.c_size_t, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int]),
    "dlrm_mlp_workspace_size": (C.c_size_t, [C.c_void_p, C.c_int, C.c_int]),
    "dlrm_forward_lengths": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                       C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_offsets_from_lengths_workspace_size": (C.c_size_t, [C.c_int64]),
    "dlrm_offsets_from_lengths": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_check_error": (C.c_int, [C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p]),
    "dlrm_embbag_fwd": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p,
                                  C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_interact_fwd": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                                    C.c_void_p]),
    "dlrm_embbag_interact_fwd": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p,
                                           C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_mlp_fwd": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_int,
                               C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_forward": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                               C.c_int64, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_grads_size": (C.c_size_t, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int64]),
    "dlrm_grads_offsets": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int64, C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dlrm_backward": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                                C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p,
                                C.c_size_t, C.c_void_p]),
    "dlrm_sparse_sgd": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_void_p,
                                  C.c_size_t, C.c_void_p, C.c_void_p]),
    "dlrm_embedding_row_grads": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int64, C.c_void_p,
                                           C.c_size_t, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dlrm_forward_noalloc": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                       C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dlrm_gemm_f32_workspace_size": (C.c_size_t, [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]),
    "dlrm_row_bytes": (C.c_size_t, [C.c_int, C.c_int]),
    "dlrm_embbag_cat_fwd": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p,
                                      C.c_int, C.c_int, C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_forward_cat": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                                   C.c_int64, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_quantize_rows_u8": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int, C.c_void_p, C.c_void_p]),
    "dlrm_gemm_f32": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int,
                                C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_size_t, C.c_void_p]),
    "dlrm_tf32_split": (C.c_int, [C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int,
                                  C.c_void_p]),
    "dlrm_gemm_tf32x3_workspace_size": (C.c_size_t, [C.c_int, C.c_int, C.c_int]),
    "dlrm_gemm_tf32x3": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                                   C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_size_t,
                                   C.c_void_p]),
}


def lib():
    """Load libdlrm.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libdlrm.so is not built ({LIB_PATH}); run `python -m embedding_bags_dot_b200.build`")
            L = C.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def status_str(s: int) -> str:
    try:
        return lib().dlrm_status_str(int(s)).decode()
    except Exception:  # noqa: BLE001 - only used for messages
        return "?"


def _check(status: int, where: str) -> int:
    if status != OK:
        raise DlrmError(status, where)
    return status


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr() if t.numel() else None


def _stream(stream):
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def dlrm_launch_count() -> int:
    return int(lib().dlrm_launch_count())


def dlrm_set_wait_polls(polls: int) -> None:
    """Test hook: polls of the first bounded waits on the current device (< 0: the defaults)."""
    _check(lib().dlrm_set_wait_polls(int(polls)), "dlrm_set_wait_polls")


def dlrm_ld(n: int, dt) -> int:
    return int(lib().dlrm_ld(int(n), DT_CODE.get(dt, dt)))


# ----------------------------------------------------------------- model containers

class Tables:
    """K tables in one contiguous device buffer ([sum rows][d], or [sum rows][record bytes] uint8 for
    row-wise 8-bit tables) plus host row counts."""

    def __init__(self, data: torch.Tensor, rows, d: int):
        assert data.is_cuda and data.is_contiguous()
        self.data = data
        self.rows = [int(r) for r in rows]
        self.d = int(d)
        self._rows = (C.c_int64 * len(self.rows))(*self.rows)
        self.struct = dlrm_tables(data.data_ptr(), self._rows, len(self.rows), self.d, DT_CODE[data.dtype])

    @property
    def K(self):
        return len(self.rows)

    def ref(self):
        return C.byref(self.struct)


class MLP:
    """Layers W[l] ([out][dlrm_ld(in)] device tensors) and fp32 biases b[l]."""

    def __init__(self, Ws, bs, dims):
        self.Ws, self.bs, self.dims = list(Ws), list(bs), [int(x) for x in dims]
        assert len(self.Ws) == len(self.bs) == len(self.dims) - 1
        self.dt = DT_CODE[self.Ws[0].dtype]
        self._dims = (C.c_int * len(self.dims))(*self.dims)
        self._W = (C.c_void_p * len(self.Ws))(*[w.data_ptr() for w in self.Ws])
        self._b = (C.c_void_p * len(self.bs))(*[b.data_ptr() for b in self.bs])
        self.struct = dlrm_mlp(len(self.Ws), self._dims, self._W, self._b, self.dt)

    def ref(self):
        return C.byref(self.struct)


def _ref(x):
    return None if x is None else x.ref()


# ----------------------------------------------------------------- entry points (C names)

def dlrm_workspace_size(T: Tables, bot: MLP, top: MLP, B: int, training: int = 0) -> int:
    return int(lib().dlrm_workspace_size(_ref(T), _ref(bot), _ref(top), int(B), int(training)))


def dlrm_mlp_workspace_size(mlp: MLP, B: int, in_dt) -> int:
    return int(lib().dlrm_mlp_workspace_size(mlp.ref(), int(B), int(DT_CODE.get(in_dt, in_dt))))


def _nbytes(buf) -> int:
    """Size in bytes of a caller buffer (a tensor), passed to the C entry points, which refuse short ones."""
    if buf is None:
        return 0
    return int(buf.numel() * buf.element_size())


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zero-filled workspace (the error record must start at zero)."""
    return torch.zeros(max(int(nbytes), ERR_RECORD_BYTES), dtype=torch.uint8, device=device)


def dlrm_check_error(ws: torch.Tensor, stream=None):
    """Returns (status, flags, n_skipped_indices, n_bad_bags) and clears the record."""
    info = (C.c_int64 * 3)()
    s = lib().dlrm_check_error(_ptr(ws), _nbytes(ws), _stream(stream), info)
    return int(s), int(info[0]), int(info[1]), int(info[2])


def dlrm_embbag_fwd(T: Tables, B: int, offsets, indices, pooled, bag_len=None, ws=None, stream=None):
    return _check(lib().dlrm_embbag_fwd(T.ref(), int(B), _ptr(offsets), _ptr(indices), int(indices.numel()),
                                        _ptr(pooled), _ptr(bag_len), _ptr(ws), _nbytes(ws), _stream(stream)),
                  "dlrm_embbag_fwd")


def dlrm_interact_fwd(B: int, K: int, d: int, x_dense, pooled, concat, ld: int, out_dt=None, stream=None):
    out_dt = DT_CODE[concat.dtype] if out_dt is None else DT_CODE.get(out_dt, out_dt)
    return _check(lib().dlrm_interact_fwd(int(B), int(K), int(d), _ptr(x_dense), _ptr(pooled), _ptr(concat), int(ld),
                                          int(out_dt), _stream(stream)), "dlrm_interact_fwd")


def dlrm_embbag_interact_fwd(T: Tables, B: int, offsets, indices, x_dense, concat, ld: int, out_dt=None, ws=None,
                             stream=None):
    out_dt = DT_CODE[concat.dtype] if out_dt is None else DT_CODE.get(out_dt, out_dt)
    return _check(lib().dlrm_embbag_interact_fwd(T.ref(), int(B), _ptr(offsets), _ptr(indices), int(indices.numel()),
                                                 _ptr(x_dense), _ptr(concat), int(ld), int(out_dt), _ptr(ws),
                                                 _nbytes(ws), _stream(stream)), "dlrm_embbag_interact_fwd")


def _need(t, dtype, rows: int, ld: int, width: int, where: str) -> None:
    """Refuses a buffer of the wrong dtype, or too short for `rows` rows of `width` values `ld` apart: the C
    entry points receive bare pointers and would read or write past its end."""
    if t is None or (dtype is not None and t.dtype != dtype) or \
            (rows > 0 and t.numel() < (rows - 1) * ld + width):
        raise DlrmError(ERR_INVALID_ARG, where)


def dlrm_mlp_fwd(mlp: MLP, B: int, inp, ld_in: int, out, ld_out: int, final_act: int, ws, stream=None):
    """out: fp32 [B][ld_out] (the last layer's output is always fp32); inp: [B][ld_in] fp32 or the MLP dtype."""
    _need(inp, None, int(B), int(ld_in), mlp.dims[0], "dlrm_mlp_fwd")
    _need(out, torch.float32, int(B), int(ld_out), mlp.dims[-1], "dlrm_mlp_fwd")
    return _check(lib().dlrm_mlp_fwd(mlp.ref(), int(B), _ptr(inp), DT_CODE[inp.dtype], int(ld_in), _ptr(out),
                                     int(ld_out), int(final_act), _ptr(ws), _nbytes(ws), _stream(stream)),
                  "dlrm_mlp_fwd")


def dlrm_forward(T: Tables, bot: MLP, top: MLP, B: int, dense, offsets, indices, y_hat, ws, stream=None):
    _need(dense, torch.float32, int(B), bot.dims[0], bot.dims[0], "dlrm_forward")
    _need(y_hat, torch.float32, int(B), 1, 1, "dlrm_forward")
    return _check(lib().dlrm_forward(T.ref(), bot.ref(), top.ref(), int(B), _ptr(dense), _ptr(offsets),
                                     _ptr(indices), int(indices.numel()), _ptr(y_hat), _ptr(ws), _nbytes(ws),
                                     _stream(stream)), "dlrm_forward")


def dlrm_forward_lengths(T: Tables, bot: MLP, top: MLP, B: int, dense, lengths, indices, y_hat, ws, stream=None):
    """dlrm_forward with uint8 bag lengths [K * B] in place of CSR offsets."""
    if lengths.dtype != torch.uint8:
        raise DlrmError(ERR_INVALID_ARG, "dlrm_forward_lengths")
    return _check(lib().dlrm_forward_lengths(T.ref(), bot.ref(), top.ref(), int(B), _ptr(dense), _ptr(lengths),
                                             _ptr(indices), int(indices.numel()), _ptr(y_hat), _ptr(ws),
                                             _nbytes(ws), _stream(stream)), "dlrm_forward_lengths")


def dlrm_offsets_from_lengths_workspace_size(n: int) -> int:
    return int(lib().dlrm_offsets_from_lengths_workspace_size(int(n)))


def dlrm_offsets_from_lengths(lengths, offsets, ws, stream=None):
    """offsets[i] = sum of lengths[0..i) for i <= n; uint8 lengths [n], int32 offsets [n + 1]."""
    n = lengths.numel()
    if lengths.dtype != torch.uint8 or offsets.dtype != torch.int32 or offsets.numel() < n + 1:
        raise DlrmError(ERR_INVALID_ARG, "dlrm_offsets_from_lengths")
    return _check(lib().dlrm_offsets_from_lengths(_ptr(lengths), int(n), _ptr(offsets), _ptr(ws), _nbytes(ws),
                                                  _stream(stream)), "dlrm_offsets_from_lengths")


def dlrm_embbag_cat_fwd(T: Tables, B: int, offsets, indices, x_dense, concat, ld: int, out_dt=None, ws=None,
                        stream=None):
    """Concat-only interaction: concat rows [x_dense, e_1 .. e_K, zeros]."""
    out_dt = DT_CODE[concat.dtype] if out_dt is None else DT_CODE.get(out_dt, out_dt)
    return _check(lib().dlrm_embbag_cat_fwd(T.ref(), int(B), _ptr(offsets), _ptr(indices), int(indices.numel()),
                                            _ptr(x_dense), _ptr(concat), int(ld), int(out_dt), _ptr(ws),
                                            _nbytes(ws), _stream(stream)), "dlrm_embbag_cat_fwd")


def dlrm_forward_cat(T: Tables, bot: MLP, top: MLP, B: int, dense, offsets, indices, y_hat, ws, stream=None):
    """dlrm_forward with the concat-only interaction (top MLP input width d (K + 1))."""
    return _check(lib().dlrm_forward_cat(T.ref(), bot.ref(), top.ref(), int(B), _ptr(dense), _ptr(offsets),
                                         _ptr(indices), int(indices.numel()), _ptr(y_hat), _ptr(ws), _nbytes(ws),
                                         _stream(stream)), "dlrm_forward_cat")


def dlrm_forward_noalloc(T: Tables, bot: MLP, top: MLP, B: int, dense, offsets, indices, y_hat, err_flags=None,
                         stream=None):
    """dlrm_forward without a workspace: the library's fixed device scratch array is used instead
    (for callers that cannot allocate device memory; see include/dlrm.h)."""
    return _check(lib().dlrm_forward_noalloc(T.ref(), bot.ref(), top.ref(), int(B), _ptr(dense), _ptr(offsets),
                                             _ptr(indices), int(indices.numel()), _ptr(y_hat), _ptr(err_flags),
                                             _stream(stream)), "dlrm_forward_noalloc")


def dlrm_row_bytes(d: int, dt) -> int:
    return int(lib().dlrm_row_bytes(int(d), DT_CODE.get(dt, dt)))


def dlrm_quantize_rows_u8(src, dst, stream=None):
    """Row-wise 8-bit records dst (uint8 [rows][dlrm_row_bytes(d, U8ROW)]) from src (fp32 or bf16 [rows][d])."""
    rows, d = src.shape
    assert dst.dtype == torch.uint8 and dst.shape[0] == rows and dst.shape[1] == dlrm_row_bytes(d, U8ROW)
    return _check(lib().dlrm_quantize_rows_u8(_ptr(src), DT_CODE[src.dtype], int(rows), int(d), _ptr(dst),
                                              _stream(stream)), "dlrm_quantize_rows_u8")


# ----------------------------------------------------------------- fp32 GEMM (tensor cores, 3xTF32)

def dlrm_gemm_f32_workspace_size(I: int, J: int, R: int, a_mn: bool, b_mn: bool) -> int:
    return int(lib().dlrm_gemm_f32_workspace_size(int(I), int(J), int(R), int(bool(a_mn)), int(bool(b_mn))))


def dlrm_gemm_f32(I: int, J: int, R: int, A, lda: int, a_mn: bool, B, ldb: int, b_mn: bool, C, ldc: int, ws,
                  stream=None):
    """C[i][j] = sum_r A(i, r) B(j, r) in fp32 on the tensor cores; A(i, r) = A[i][r], or A[r][i] when a_mn
    (B likewise)."""
    return _check(lib().dlrm_gemm_f32(int(I), int(J), int(R), _ptr(A), int(lda), int(bool(a_mn)), _ptr(B), int(ldb),
                                      int(bool(b_mn)), _ptr(C), int(ldc), _ptr(ws), _nbytes(ws), _stream(stream)),
                  "dlrm_gemm_f32")


def dlrm_tf32_split(rows: int, cols: int, src, lds: int, hi, lo, ldd: int, stream=None):
    """hi = src rounded to the nearest TF32 value, lo = src - hi (exact)."""
    return _check(lib().dlrm_tf32_split(int(rows), int(cols), _ptr(src), int(lds), _ptr(hi), _ptr(lo), int(ldd),
                                        _stream(stream)), "dlrm_tf32_split")


def dlrm_gemm_tf32x3_workspace_size(I: int, J: int, R: int) -> int:
    return int(lib().dlrm_gemm_tf32x3_workspace_size(int(I), int(J), int(R)))


def dlrm_gemm_tf32x3(I: int, J: int, R: int, A_hi, A_lo, lda: int, a_mn: bool, B_hi, B_lo, ldb: int, b_mn: bool, C,
                     ldc: int, ws, stream=None):
    """dlrm_gemm_f32 on operands already split by dlrm_tf32_split."""
    return _check(lib().dlrm_gemm_tf32x3(int(I), int(J), int(R), _ptr(A_hi), _ptr(A_lo), int(lda), int(bool(a_mn)),
                                         _ptr(B_hi), _ptr(B_lo), int(ldb), int(bool(b_mn)), _ptr(C), int(ldc),
                                         _ptr(ws), _nbytes(ws), _stream(stream)), "dlrm_gemm_tf32x3")


# ----------------------------------------------------------------- training step (fp32)

def dlrm_grads_size(T: Tables, bot: MLP, top: MLP, B: int, nnz: int) -> int:
    return int(lib().dlrm_grads_size(T.ref(), bot.ref(), top.ref(), int(B), int(nnz)))


def dlrm_grads_offsets(T: Tables, bot: MLP, top: MLP, B: int, nnz: int) -> dict:
    """Byte offsets of every gradient inside the gradient buffer."""
    nb, nt = len(bot.Ws), len(top.Ws)
    arrs = [(C.c_size_t * n)() for n in (nb, nb, nt, nt)]
    dE, loss = C.c_size_t(), C.c_size_t()
    _check(lib().dlrm_grads_offsets(T.ref(), bot.ref(), top.ref(), int(B), int(nnz), *arrs, C.byref(dE),
                                    C.byref(loss)), "dlrm_grads_offsets")
    return {"bot_dW": list(arrs[0]), "bot_db": list(arrs[1]), "top_dW": list(arrs[2]), "top_db": list(arrs[3]),
            "dE": dE.value, "loss": loss.value}


def dlrm_backward(T: Tables, bot: MLP, top: MLP, B: int, dense, offsets, indices, labels, grads, ws, loss=None,
                  y_hat=None, stream=None):
    return _check(lib().dlrm_backward(T.ref(), bot.ref(), top.ref(), int(B), _ptr(dense), _ptr(offsets),
                                      _ptr(indices), int(indices.numel()), _ptr(labels), _ptr(loss), _ptr(y_hat),
                                      _ptr(grads), _nbytes(grads), _ptr(ws), _nbytes(ws), _stream(stream)),
                  "dlrm_backward")


def dlrm_sparse_sgd(T: Tables, bot: MLP, top: MLP, B: int, nnz: int, lr: float, grads, n_touched=None, stream=None):
    return _check(lib().dlrm_sparse_sgd(T.ref(), bot.ref(), top.ref(), int(B), int(nnz), float(lr), _ptr(grads),
                                        _nbytes(grads), _ptr(n_touched), _stream(stream)), "dlrm_sparse_sgd")


def dlrm_embedding_row_grads(T: Tables, bot: MLP, top: MLP, B: int, nnz: int, grads, rows, row_grads, n_rows,
                             stream=None):
    return _check(lib().dlrm_embedding_row_grads(T.ref(), bot.ref(), top.ref(), int(B), int(nnz), _ptr(grads),
                                                 _nbytes(grads), _ptr(rows), _ptr(row_grads), _ptr(n_rows),
                                                 _stream(stream)),
                  "dlrm_embedding_row_grads")


# ----------------------------------------------------------------- table-wise model parallelism

def _parts_args(first_table, n_tables, ptrs):
    n = len(first_table)
    return (n, (C.c_int * n)(*[int(x) for x in first_table]), (C.c_int * n)(*[int(x) for x in n_tables]),
            (C.c_void_p * n)(*ptrs))


def dlrm_pooled_assemble(B: int, K: int, d: int, first_table, n_tables, parts, out, stream=None):
    """out[b][first_p + j] = parts[p][b][j] for every part p (fp32 device tensors)."""
    n, ft, nt, pp = _parts_args(first_table, n_tables, [_ptr(p) for p in parts])
    return _check(lib().dlrm_pooled_assemble(int(B), int(K), int(d), n, ft, nt, pp, _ptr(out), _stream(stream)),
                  "dlrm_pooled_assemble")


def dlrm_pooled_split(B: int, K: int, d: int, first_table, n_tables, inp, parts, stream=None):
    """parts[p][b][j] = inp[b][first_p + j] (the inverse of dlrm_pooled_assemble)."""
    n, ft, nt, pp = _parts_args(first_table, n_tables, [_ptr(p) for p in parts])
    return _check(lib().dlrm_pooled_split(int(B), int(K), int(d), n, ft, nt, _ptr(inp), pp, _stream(stream)),
                  "dlrm_pooled_split")


def dlrm_embbag_sgd_scratch_size(T: Tables, B: int, nnz: int) -> int:
    return int(lib().dlrm_embbag_sgd_scratch_size(T.ref(), int(B), int(nnz)))


def dlrm_embbag_sgd(T: Tables, B: int, offsets, indices, dE, lr: float, scratch, n_touched=None, stream=None):
    """T[r] -= lr * (sum of dE over the occurrences of row r), for the rows the bags touch."""
    return _check(lib().dlrm_embbag_sgd(T.ref(), int(B), _ptr(offsets), _ptr(indices), int(indices.numel()), _ptr(dE),
                                        float(lr), _ptr(scratch), _nbytes(scratch), _ptr(n_touched), _stream(stream)),
                  "dlrm_embbag_sgd")


def dlrm_backward_pooled_workspace_size(K: int, d: int, bot: MLP, top: MLP, B: int) -> int:
    return int(lib().dlrm_backward_pooled_workspace_size(int(K), int(d), bot.ref(), top.ref(), int(B)))


def dlrm_grads_pooled_size(K: int, d: int, bot: MLP, top: MLP, B: int) -> int:
    return int(lib().dlrm_grads_pooled_size(int(K), int(d), bot.ref(), top.ref(), int(B)))


def dlrm_grads_pooled_offsets(K: int, d: int, bot: MLP, top: MLP, B: int) -> dict:
    nb, nt = len(bot.Ws), len(top.Ws)
    arrs = [(C.c_size_t * n)() for n in (nb, nb, nt, nt)]
    dE, loss, end = C.c_size_t(), C.c_size_t(), C.c_size_t()
    _check(lib().dlrm_grads_pooled_offsets(int(K), int(d), bot.ref(), top.ref(), int(B), *arrs, C.byref(dE),
                                           C.byref(loss), C.byref(end)), "dlrm_grads_pooled_offsets")
    return {"bot_dW": list(arrs[0]), "bot_db": list(arrs[1]), "top_dW": list(arrs[2]), "top_db": list(arrs[3]),
            "dE": dE.value, "loss": loss.value, "dense_end": end.value}


def dlrm_backward_pooled(K: int, d: int, bot: MLP, top: MLP, B: int, dense, pooled, labels, grads, ws, loss=None,
                         y_hat=None, stream=None):
    return _check(lib().dlrm_backward_pooled(int(K), int(d), bot.ref(), top.ref(), int(B), _ptr(dense), _ptr(pooled),
                                             _ptr(labels), _ptr(loss), _ptr(y_hat), _ptr(grads), _nbytes(grads),
                                             _ptr(ws), _nbytes(ws), _stream(stream)), "dlrm_backward_pooled")


def dlrm_mlp_sgd(K: int, d: int, bot: MLP, top: MLP, B: int, lr: float, grads, stream=None):
    return _check(lib().dlrm_mlp_sgd(int(K), int(d), bot.ref(), top.ref(), int(B), float(lr), _ptr(grads),
                                     _nbytes(grads), _stream(stream)), "dlrm_mlp_sgd")


def grads_view(grads: torch.Tensor, off: int, shape) -> torch.Tensor:
    """fp32 view of part of a gradient buffer at a byte offset."""
    n = 1
    for x in shape:
        n *= int(x)
    return grads[off:off + 4 * n].view(torch.float32).view(*shape)
