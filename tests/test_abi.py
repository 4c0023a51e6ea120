"""The C-ABI library loads and exports every entry point its headers declare
(CPU only: no kernel is launched). Host-side argument checks run before any
CUDA call, so they are exercised here too."""
import ctypes as C
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(dlrm_\w+)\s*\(", src, flags=re.M):
            if not m.group(0).lstrip().startswith("typedef"):
                names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from embedding_bags_dot_b200 import _abi, build
    if not os.path.exists(_abi.LIB_PATH):
        build.build()
    return _abi.lib()


def test_headers_declare_the_boundary():
    names = _declared()
    for want in ("dlrm_embbag_fwd", "dlrm_interact_fwd", "dlrm_embbag_interact_fwd", "dlrm_mlp_fwd", "dlrm_forward",
                 "dlrm_check_error", "dlrm_workspace_size"):
        assert want in names, want


def test_every_declared_symbol_is_exported(lib):
    from embedding_bags_dot_b200 import _abi
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    missing = sorted(n for n in _declared() if n not in exported)
    assert not missing, f"declared but not exported: {missing}"
    for n in _declared():
        assert hasattr(lib, n)


def test_host_side_helpers(lib):
    import embedding_bags_dot_b200 as E
    assert E.dlrm_ld(479, "bf16") == 480 and E.dlrm_ld(479, "f32") == 480 and E.dlrm_ld(13, "f32") == 16
    assert E.dlrm_ld(16, "bf16") == 16 and E.dlrm_ld(1, "bf16") == 8
    assert lib.dlrm_status_str(0) == b"ok"
    assert b"out of range" in lib.dlrm_status_str(3)


def test_argument_checks_without_gpu(lib):
    import embedding_bags_dot_b200 as E
    # null tables / null everything: rejected before any CUDA call
    assert lib.dlrm_embbag_fwd(None, 4, None, None, 0, None, None, None, None) == E.ERR_INVALID_ARG
    assert lib.dlrm_forward(None, None, None, 4, None, None, None, 0, None, None, None) == E.ERR_INVALID_ARG
    assert lib.dlrm_interact_fwd(4, 0, 8, None, None, None, 64, 0, None) == E.ERR_INVALID_ARG
    assert lib.dlrm_interact_fwd(4, 300, 8, None, None, None, 10 ** 6, 0, None) == E.ERR_UNSUPPORTED
    assert lib.dlrm_check_error(None, None, None) == E.ERR_INVALID_ARG
    # workspace size from host structs only (fake, never dereferenced, device pointers)
    rows = (C.c_int64 * 3)(10, 20, 30)
    T = E._abi.dlrm_tables(256, rows, 3, 16, E.F32)
    dims_b = (C.c_int * 3)(13, 32, 16)
    dims_t = (C.c_int * 3)(16 + 6, 8, 1)
    W = (C.c_void_p * 2)(256, 512)
    b = (C.c_void_p * 2)(768, 1024)
    bot = E._abi.dlrm_mlp(2, dims_b, W, b, E.F32)
    top = E._abi.dlrm_mlp(2, dims_t, W, b, E.F32)
    n = lib.dlrm_workspace_size(C.byref(T), C.byref(bot), C.byref(top), 100, 0)
    # error record + x_dense (100*16*4) + concat (100*24*4) + 2 hidden buffers (100*32*4)
    assert n >= 256 + 6400 + 9600 + 2 * 12800
    assert lib.dlrm_workspace_size(None, C.byref(bot), C.byref(top), 100, 0) == 0


def test_product_path_has_no_cpu_fallback():
    """The binding must not import the oracle, and must raise when the library is missing."""
    src = open(os.path.join(ROOT, "embedding_bags_dot_b200", "_abi.py")).read()
    assert "oracle" not in src.replace("never", "")
    for f in glob.glob(os.path.join(ROOT, "embedding_bags_dot_b200", "**", "*.*"), recursive=True):
        if f.endswith((".py", ".cu", ".cuh")):
            assert "import oracle" not in open(f).read() and "from oracle" not in open(f).read(), f
