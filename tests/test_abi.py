"""The C-ABI library loads and exports every entry point its headers declare
(CPU only: no kernel is launched). Host-side argument checks run before any
CUDA call, so they are exercised here too."""
import ctypes as C
import glob
import os
import re
import subprocess

import pytest
import torch

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
    assert lib.dlrm_embbag_fwd(None, 4, None, None, 0, None, None, None, 0, None) == E.ERR_INVALID_ARG
    assert lib.dlrm_forward(None, None, None, 4, None, None, None, 0, None, None, 0, None) == E.ERR_INVALID_ARG
    assert lib.dlrm_interact_fwd(4, 0, 8, None, None, None, 64, 0, None) == E.ERR_INVALID_ARG
    assert lib.dlrm_interact_fwd(4, 300, 8, None, None, None, 10 ** 6, 0, None) == E.ERR_UNSUPPORTED
    assert lib.dlrm_check_error(None, 0, None, None) == E.ERR_INVALID_ARG
    assert lib.dlrm_check_error(256, 255, None, None) == E.ERR_WORKSPACE
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


def _kernel_bodies(src):
    """(name, body) of every __global__ function definition in a CUDA source."""
    out = []
    for m in re.finditer(r"__global__", src):
        head_end = src.index("{\n", m.end())
        name = re.findall(r"(\w+)\s*\(", src[m.end():head_end])
        depth, i = 0, head_end
        while True:
            depth += {"{": 1, "}": -1}.get(src[i], 0)
            i += 1
            if depth == 0:
                break
        out.append((name[-1] if name else "?", src[head_end:i]))
    return out


def test_every_kernel_is_a_programmatic_dependent_that_waits():
    """Every kernel is launched through launch_pdl (no <<<>>> launches), waits (pdl_wait) before it may
    touch global memory, and never lets its dependent start early (no griddepcontrol.launch_dependents)."""
    srcs = glob.glob(os.path.join(ROOT, "embedding_bags_dot_b200", "csrc", "*.cu"))
    n = 0
    for f in srcs:
        src = open(f).read()
        assert "<<<" not in src, f"{f}: a launch bypasses launch_pdl"
        assert "launch_dependents" not in src, f"{f}: a kernel triggers its dependent early"
        for name, body in _kernel_bodies(src):
            assert "pdl_wait();" in body, f"{os.path.basename(f)}: {name} never waits for the previous kernel"
            n += 1
    assert n >= 50


def _cpu_mlp(dims, dt):
    E = pytest.importorskip("embedding_bags_dot_b200")
    td = {"f32": torch.float32, "bf16": torch.bfloat16}[dt]
    Ws = [torch.zeros((dims[l + 1], E.dlrm_ld(dims[l], dt)), dtype=td) for l in range(len(dims) - 1)]
    bs = [torch.zeros(dims[l + 1]) for l in range(len(dims) - 1)]
    return E.MLP(Ws, bs, dims)


def test_mlp_workspace_size_follows_the_documented_layout(lib):
    """Error record (256 B), then one activation buffer per alternating hidden output (none for one layer,
    one for two, two otherwise) of the widest hidden output, then the input converted to a 16-bit MLP
    dtype when it comes in another dtype, then (fp32 MLPs) the 3xTF32 pair buffers; every piece rounded up
    to 256 bytes."""
    import embedding_bags_dot_b200 as E
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    B = 1000

    def f32tc(dims, B):
        """fp32 MLPs add their 3xTF32 pair buffers: split weights, split input, two hidden pair buffers."""
        ldf = lambda n: (n + 3) // 4 * 4  # noqa: E731
        w = sum(2 * a256(4 * dims[l + 1] * ldf(dims[l])) for l in range(len(dims) - 1))
        return w + 6 * a256(4 * B * ldf(max(dims)))
    assert E.dlrm_mlp_workspace_size(_cpu_mlp([13, 64], "f32"), B, "f32") == 256 + f32tc([13, 64], B)
    assert E.dlrm_mlp_workspace_size(_cpu_mlp([13, 64], "bf16"), B, "f32") == 256 + a256(16 * 2 * B)
    assert E.dlrm_mlp_workspace_size(_cpu_mlp([13, 512, 128], "bf16"), B, "f32") == 256 + a256(512 * 2 * B) + a256(16 * 2 * B)
    assert E.dlrm_mlp_workspace_size(_cpu_mlp([13, 512, 256, 128], "bf16"), B, "bf16") == 256 + 2 * a256(512 * 2 * B)
    assert E.dlrm_mlp_workspace_size(_cpu_mlp([479, 1024, 1024, 512, 256, 1], "bf16"), 77, "bf16") == \
        256 + 2 * a256(1024 * 2 * 77)
    assert E.dlrm_mlp_workspace_size(_cpu_mlp([13, 100, 3], "f32"), 5, "f32") == \
        256 + a256(100 * 4 * 5) + f32tc([13, 100, 3], 5)
    assert E.dlrm_mlp_workspace_size(_cpu_mlp([13, 64], "f32"), -1, "f32") == 0


def _fake_model(E, K=3, d=16, B=100, dt=None):
    """Host structs of a small fp32 model whose device pointers are fake (16-byte aligned, never
    dereferenced: every call below returns from its host-side checks)."""
    dt = E.F32 if dt is None else dt
    keep = {}
    keep["rows"] = (C.c_int64 * K)(*[10 * (k + 1) for k in range(K)])
    keep["T"] = E._abi.dlrm_tables(1 << 20, keep["rows"], K, d, dt)
    keep["db"] = (C.c_int * 3)(13, 32, d)
    keep["dt"] = (C.c_int * 3)(d + K * (K + 1) // 2, 8, 1)
    keep["W"] = (C.c_void_p * 2)(2 << 20, 3 << 20)
    keep["b"] = (C.c_void_p * 2)(4 << 20, 5 << 20)
    keep["bot"] = E._abi.dlrm_mlp(2, keep["db"], keep["W"], keep["b"], dt)
    keep["top"] = E._abi.dlrm_mlp(2, keep["dt"], keep["W"], keep["b"], dt)
    return keep


def test_c_abi_refuses_a_short_buffer_before_launching(lib):
    """Through the C ABI itself (no binding in between): every entry point that takes caller scratch
    memory refuses a buffer one byte shorter than its size query, with DLRM_ERR_WORKSPACE and no launch,
    and accepts the exact size as far as the host-side checks go."""
    import embedding_bags_dot_b200 as E
    m = _fake_model(E)
    T, bot, top = C.byref(m["T"]), C.byref(m["bot"]), C.byref(m["top"])
    B, nnz, fake = 100, 300, 6 << 20
    before = E.dlrm_launch_count()
    need = lib.dlrm_workspace_size(T, bot, top, B, 0)
    assert lib.dlrm_forward(T, bot, top, B, fake, fake, fake, nnz, fake, fake, need - 1, None) == E.ERR_WORKSPACE
    assert lib.dlrm_forward_cat(T, bot, top, B, fake, fake, fake, nnz, fake, fake, need - 1, None) == E.ERR_INVALID_ARG
    assert lib.dlrm_forward_lengths(T, bot, top, B, fake, fake, fake, nnz, fake, fake, need - 1, None) == E.ERR_WORKSPACE
    need_m = lib.dlrm_mlp_workspace_size(bot, B, E.F32)
    assert lib.dlrm_mlp_fwd(bot, B, fake, E.F32, 13, fake, 16, E.ACT_RELU, fake, need_m - 1, None) == E.ERR_WORKSPACE
    assert lib.dlrm_embbag_fwd(T, B, fake, fake, nnz, fake, None, fake, E.ERR_RECORD_BYTES - 1, None) == E.ERR_WORKSPACE
    assert lib.dlrm_embbag_interact_fwd(T, B, fake, fake, nnz, fake, fake, 24, E.F32, fake, E.ERR_RECORD_BYTES - 1,
                                        None) == E.ERR_WORKSPACE
    need_t = lib.dlrm_workspace_size(T, bot, top, B, 1)
    need_g = lib.dlrm_grads_size(T, bot, top, B, nnz)
    assert need_t > 0 and need_g > 0
    args = (T, bot, top, B, fake, fake, fake, nnz, fake, None, None)
    assert lib.dlrm_backward(*args, fake, need_g, fake, need_t - 1, None) == E.ERR_WORKSPACE
    assert lib.dlrm_backward(*args, fake, need_g - 1, fake, need_t, None) == E.ERR_WORKSPACE
    assert lib.dlrm_sparse_sgd(T, bot, top, B, nnz, 0.01, fake, need_g - 1, None, None) == E.ERR_WORKSPACE
    assert lib.dlrm_embedding_row_grads(T, bot, top, B, nnz, fake, need_g - 1, fake, fake, fake, None) == E.ERR_WORKSPACE
    for a_mn, b_mn in ((0, 0), (1, 1)):
        need_f = lib.dlrm_gemm_f32_workspace_size(64, 48, 40, a_mn, b_mn)
        assert lib.dlrm_gemm_f32(64, 48, 40, fake, 64, a_mn, fake, 48, b_mn, fake, 48, fake, need_f - 1, None) == \
            E.ERR_WORKSPACE
    need_x = lib.dlrm_gemm_tf32x3_workspace_size(64, 48, 40)
    assert lib.dlrm_gemm_tf32x3(64, 48, 40, fake, fake, 40, 0, fake, fake, 40, 0, fake, 48, fake, need_x - 1, None) == \
        E.ERR_WORKSPACE
    assert lib.dlrm_offsets_from_lengths(fake, 1000, fake, fake,
                                         lib.dlrm_offsets_from_lengths_workspace_size(1000) - 1, None) == E.ERR_WORKSPACE
    assert E.dlrm_launch_count() == before


def test_bindings_pass_the_buffer_size_through(lib):
    import embedding_bags_dot_b200 as E
    mlp = _cpu_mlp([13, 512, 256, 128], "bf16")
    B = 1000
    need = E.dlrm_mlp_workspace_size(mlp, B, torch.float32)
    x, out = torch.zeros((B, 13)), torch.zeros((B, 128))
    before = E.dlrm_launch_count()
    with pytest.raises(E.DlrmError) as e:
        E.dlrm_mlp_fwd(mlp, B, x, 13, out, 128, E.ACT_RELU, torch.zeros(need - 16, dtype=torch.uint8), stream=0)
    assert e.value.status == E.ERR_WORKSPACE
    assert E.dlrm_launch_count() == before


def test_bindings_refuse_a_mistyped_or_short_tensor(lib):
    """The C entry points take bare pointers; the binding refuses, before any launch, an MLP output that is
    not fp32 (the last layer always writes fp32) or too short, and a too-short input. A bf16 output buffer,
    half the bytes the layer writes, once made an experiment write past its end on the GPU."""
    import embedding_bags_dot_b200 as E
    mlp = _cpu_mlp([479, 1024], "bf16")
    B = 64
    ws = torch.zeros(E.dlrm_mlp_workspace_size(mlp, B, torch.bfloat16), dtype=torch.uint8)
    x = torch.zeros((B, 480), dtype=torch.bfloat16)
    before = E.dlrm_launch_count()
    for inp, out in [(x, torch.zeros((B, 1024), dtype=torch.bfloat16)),        # output not fp32
                     (x, torch.zeros((B - 1, 1024))),                          # output one row short
                     (x[: B - 1], torch.zeros((B, 1024)))]:                    # input one row short
        with pytest.raises(E.DlrmError) as e:
            E.dlrm_mlp_fwd(mlp, B, inp, 480, out, 1024, E.ACT_RELU, ws, stream=0)
        assert e.value.status == E.ERR_INVALID_ARG
    assert E.dlrm_launch_count() == before


def test_lengths_workspace_and_argument_checks(lib):
    """dlrm_offsets_from_lengths needs the error record plus one int per 8,192-length chunk (and one more);
    the bindings refuse lengths that are not uint8 and offsets that are not int32 or too short, before
    anything is launched."""
    import embedding_bags_dot_b200 as E
    for n, chunks in ((0, 0), (1, 1), (8192, 1), (8193, 2), (1_703_936, 208)):
        assert E.dlrm_offsets_from_lengths_workspace_size(n) == 256 + 4 * (chunks + 1)
    assert E.dlrm_offsets_from_lengths_workspace_size(-1) == 0
    before = E.dlrm_launch_count()
    ws = torch.zeros(4096, dtype=torch.uint8)
    for lens, offs in ((torch.zeros(10, dtype=torch.int32), torch.zeros(11, dtype=torch.int32)),
                       (torch.zeros(10, dtype=torch.uint8), torch.zeros(11, dtype=torch.int64)),
                       (torch.zeros(10, dtype=torch.uint8), torch.zeros(10, dtype=torch.int32))):
        with pytest.raises(E.DlrmError) as e:
            E.dlrm_offsets_from_lengths(lens, offs, ws, stream=0)
        assert e.value.status == E.ERR_INVALID_ARG
    with pytest.raises(E.DlrmError) as e:
        E.dlrm_offsets_from_lengths(torch.zeros(100_000, dtype=torch.uint8), torch.zeros(100_001, dtype=torch.int32),
                                    torch.zeros(64, dtype=torch.uint8), stream=0)
    assert e.value.status == E.ERR_WORKSPACE
    mlp = _cpu_mlp([13, 64], "f32")
    with pytest.raises(E.DlrmError) as e:
        E.dlrm_forward_lengths(None, mlp, mlp, 4, torch.zeros((4, 13)), torch.zeros(8, dtype=torch.int32),
                               torch.zeros(8, dtype=torch.int32), torch.zeros(4), ws, stream=0)
    assert e.value.status == E.ERR_INVALID_ARG
    assert E.dlrm_launch_count() == before
