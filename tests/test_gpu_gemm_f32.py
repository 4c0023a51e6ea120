"""fp32 GEMM on the tensor cores (dlrm_gemm_f32, 3xTF32) against fp64 numpy,
for the four operand orders (K-major / MN-major A and B), ragged edges in
every dimension, reductions shorter than one 32-deep stage and long ones cut
into fixed r-ranges.

The method's error per product is about 2^-20 |A(i,r) B(j,r)|, so the result
is held to the fp32 rule: |C - C64| <= 1e-5 (|C64| + sum_r |A(i,r) B(j,r)|).
Small-integer operands have exact products and sums: those must match exactly."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import assert_close, to_np

pytestmark = pytest.mark.gpu


def _run(A, a_mn, B, b_mn, I, J, R):
    lda, ldb = A.shape[1], B.shape[1]
    ldc = (J + 3) // 4 * 4
    C = torch.full((I, ldc), float("nan"), device="cuda")
    ws = E.alloc_workspace(E.dlrm_gemm_f32_workspace_size(I, J, R, a_mn, b_mn))
    E.dlrm_gemm_f32(I, J, R, A.cuda(), lda, a_mn, B.cuda(), ldb, b_mn, C, ldc, ws)
    assert E.dlrm_check_error(ws)[0] == 0
    return to_np(C)[:, :J]


def _operand(rows_i, R, mn, g, kind):
    # logical X(i, r); stored [i][r] (K-major) or [r][i] (MN-major) with a padded leading dimension
    if kind == "int":
        X = torch.randint(-8, 9, (rows_i, R), generator=g).float()
    else:
        X = torch.randn((rows_i, R), generator=g)
    S = X.t().contiguous() if mn else X
    cols = S.shape[1]
    ld = (cols + 3) // 4 * 4 + 4
    out = torch.zeros((S.shape[0], ld))
    out[:, :cols] = S
    return X.double().numpy(), out


SHAPES = [(256, 256, 32), (300, 200, 100), (65, 40, 7), (1000, 1024, 479), (128, 16, 4100), (5000, 300, 200),
          (257, 129, 1025), (16, 512, 20000), (1024, 1024, 65536)]


@pytest.mark.parametrize("I,J,R", SHAPES)
@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (False, True), (True, True), (True, False)])
def test_gemm_f32_random(I, J, R, a_mn, b_mn):
    g = torch.Generator().manual_seed(I * 31 + J * 7 + R + 3 * a_mn + b_mn)
    A64, A = _operand(I, R, a_mn, g, "randn")
    B64, B = _operand(J, R, b_mn, g, "randn")
    got = _run(A, a_mn, B, b_mn, I, J, R)
    want = A64 @ B64.T
    assert_close(got, want, "f32", f"gemm {I}x{J}x{R} a_mn={a_mn} b_mn={b_mn}", np.abs(A64) @ np.abs(B64).T)


@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (False, True), (True, True), (True, False)])
def test_gemm_f32_exact_on_small_integers(a_mn, b_mn):
    I, J, R = 300, 200, 777
    g = torch.Generator().manual_seed(5)
    A64, A = _operand(I, R, a_mn, g, "int")
    B64, B = _operand(J, R, b_mn, g, "int")
    got = _run(A, a_mn, B, b_mn, I, J, R)
    assert np.array_equal(got, A64 @ B64.T)


@pytest.mark.parametrize("R", [64, 1024, 65536])
def test_gemm_f32_long_same_sign_sums_do_not_drift(R):
    # all terms positive: an accumulator that rounds toward zero loses ~R/8 units in the last place
    # (1e-5 of the sum at R = 1024); fp32 with round-to-nearest stays near 1e-7
    I = J = 256
    g = torch.Generator().manual_seed(R + 1)
    A = torch.rand((I, R), generator=g)
    B = torch.rand((J, R), generator=g)
    got = _run(A, False, B, False, I, J, R)
    A64, B64 = A.double().numpy(), B.double().numpy()
    want = A64 @ B64.T
    rel = np.abs(got - want) / want
    assert rel.max() <= 1e-6, rel.max()


def test_gemm_f32_bit_reproducible():
    I, J, R = 512, 384, 30000   # long reduction: split into fixed r-ranges
    g = torch.Generator().manual_seed(9)
    _, A = _operand(I, R, True, g, "randn")
    _, B = _operand(J, R, True, g, "randn")
    a = _run(A, True, B, True, I, J, R)
    b = _run(A, True, B, True, I, J, R)
    assert np.array_equal(a, b)


def test_split_and_pair_gemm_match_the_one_call_gemm():
    I, J, R = 700, 300, 2000
    g = torch.Generator().manual_seed(11)
    _, A = _operand(I, R, False, g, "randn")
    _, B = _operand(J, R, True, g, "randn")
    want = _run(A, False, B, True, I, J, R)
    Ad, Bd = A.cuda(), B.cuda()
    Ah, Al = torch.empty_like(Ad), torch.empty_like(Ad)
    Bh, Bl = torch.empty_like(Bd), torch.empty_like(Bd)
    E.dlrm_tf32_split(Ad.shape[0], Ad.shape[1], Ad, Ad.shape[1], Ah, Al, Ad.shape[1])
    E.dlrm_tf32_split(Bd.shape[0], Bd.shape[1], Bd, Bd.shape[1], Bh, Bl, Bd.shape[1])
    # the split is exact and hi is a TF32 number (13 low mantissa bits clear)
    assert torch.equal(Ah + Al, Ad)
    assert int((Ah.view(torch.int32) & 0x1FFF).abs().max()) == 0
    assert float((Al.abs() - Ah.abs() * 2.0 ** -11).max()) <= 0   # |lo| <= half a TF32 unit of |hi|
    ldc = (J + 3) // 4 * 4
    C = torch.full((I, ldc), float("nan"), device="cuda")
    ws = E.alloc_workspace(E.dlrm_gemm_tf32x3_workspace_size(I, J, R))
    E.dlrm_gemm_tf32x3(I, J, R, Ah, Al, Ad.shape[1], False, Bh, Bl, Bd.shape[1], True, C, ldc, ws)
    assert E.dlrm_check_error(ws)[0] == 0
    assert np.array_equal(to_np(C)[:, :J], want)
