"""Tensor-core (tcgen05) fully connected layer against the fp64 oracle, through
dlrm_mlp_fwd with one layer, on shapes that exercise a single tile, ragged
M / N / K edges, K below one 64-wide slice and many tiles per CTA.

bf16 x bf16 products are exact in fp32 and the accumulation is fp32, so with
an fp32 output the layer is held to the fp32 rule (rtol 1e-5 against the sum
of |terms|); a layout or descriptor mistake shows up as O(1) errors."""
import numpy as np
import pytest
import torch

import embedding_bags_dot_b200 as E
from gpucase import assert_close, scale_mlp, to_np
from oracle import oracle as O

pytestmark = pytest.mark.gpu

TD = {"bf16": torch.bfloat16, "f16": torch.float16}


def _layer(M, N, K, dt, seed):
    g = torch.Generator().manual_seed(seed)
    ld = E.dlrm_ld(K, dt)
    x = torch.zeros((M, ld), dtype=TD[dt])
    x[:, :K] = torch.randn((M, K), generator=g).to(TD[dt])
    W = torch.zeros((N, ld), dtype=TD[dt])
    W[:, :K] = (torch.randn((N, K), generator=g) / np.sqrt(K)).to(TD[dt])
    b = torch.randn(N, generator=g, dtype=torch.float32) * 0.1
    return x, W, b, ld


# M >= 4096 takes the SM-pair (cta_group::2, 256x256 tile) kernel, smaller M the single-SM one: 128 x 64
# tiles while 128 x 256 tiles would fill at most half the SMs (below 128 rows the A box holds only the
# batch's rows), 128 x 256 tiles otherwise ((3000, 1024, 479), (4000, 600, 100))
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (333, 200, 100), (1000, 1024, 479), (65, 40, 16),
                                   (4096, 512, 1024), (300, 768, 256), (129, 257, 65),
                                   (5000, 300, 200), (8192, 1024, 479), (4100, 40, 16), (70000, 256, 512),
                                   (5000, 512, 13), (100, 64, 5), (3000, 1024, 479), (4000, 600, 100),
                                   (2, 1000, 1024)])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_linear_tc_fp32_out(M, N, K, dt):
    x, W, b, ld = _layer(M, N, K, dt, seed=M * 7 + N + K)
    mlp = E.MLP([W.cuda()], [b.cuda()], [K, N])
    out = torch.full((M, N + 4 - N % 4 if N % 4 else N), float("nan"), device="cuda")
    ldo = out.shape[1]
    ws = E.alloc_workspace(E.dlrm_mlp_workspace_size(mlp, M, x.dtype))
    E.dlrm_mlp_fwd(mlp, M, x.cuda(), ld, out, ldo, E.ACT_NONE, ws)
    assert E.dlrm_check_error(ws)[0] == 0
    xs = x[:, :K].double().numpy()
    Ws = W[:, :K].double().numpy()
    want = O.mlp([Ws], [b.double().numpy()], xs, relu_last=False)
    assert_close(to_np(out)[:, :N], want, "f32", f"tc linear {M}x{N}x{K} {dt}", scale_mlp([Ws], [b.double().numpy()], xs))


@pytest.mark.parametrize("act", [E.ACT_RELU, E.ACT_SIGMOID])
def test_linear_tc_two_layers_bf16_hidden(act):
    # hidden layer output is stored in bf16 (tcgen05 epilogue with ReLU); final layer fp32 with act
    M, K, H, N = 777, 300, 512, 96
    x, W1, b1, ld = _layer(M, K, K, "bf16", seed=1)
    x = x[:, :ld]
    g = torch.Generator().manual_seed(2)
    W1 = torch.zeros((H, E.dlrm_ld(K, "bf16")), dtype=torch.bfloat16)
    W1[:, :K] = (torch.randn((H, K), generator=g) / np.sqrt(K)).bfloat16()
    b1 = torch.randn(H, generator=g) * 0.1
    W2 = (torch.randn((N, H), generator=g) / np.sqrt(H)).bfloat16()
    b2 = torch.randn(N, generator=g) * 0.1
    mlp = E.MLP([W1.cuda(), W2.cuda()], [b1.cuda(), b2.cuda()], [K, H, N])
    out = torch.empty((M, N), device="cuda")
    ws = E.alloc_workspace(E.dlrm_mlp_workspace_size(mlp, M, x.dtype))
    E.dlrm_mlp_fwd(mlp, M, x.cuda(), ld, out, N, act, ws)
    assert E.dlrm_check_error(ws)[0] == 0
    Ws = [W1[:, :K].double().numpy(), W2.double().numpy()]
    bs = [b1.double().numpy(), b2.double().numpy()]
    xs = x[:, :K].double().numpy()
    want = O.mlp(Ws, bs, xs, relu_last=(act == E.ACT_RELU))
    if act == E.ACT_SIGMOID:
        want = 1 / (1 + np.exp(-want))
    assert_close(to_np(out), want, "bf16", "two-layer bf16 MLP", scale_mlp(Ws, bs, xs, sigmoid=(act == E.ACT_SIGMOID)))


# serving-size batches (a handful of rows) through the same layer path: the A box holds the batch's rows
# rounded up to 8, and the 128-row MMA's rows past them never reach the output
@pytest.mark.parametrize("M,N,K", [(1, 256, 479), (5, 1024, 1024), (8, 40, 13), (16, 300, 200), (9, 64, 5),
                                   (32, 512, 1024), (33, 512, 1024), (31, 1000, 1100)])
@pytest.mark.parametrize("dt", ["bf16", "f16", "f32"])
def test_linear_small_batch(M, N, K, dt):
    if dt == "f32":
        g = torch.Generator().manual_seed(M * 3 + N)
        ld = E.dlrm_ld(K, "f32")
        x = torch.zeros((M, ld))
        x[:, :K] = torch.randn((M, K), generator=g)
        W = torch.zeros((N, ld))
        W[:, :K] = torch.randn((N, K), generator=g) / np.sqrt(K)
        b = torch.randn(N, generator=g) * 0.1
    else:
        x, W, b, ld = _layer(M, N, K, dt, seed=M * 11 + N)
    mlp = E.MLP([W.cuda()], [b.cuda()], [K, N])
    out = torch.full((M, N), float("nan"), device="cuda")
    ws = E.alloc_workspace(E.dlrm_mlp_workspace_size(mlp, M, x.dtype))
    E.dlrm_mlp_fwd(mlp, M, x.cuda(), ld, out, N, E.ACT_RELU, ws)
    assert E.dlrm_check_error(ws)[0] == 0
    xs, Ws, bs = x[:, :K].double().numpy(), W[:, :K].double().numpy(), b.double().numpy()
    want = O.mlp([Ws], [bs], xs, relu_last=True)
    assert_close(to_np(out), want, "f32", f"small-batch linear {M}x{N}x{K} {dt}", scale_mlp([Ws], [bs], xs))


# the bottom-MLP shape (13 dense features -> 512 -> 256 -> N3) through dlrm_mlp_fwd, many batch sizes
@pytest.mark.parametrize("B", [1, 127, 300, 1000, 20000])
@pytest.mark.parametrize("dt,n3", [("bf16", 128), ("f16", 64), ("bf16", 256), ("bf16", 64)])
def test_fused_bottom_mlp(B, dt, n3):
    g = torch.Generator().manual_seed(B + n3)
    dims = [13, 512, 256, n3]
    Ws, bs, Wd, bd = [], [], [], []
    for l in range(3):
        K, N = dims[l], dims[l + 1]
        W = torch.zeros((N, E.dlrm_ld(K, dt)), dtype=TD[dt])
        W[:, :K] = (torch.randn((N, K), generator=g) * np.sqrt(2.0 / K)).to(TD[dt])
        b = torch.randn(N, generator=g) * 0.1
        Ws.append(W[:, :K].double().numpy())
        bs.append(b.double().numpy())
        Wd.append(W.cuda())
        bd.append(b.cuda())
    x = torch.randn((B, 13), generator=g).abs()   # dense features: log1p-like, non-negative
    mlp = E.MLP(Wd, bd, dims)
    out = torch.full((B, n3), float("nan"), device="cuda")
    ws = E.alloc_workspace(E.dlrm_mlp_workspace_size(mlp, B, x.dtype))
    E.dlrm_mlp_fwd(mlp, B, x.cuda(), 13, out, n3, E.ACT_RELU, ws)
    assert E.dlrm_check_error(ws)[0] == 0
    want = O.mlp(Ws, bs, x.double().numpy(), relu_last=True)
    assert_close(to_np(out), want, "bf16", f"fused bottom MLP B={B} {dt} N3={n3}", scale_mlp(Ws, bs, x.double().numpy()))


# three bf16 layers from fp32 input run as one kernel (h1, h2 kept on chip) for widths that are multiples of 64
# up to 512 / 256 / 128 and up to 16 inputs: other widths, ragged batches, a K below 16
@pytest.mark.parametrize("dims", [(13, 192, 128, 64), (7, 64, 64, 128), (16, 512, 64, 64), (1, 448, 192, 128)])
@pytest.mark.parametrize("B", [1, 129, 256, 300, 4999])   # from 256 rows on, SM pairs share each weight k-block
def test_three_layer_mlp_one_kernel(dims, B):
    g = torch.Generator().manual_seed(B * 5 + dims[1])
    Ws, bs, Wd, bd = [], [], [], []
    for l in range(3):
        K, N = dims[l], dims[l + 1]
        W = torch.zeros((N, E.dlrm_ld(K, "bf16")), dtype=torch.bfloat16)
        W[:, :K] = (torch.randn((N, K), generator=g) * np.sqrt(2.0 / K)).bfloat16()
        if K % 8:
            W[:, K:] = float("nan")    # row padding is never read as a weight
        b = torch.randn(N, generator=g) * 0.1
        Ws.append(W[:, :K].double().numpy())
        bs.append(b.double().numpy())
        Wd.append(W.cuda())
        bd.append(b.cuda())
    x = torch.randn((B, dims[0]), generator=g)
    mlp = E.MLP(Wd, bd, list(dims))
    out = torch.full((B, dims[3]), float("nan"), device="cuda")
    ws = E.alloc_workspace(E.dlrm_mlp_workspace_size(mlp, B, x.dtype))
    n0 = E.dlrm_launch_count()
    E.dlrm_mlp_fwd(mlp, B, x.cuda(), dims[0], out, dims[3], E.ACT_RELU, ws)
    assert E.dlrm_launch_count() - n0 == 1, "three layers, one launch"
    assert E.dlrm_check_error(ws)[0] == 0
    xs = x.bfloat16().double().numpy()     # the input rounded to bf16, as every bf16 layer path does
    want = O.mlp(Ws, bs, xs, relu_last=True)
    assert_close(to_np(out), want, "bf16", f"one-kernel MLP {dims} B={B}", scale_mlp(Ws, bs, xs))


# at 4096+ rows the last hidden layer (width <= 256) and the one-column sigmoid output run as one kernel
@pytest.mark.parametrize("B,h,dt", [(4096, 256, "bf16"), (5000, 200, "bf16"), (4100, 256, "f16"), (3000, 256, "bf16")])
def test_last_hidden_layer_with_logit(B, h, dt):
    g = torch.Generator().manual_seed(B + h)
    dims = [479, 512, h, 1]
    Ws, bs, Wd, bd = [], [], [], []
    for l in range(3):
        K, N = dims[l], dims[l + 1]
        W = torch.zeros((N, E.dlrm_ld(K, dt)), dtype=TD[dt])
        W[:, :K] = (torch.randn((N, K), generator=g) * np.sqrt(2.0 / K)).to(TD[dt])
        b = torch.randn(N, generator=g) * 0.1
        Ws.append(W[:, :K].double().numpy())
        bs.append(b.double().numpy())
        Wd.append(W.cuda())
        bd.append(b.cuda())
    ld = E.dlrm_ld(479, dt)
    x = torch.zeros((B, ld), dtype=TD[dt])
    x[:, :479] = torch.randn((B, 479), generator=g).to(TD[dt])
    mlp = E.MLP(Wd, bd, dims)
    y = torch.full((B, 1), float("nan"), device="cuda")
    ws = E.alloc_workspace(E.dlrm_mlp_workspace_size(mlp, B, x.dtype))
    E.dlrm_mlp_fwd(mlp, B, x.cuda(), ld, y, 1, E.ACT_SIGMOID, ws)
    assert E.dlrm_check_error(ws)[0] == 0
    xs = x[:, :479].double().numpy()
    z = O.mlp(Ws, bs, xs, relu_last=False)
    want = 1 / (1 + np.exp(-z))
    assert_close(to_np(y), want, "bf16", f"last hidden layer + logit B={B} h={h} {dt}",
                 scale_mlp(Ws, bs, xs, sigmoid=True))
