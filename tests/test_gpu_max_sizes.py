"""The largest token count the calls accept, T = 2^22 (the bound the exact
activation sum sets: 2^22 tokens x 65504 x 2^24 units < 2^63), on a narrow
layer so that the oracle still finishes in seconds: the activation statistic
at its largest possible sums, the whole path (statistic, alpha search, clip
search, packing) against the oracle, and the W4A16 product in both
tensor-core forms; and a weight matrix of more than 2^31 elements.  The host
check past the token bound is in test_abi.py."""

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O
from synthetic import OutlierSpec, heavy_tailed_activations, random_layer

from gpu_helpers import check_selection, layer_parity, need_cuda, to_dev

pytestmark = pytest.mark.gpu

T_MAX = 1 << 22


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


def test_act_stats_at_the_largest_exact_sum():
    """Column 0 holds +65504 in every token and column 1 -65504 (the largest
    sums of magnitudes the int64 accumulator must hold, 2^22 x 65504 x 2^24
    units), column 2 the smallest subnormal 2^-24 (one unit per token); the
    other columns are heavy-tailed.  abar is bit-exact against the oracle."""
    inn = 64
    X = heavy_tailed_activations(T_MAX, inn, OutlierSpec(0.05, 20.0, 50.0), seed=22)
    X[:, 0] = 65504.0
    X[:, 1] = -65504.0
    X[:, 2] = 2.0 ** -24
    abar = torch.empty(inn, dtype=torch.float64, device="cuda")
    awq.awq_act_stats(to_dev(X), abar)
    torch.cuda.synchronize()
    got = abar.cpu().numpy()
    assert np.array_equal(got, O.act_stats(X.numpy()))
    assert got[0] == 65504.0 and got[1] == 65504.0 and got[2] == 2.0 ** -24


def test_whole_path_at_the_maximum_token_count():
    """X [2^22 x 128], W [64 x 128], INT4 g128, 20 alphas and 20 clip ratios:
    abar and s bit-exact, per-alpha MSE within 1e-3, the same alpha and clip
    choices unless tied within 1e-4, the packed output bit-exact."""
    X, W = random_layer(T_MAX, 128, 64, seed=4242)
    layer_parity(X, W, 4, 20, 20)


@pytest.mark.parametrize("form", ["dequantise_once", "fused"])
def test_w4a16_at_the_maximum_token_count(form):
    """Y = RN16(X Wd^T) for 2^22 tokens (in = 128, out = 64, g128): the
    weights dequantised once into the workspace and one fp16 GEMM, or
    dequantised tile by tile inside the GEMM (256-byte workspace).  Sampled
    rows across all of T (and the last 300) within half an fp16 ulp of the
    result plus 2^-11 sum_j |x_j| |w_j| of the oracle's fp64 product."""
    X, W = random_layer(T_MAX, 128, 64, seed=4343)
    qw, qz, sc = O.quant_pack(W.numpy(), None, None, 4, 128)
    cfg = awq.AwqConfig.make()
    Xd = to_dev(X)
    Y = torch.empty((T_MAX, 64), dtype=torch.float16, device="cuda")
    n = awq.awq_w4a16_workspace_size(T_MAX, 128, 64, cfg) if form == "dequantise_once" else 256
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    awq.awq_w4a16_gemm(Xd, torch.from_numpy(qw).cuda(), torch.from_numpy(qz).cuda(),
                       torch.from_numpy(np.ascontiguousarray(sc)).cuda(), cfg, Y, ws)
    awq.awq_device_status(ws)
    torch.cuda.synchronize()
    rows = np.r_[np.arange(0, T_MAX, 997), np.arange(T_MAX - 300, T_MAX)]
    Yg = Y.cpu().numpy()[rows].astype(np.float64)
    Xs = X.numpy()[rows]
    Yo = O.w4a16_matmul(Xs, qw, qz, sc, 128)
    Wd = np.abs(O.dequant_packed(qw, qz, sc, 128).astype(np.float64))
    acc = np.abs(Xs.astype(np.float64)) @ Wd.T * 2.0 ** -11
    a = np.abs(Yo) + acc
    ulp = np.exp2(np.floor(np.log2(np.maximum(a, 2.0 ** -14))) - 10)
    err = np.abs(Yg - Yo)
    assert np.all(err <= 0.5 * ulp + acc), err.max()


def test_weight_matrix_past_2_31_elements():
    """W [2^20 + 64, 2048] holds 2^31 + 131072 weights, so row and element
    offsets past 2^31 must be 64-bit in every kernel that walks W or the
    candidate operand (candidates, scored GEMM, clip search, packing).
    n_alpha = 1 (alpha = 0: s = 1, plain quantisation) keeps the check per
    row: the clip indices and the packed output are compared with the oracle
    on 8-row blocks at both ends of W and on both sides of element 2^31."""
    T, inn, out = 64, 2048, (1 << 20) + 64
    X = heavy_tailed_activations(T, inn, OutlierSpec(0.01, 20.0, 50.0), seed=31)
    gen = torch.Generator(device="cuda").manual_seed(31)
    Wd = (0.02 * torch.randn((out, inn), generator=gen, device="cuda")).half()
    cfg = awq.AwqConfig.make(n_alpha=1, n_clip=20)
    ws = awq.alloc_workspace(T, inn, out, cfg)
    res = awq.quantize_layer(to_dev(X), Wd, cfg, ws=ws)
    awq.awq_device_status(ws)
    torch.cuda.synchronize()
    Xn = X.numpy()
    assert np.array_equal(res.abar.cpu().numpy(), O.act_stats(Xn))
    assert int(res.best_idx.item()) == 0 and bool(torch.all(res.s_best == 1.0))
    ones = np.ones(inn, dtype=np.float32)
    Gk = O.block_grams(Xn, 128)
    rng = np.random.default_rng(31)
    blocks = [0, (1 << 20) - 8, 1 << 20, out - 8] + [8 * int(b) for b in rng.integers(0, out // 8, 4)]
    for o0 in blocks:
        Wn = Wd[o0:o0 + 8].cpu().numpy()
        idx_o, E = O.search_clip(Xn, Wn, ones, 4, 128, 20, 0.5, Gk=Gk)
        idx_g = res.clip_idx[o0:o0 + 8].cpu().numpy()
        for o, k in zip(*np.nonzero(idx_g != idx_o)):
            check_selection(int(idx_g[o, k]), E[o, k], f"clip row {o0 + o} group {k}")
        qw, qz, sc = O.quant_pack(Wn, ones, idx_g, 4, 128, 20, 0.5)
        w = o0 // 8
        assert np.array_equal(res.qweight[:, w:w + 1].cpu().numpy(), qw), o0
        assert np.array_equal(res.qzeros[:, w:w + 1].cpu().numpy(), qz), o0
        assert np.array_equal(res.scales[:, o0:o0 + 8].cpu().numpy().view(np.uint16), sc.view(np.uint16)), o0
