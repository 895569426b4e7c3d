"""GPU parity of the W4A16 GEMM on the packed output (the step after the
search; "05 — AWQ: Activation-Aware Weight Scaling" §5 layout, weights
dequantised on the fly): Y = RN16(X Wd^T) with Wd = RN16((q - z) scale),
against the oracle's fp64 product of the same fp16 weights.  Bound per output:
half an fp16 ulp of the result plus 2^-11 sum_j |X_tj| |Wd_oj| for the fp32
accumulation of up to 4096 products (two roundings per addition at most)."""

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O
from synthetic import OutlierSpec, heavy_tailed_activations, random_layer, workload_inputs

from gpu_helpers import need_cuda, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


def _ulp16(v):
    a = np.abs(np.asarray(v, dtype=np.float64))
    return np.exp2(np.floor(np.log2(np.maximum(a, 2.0 ** -14))) - 10)


def _gpu_w4a16(X, qw, qz, sc, cfg, split_ws=False):
    """split_ws: a workspace of awq_w4a16_workspace_size() bytes (split-K for
    few tokens); otherwise the 256-byte minimum (never splits)."""
    Xd = to_dev(X)
    T, out = Xd.shape[0], sc.shape[1]
    Y = torch.empty((T, out), dtype=torch.float16, device="cuda")
    n = awq.awq_w4a16_workspace_size(T, Xd.shape[1], out, cfg) if split_ws else 256
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    awq.awq_w4a16_gemm(Xd, torch.from_numpy(qw).cuda(), torch.from_numpy(qz).cuda(),
                       torch.from_numpy(np.ascontiguousarray(sc)).cuda(), cfg, Y, ws)
    awq.awq_device_status(ws)
    torch.cuda.synchronize()
    return Y.cpu().numpy()


def _check(Yg, X, qw, qz, sc, group):
    Xn = np.asarray(X, dtype=np.float64)
    Yo = O.w4a16_matmul(X, qw, qz, sc, group)
    Wd = np.abs(O.dequant_packed(qw, qz, sc, group).astype(np.float64))
    acc = np.abs(Xn) @ Wd.T * 2.0 ** -11
    tol = 0.5 * _ulp16(np.abs(Yo) + acc) + acc
    err = np.abs(Yg.astype(np.float64) - Yo)
    assert np.all(err <= tol), (err.max(), np.unravel_index(np.argmax(err - tol), err.shape))


def test_w4a16_exact_integer_case():
    """Step 1, zero 8, integer X: every sum is an integer below 2^11, so the
    fp32 accumulation and the fp16 output are exact."""
    W = np.zeros((288, 256), dtype=np.float16)
    rng = np.random.default_rng(7)
    W[:] = rng.integers(-8, 8, size=W.shape)
    W[:, 0], W[:, 1], W[:, 128], W[:, 129] = -8.0, 7.0, -8.0, 7.0  # step 1, zero 8 in both groups
    qw, qz, sc = O.quant_pack(W, None, None, 4, 128)
    assert np.all(sc == np.float16(1.0))
    X = rng.integers(-2, 3, size=(300, 256)).astype(np.float16)
    Yg = _gpu_w4a16(torch.from_numpy(X), qw, qz, sc, awq.AwqConfig.make())
    want = X.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(Yg.astype(np.int64), want)


def _random_packed(inn, out, group, rng, pow2_scales):
    """qweight / qzeros / scales with random codes and zero points; scales
    2^e (e in -4..2) or random fp16 values in [2^-8, 4)."""
    q = rng.integers(0, 16, size=(out, inn)).astype(np.uint32)
    z = rng.integers(0, 16, size=(out, inn // group)).astype(np.uint32)
    qw = np.zeros((inn, out // 8), dtype=np.uint32)
    qz = np.zeros((inn // group, out // 8), dtype=np.uint32)
    for e in range(8):
        qw |= q[e::8, :].T << np.uint32(4 * e)
        qz |= z[e::8, :].T << np.uint32(4 * e)
    if pow2_scales:
        sc = np.exp2(rng.integers(-4, 3, size=(inn // group, out))).astype(np.float16)
    else:
        sc = np.exp2(rng.uniform(-8, 2, size=(inn // group, out))).astype(np.float16)
    return qw.view(np.int32), qz.view(np.int32), sc


@pytest.mark.parametrize("group", [128, 64, 32])
def test_w4a16_exact_pow2_scales(group):
    """Power-of-two scales, zero points across 0..15, integer X in [-3, 3]:
    every dequantised weight (q - z) 2^e is exact, every product and every
    fp32 partial sum is a multiple of 2^-4 below 2^20, so the fp32 sum is the
    exact sum and Y = RN16 of it, bit for bit."""
    rng = np.random.default_rng(group)
    inn, out, T = 512, 288, 333
    qw, qz, sc = _random_packed(inn, out, group, rng, pow2_scales=True)
    X = rng.integers(-3, 4, size=(T, inn)).astype(np.float16)
    Yg = _gpu_w4a16(torch.from_numpy(X), qw, qz, sc, awq.AwqConfig.make(group_size=group))
    want = O.w4a16_matmul(X, qw, qz, sc, group).astype(np.float16)
    assert np.array_equal(Yg.view(np.uint16), want.view(np.uint16))


@pytest.mark.parametrize("group", [128, 32])
def test_w4a16_dequantised_weights_bitwise(group):
    """Any fp16 scale: with one-hot rows of X (row t has a single 1 at input
    channel t), Y[t, o] is one dequantised weight, RN16((q - z) scale), so
    the on-the-fly conversion (subtract the zero, multiply by the scale, one
    fp16 rounding) is compared bit for bit with the oracle's dequant_packed."""
    rng = np.random.default_rng(100 + group)
    inn, out = 256, 160
    qw, qz, sc = _random_packed(inn, out, group, rng, pow2_scales=False)
    X = np.eye(inn, dtype=np.float16)
    Yg = _gpu_w4a16(torch.from_numpy(X), qw, qz, sc, awq.AwqConfig.make(group_size=group))
    Wd = O.dequant_packed(qw, qz, sc, group)  # [out, in] fp16
    assert np.array_equal(Yg.view(np.uint16), Wd.T.view(np.uint16))
    # the scales were not powers of two: the fp16 product did round somewhere
    exact = (O.unpack_nibbles(qw).astype(np.float64) -
             np.repeat(O.unpack_nibbles(qz).astype(np.float64), group, axis=1)) * \
        np.repeat(sc.astype(np.float64).T, group, axis=1)
    assert np.any(Wd.astype(np.float64) != exact)


@pytest.mark.parametrize("T,inn,out,w_bit,group,zp", [
    (200, 384, 288, 4, 128, 1), (1, 512, 160, 3, 64, 1), (300, 256, 96, 4, 32, 1),
    (2000, 1024, 768, 4, 128, 1), (129, 640, 544, 3, 128, 0)])
def test_w4a16_parity(T, inn, out, w_bit, group, zp):
    X, W = random_layer(T, inn, out, seed=T + inn + out + group)
    Wn = W.numpy()
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[9]
    qw, qz, sc = O.quant_pack(Wn, s, None, w_bit, group, zero_point=bool(zp))
    # the layer's input after the fold: X / s, as fp16
    Xs = (X.numpy().astype(np.float32) / s[None, :]).astype(np.float16)
    cfg = awq.AwqConfig.make(w_bit=w_bit, group_size=group, zero_point=zp)
    Yg = _gpu_w4a16(torch.from_numpy(Xs), qw, qz, sc, cfg)
    _check(Yg, Xs, qw, qz, sc, group)


def test_w4a16_on_the_searched_q_proj_layer():
    """The full q_proj workload: search, clip and pack on the GPU, then the
    W4A16 GEMM of X / s* (T = 65536, in = out = 4096) against the oracle on
    256 sampled tokens; and its output error against the fp16 X W^T stays
    the quantisation error the search measured."""
    d = workload_inputs(1)
    _, X, W = d["groups"][0]
    cfg = awq.AwqConfig.make(w_bit=4, n_alpha=20, n_clip=20)
    Xd, Wd = to_dev(X), to_dev(W)
    res = awq.quantize_layer(Xd, Wd, cfg)
    Xs = (Xd.float() / res.s_best[None, :]).half()  # the fold of 1/s* into the input
    Y = torch.empty((Xd.shape[0], Wd.shape[0]), dtype=torch.float16, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    awq.awq_w4a16_gemm(Xs, res.qweight, res.qzeros, res.scales, cfg, Y, ws)
    awq.awq_device_status(ws)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(1).choice(Xd.shape[0], 256, replace=False))
    qw, qz, sc = res.qweight.cpu().numpy(), res.qzeros.cpu().numpy(), res.scales.cpu().numpy()
    _check(Y[torch.from_numpy(rows).cuda()].cpu().numpy(), Xs[torch.from_numpy(rows).cuda()].cpu().numpy(),
           qw, qz, sc, 128)
    # the packed layer reproduces X W^T to the searched error level
    Yref = Xd[torch.from_numpy(rows).cuda()].float() @ Wd.float().T
    mse = float(((Y[torch.from_numpy(rows).cuda()].float() - Yref) ** 2).mean())
    assert mse < 1.5 * float(res.mse.min()) + 1e-6, (mse, float(res.mse.min()))


@pytest.mark.parametrize("T", [1, 16, 100, 300])
def test_w4a16_split_k_for_few_tokens(T):
    """Few tokens leave most SMs without an output tile: with the workspace
    awq_w4a16_workspace_size() asks for, K is split and the fp32 partial sums
    are added in a fixed order.  Exact sums stay exact (bit-equal to the
    unsplit GEMM and the oracle); a searched layer stays within the bound."""
    cfg = awq.AwqConfig.make()
    inn, out = 4096, 1024
    assert awq.awq_w4a16_workspace_size(T, inn, out, cfg) > 256  # this shape splits
    rng = np.random.default_rng(T)
    qw, qz, sc = _random_packed(inn, out, 128, rng, pow2_scales=True)
    X = rng.integers(-3, 4, size=(T, inn)).astype(np.float16)
    a = _gpu_w4a16(torch.from_numpy(X), qw, qz, sc, cfg, split_ws=True)
    b = _gpu_w4a16(torch.from_numpy(X), qw, qz, sc, cfg, split_ws=False)
    want = O.w4a16_matmul(X, qw, qz, sc, 128).astype(np.float16)
    assert np.array_equal(a.view(np.uint16), want.view(np.uint16))
    assert np.array_equal(b.view(np.uint16), want.view(np.uint16))
    Xr, W = random_layer(T, inn, out, seed=T + 5)
    s = O.scale_grid(O.act_stats(Xr.numpy()), O.alpha_grid(20))[9]
    qw, qz, sc = O.quant_pack(W.numpy(), s, None, 4, 128)
    Xs = (Xr.numpy().astype(np.float32) / s[None, :]).astype(np.float16)
    _check(_gpu_w4a16(torch.from_numpy(Xs), qw, qz, sc, cfg, split_ws=True), Xs, qw, qz, sc, 128)


@pytest.mark.parametrize("T,group", [(1024, 128), (3000, 32), (4096, 64)])
def test_w4a16_dequantise_once_for_many_tokens(T, group):
    """From 1024 tokens on, with the workspace awq_w4a16_workspace_size() asks
    for (the fp16 weights), the product dequantises the packed weights once,
    RN16((q - z) scale) as the fused kernel does per tile, and runs one fp16
    GEMM: exact sums stay bit-exact, and it agrees with the fused kernel."""
    cfg = awq.AwqConfig.make(group_size=group)
    inn, out = 1024, 800
    assert awq.awq_w4a16_workspace_size(T, inn, out, cfg) >= inn * out * 2
    rng = np.random.default_rng(T + group)
    qw, qz, sc = _random_packed(inn, out, group, rng, pow2_scales=True)
    X = rng.integers(-3, 4, size=(T, inn)).astype(np.float16)
    a = _gpu_w4a16(torch.from_numpy(X), qw, qz, sc, cfg, split_ws=True)
    want = O.w4a16_matmul(X, qw, qz, sc, group).astype(np.float16)
    assert np.array_equal(a.view(np.uint16), want.view(np.uint16))
    Xr, W = random_layer(T, inn, out, seed=T + group)
    s = O.scale_grid(O.act_stats(Xr.numpy()), O.alpha_grid(20))[9]
    qw, qz, sc = O.quant_pack(W.numpy(), s, None, 4, group)
    Xs = (Xr.numpy().astype(np.float32) / s[None, :]).astype(np.float16)
    a = _gpu_w4a16(torch.from_numpy(Xs), qw, qz, sc, cfg, split_ws=True)
    _check(a, Xs, qw, qz, sc, group)
    b = _gpu_w4a16(torch.from_numpy(Xs), qw, qz, sc, cfg, split_ws=False)  # the fused kernel
    _check(b, Xs, qw, qz, sc, group)



# ------------------------------------------------------------------ decode (T <= 8)
@pytest.mark.parametrize("T", [1, 2, 3, 5, 7, 8])
@pytest.mark.parametrize("inn,out,group", [(4096, 1024, 128), (512, 288, 32), (1024, 544, 64),
                                            (64, 32, 32), (320, 96, 64)])
def test_w4a16_decode_exact_sums(T, inn, out, group):
    """Up to 8 tokens the product streams the packed words on CUDA cores (per
    lane one word column, 8 input rows per batch, the warps' and the K
    splits' fp32 sums added in a fixed order).  Power-of-two scales and
    integer X keep every sum exact: Y is the oracle's RN16 of it, bit for
    bit, with the K split (the workspace awq_w4a16_workspace_size asks for)
    and without it (256 bytes: one block column over all of in).  out = 288
    and 544 leave a block with idle word columns."""
    cfg = awq.AwqConfig.make(group_size=group)
    rng = np.random.default_rng(T * 1000 + inn + out)
    qw, qz, sc = _random_packed(inn, out, group, rng, pow2_scales=True)
    X = rng.integers(-3, 4, size=(T, inn)).astype(np.float16)
    want = O.w4a16_matmul(X, qw, qz, sc, group).astype(np.float16)
    for split in (True, False):
        got = _gpu_w4a16(torch.from_numpy(X), qw, qz, sc, cfg, split_ws=split)
        assert np.array_equal(got.view(np.uint16), want.view(np.uint16)), split


@pytest.mark.parametrize("group", [128, 32])
def test_w4a16_decode_dequantised_weights_bitwise(group):
    """One-hot token rows pick single input channels (first, last, a group
    boundary, interior ones): Y[t, :] is the column RN16((q - z) scale) of
    the dequantised weights, bit for bit, for any fp16 scale."""
    rng = np.random.default_rng(300 + group)
    inn, out = 1024, 800
    qw, qz, sc = _random_packed(inn, out, group, rng, pow2_scales=False)
    cols = [0, inn - 1, group - 1, group, 517, 640, 3, 1000]
    X = np.zeros((len(cols), inn), dtype=np.float16)
    X[np.arange(len(cols)), cols] = 1.0
    Wd = O.dequant_packed(qw, qz, sc, group)
    for split in (True, False):
        Yg = _gpu_w4a16(torch.from_numpy(X), qw, qz, sc, awq.AwqConfig.make(group_size=group),
                        split_ws=split)
        assert np.array_equal(Yg.view(np.uint16), Wd[:, cols].T.view(np.uint16)), split


@pytest.mark.parametrize("T,w_bit,zp", [(1, 4, 1), (4, 3, 1), (8, 4, 0), (6, 4, 1)])
def test_w4a16_decode_searched_layer(T, w_bit, zp):
    """Packed weights of a searched 4096 x 1536 layer, decode-sized X (rows
    of the folded calibration input): within the accumulation bound."""
    inn, out = 4096, 1536
    Xr, W = random_layer(256, inn, out, seed=T + 17)
    s = O.scale_grid(O.act_stats(Xr.numpy()), O.alpha_grid(20))[11]
    qw, qz, sc = O.quant_pack(W.numpy(), s, None, w_bit, 128, zero_point=bool(zp))
    Xs = (Xr.numpy()[:T].astype(np.float32) / s[None, :]).astype(np.float16)
    cfg = awq.AwqConfig.make(w_bit=w_bit, zero_point=zp)
    for split in (True, False):
        _check(_gpu_w4a16(torch.from_numpy(Xs), qw, qz, sc, cfg, split_ws=split), Xs, qw, qz, sc, 128)


def test_w4a16_decode_strided_x_and_y():
    """X and Y rows with leading dimensions above in / out."""
    cfg = awq.AwqConfig.make()
    inn, out, T = 512, 288, 5
    rng = np.random.default_rng(9)
    qw, qz, sc = _random_packed(inn, out, 128, rng, pow2_scales=True)
    X = rng.integers(-3, 4, size=(T, inn)).astype(np.float16)
    Xbig = torch.zeros((T, inn + 64), dtype=torch.float16, device="cuda")
    Xbig[:, :inn] = torch.from_numpy(X).cuda()
    Ybig = torch.full((T, out + 32), 7.0, dtype=torch.float16, device="cuda")
    ws = torch.empty(awq.awq_w4a16_workspace_size(T, inn, out, cfg), dtype=torch.uint8, device="cuda")
    awq.awq_w4a16_gemm(Xbig[:, :inn], torch.from_numpy(qw).cuda(), torch.from_numpy(qz).cuda(),
                       torch.from_numpy(sc).cuda(), cfg, Ybig[:, :out], ws)
    awq.awq_device_status(ws)
    want = O.w4a16_matmul(X, qw, qz, sc, 128).astype(np.float16)
    Yn = Ybig.cpu().numpy()
    assert np.array_equal(Yn[:, :out].view(np.uint16), want.view(np.uint16))
    assert np.all(Yn[:, out:] == 7.0)  # nothing written past out
