"""GPU parity: every step of the CUDA path, called through the C ABI, against
the fp64 CPU oracle on the same seeded inputs.

Bars: abar, the s grid, codes, zeros, qweight, qzeros and scales bit-exact;
per-alpha MSE within 1e-3 relative; the selected alpha / clip index equal to
the oracle's unless the oracle's scores of the two differ by < 1e-4 relative;
clip errors within 1e-3 relative."""

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O
from synthetic import OutlierSpec, heavy_tailed_activations, random_layer, workload_inputs

from gpu_helpers import (MSE_RTOL, check_mse, check_selection, gpu_search, layer_parity,
                         midpoint_report, need_cuda, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


# ------------------------------------------------------------------ K1
@pytest.mark.parametrize("T,inn,ldx", [(1, 8, 8), (37, 136, 136), (1000, 520, 520), (4096 + 77, 1024, 1032),
                                       (20000, 256, 256)])
def test_act_stats_bitwise(T, inn, ldx):
    X = heavy_tailed_activations(T, ldx, OutlierSpec(0.02, 20.0, 50.0), seed=T + inn)
    X[0, :4] = torch.tensor([65504.0, -65504.0, 2 ** -24, -(2 ** -24)], dtype=torch.float16)
    Xd = to_dev(X)[:, :inn]
    abar = torch.empty(inn, dtype=torch.float64, device="cuda")
    awq.awq_act_stats(Xd, abar)
    want = O.act_stats(X[:, :inn].numpy())
    got = abar.cpu().numpy()
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:10]


# ------------------------------------------------------------------ K2
@pytest.mark.parametrize("n_alpha", [1, 3, 20])
def test_scale_grid_bitwise(n_alpha):
    rng = np.random.default_rng(n_alpha)
    abar = np.exp(rng.normal(0, 2, 4096))
    abar[:4] = [0.0, 1e-9, 1.0, 300.0]
    a_d = torch.from_numpy(abar).cuda()
    s = torch.empty((n_alpha, 4096), dtype=torch.float32, device="cuda")
    awq.awq_scale_grid(a_d, n_alpha, s)
    got = s.cpu().numpy()
    want = O.scale_grid(abar, O.alpha_grid(n_alpha))
    assert np.array_equal(got, want), midpoint_report(abar, O.alpha_grid(n_alpha), got, want)


# ------------------------------------------------------------------ K7
def _gpu_pack(W, s, clip_idx, cfg):
    out, inn = W.shape
    g = cfg.group_size
    qw = torch.empty((inn, out // 8), dtype=torch.int32, device="cuda")
    qz = torch.empty((inn // g, out // 8), dtype=torch.int32, device="cuda")
    sc = torch.empty((inn // g, out), dtype=torch.float16, device="cuda")
    awq.awq_quant_pack(to_dev(W), None if s is None else torch.from_numpy(s).cuda(),
                       None if clip_idx is None else torch.from_numpy(clip_idx).cuda(),
                       cfg, qw, qz, sc)
    torch.cuda.synchronize()
    return qw.cpu().numpy(), qz.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("out,inn,w_bit,use_s,use_clip", [
    (8, 128, 4, False, False), (72, 384, 4, True, False), (136, 256, 3, True, True),
    (512, 512, 4, True, True), (1000, 1024, 3, False, True)])
def test_quant_pack_bitwise(out, inn, w_bit, use_s, use_clip):
    X, W = random_layer(64, inn, out, seed=out + inn + w_bit)
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[13] if use_s else None
    n_clip = 20 if use_clip else 0
    clip_idx = (np.random.default_rng(out).integers(0, 20, size=(out, inn // 128)).astype(np.uint8)
                if use_clip else None)
    cfg = awq.AwqConfig.make(w_bit=w_bit, n_clip=n_clip)
    got = _gpu_pack(W, s, clip_idx, cfg)
    want = O.quant_pack(W.numpy(), s, clip_idx, w_bit, 128, max(n_clip, 1), 0.5)
    for g_, w_, name in zip(got, want, ("qweight", "qzeros", "scales")):
        assert np.array_equal(g_.view(np.uint8), w_.view(np.uint8)), name


def test_quant_pack_hand_worked(golden):
    hdr, rows = golden("pack_int4.txt")
    W = np.zeros((8, 128), dtype=np.float16)
    for o in range(8):
        for j in range(8):
            W[o, j] = ((o + j) % 16) - 8
        W[o, 126], W[o, 127] = -8.0, 7.0
    qw, qz, sc = _gpu_pack(torch.from_numpy(W), None, None, awq.AwqConfig.make())
    for r in rows:
        assert int(qw.view(np.uint32)[int(r[0]), 0]) == int(r[1], 16)
    assert int(qz.view(np.uint32)[0, 0]) == int(hdr["qzeros_hex"], 16)
    assert np.all(sc == np.float16(1.0))


# ------------------------------------------------------------------ K2-K5
SEARCH_CASES = [
    # T, in, out, w_bit, n_alpha
    (64, 128, 16, 4, 20),
    (1, 128, 8, 4, 20),
    (200, 384, 264, 3, 20),
    (256, 512, 512, 4, 20),      # the tiny 512 x 512 linear workload's shapes
    (2125, 1024, 768, 4, 20),    # > 1000 GEMM tiles: persistent schedule, both accumulators
    (130, 256, 64, 4, 1),        # alpha = 0 only: plain RTN
]


@pytest.mark.parametrize("T,inn,out,w_bit,n_alpha", SEARCH_CASES)
def test_search_scale_parity(T, inn, out, w_bit, n_alpha):
    X, W = random_layer(T, inn, out, seed=T * 7 + inn + out)
    cfg = awq.AwqConfig.make(w_bit=w_bit, n_alpha=n_alpha)
    g = gpu_search(X, W, cfg)
    Xn, Wn = X.numpy(), W.numpy()
    abar = O.act_stats(Xn)
    assert np.array_equal(g["abar"], abar)
    mse, best, s_best, S = O.search_scale(Xn, Wn, abar, w_bit, 128, n_alpha)
    check_mse(g["mse"], mse)
    check_selection(g["best"], mse, "alpha")
    assert np.array_equal(g["s_best"], S[g["best"]])


def test_search_scale_strided_x_and_determinism():
    X, W = random_layer(700, 640, 256, seed=5)
    Xd = to_dev(X)
    wide = torch.zeros((700, 768), dtype=torch.float16, device="cuda")
    wide[:, 64:704] = Xd
    Xv = wide[:, 64:704]                    # row stride 768, 128-byte aligned start
    cfg = awq.AwqConfig.make()
    ws = awq.alloc_workspace(700, 640, 256, cfg)
    outs = []
    for _ in range(2):
        abar = torch.empty(640, dtype=torch.float64, device="cuda")
        mse = torch.empty(20, dtype=torch.float64, device="cuda")
        best = torch.empty(1, dtype=torch.int32, device="cuda")
        s_best = torch.empty(640, dtype=torch.float32, device="cuda")
        awq.awq_act_stats(Xv, abar)
        awq.awq_search_scale(Xv, to_dev(W), abar, cfg, ws, s_best, mse, best)
        awq.awq_device_status(ws)
        outs.append(mse.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])  # fixed-order reductions: bitwise reproducible
    mse_o, _, _, _ = O.search_scale(X.numpy(), W.numpy(), O.act_stats(X.numpy()), 4, 128, 20)
    check_mse(outs[0], mse_o)


def test_ties_keep_alpha_zero():
    T, inn = 64, 256
    X = torch.from_numpy(np.where(np.arange(T * inn).reshape(T, inn) % 2 == 0, 1.0, -1.0)
                         .astype(np.float16))
    _, W = random_layer(4, inn, 16, seed=3)
    g = gpu_search(X, W, awq.AwqConfig.make())
    assert np.all(g["mse"] == g["mse"][0]) and g["best"] == 0 and np.all(g["s_best"] == 1.0)


# ------------------------------------------------------------------ K6
def _gpu_clip(X, W, s, cfg, with_err=True):
    Xd, Wd = to_dev(X), to_dev(W)
    T, inn = Xd.shape
    out = Wd.shape[0]
    g = cfg.group_size
    ws = awq.alloc_workspace(T, inn, out, cfg)
    idx = torch.empty((out, inn // g), dtype=torch.uint8, device="cuda")
    err = torch.empty((out, inn // g, cfg.n_clip), dtype=torch.float32, device="cuda") if with_err else None
    awq.awq_search_clip(Xd, Wd, None if s is None else torch.from_numpy(s).cuda(), cfg, ws, idx, err)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), (err.cpu().numpy() if with_err else None)


@pytest.mark.parametrize("T,inn,out,w_bit,n_clip,group", [
    (300, 256, 40, 4, 20, 128), (64, 128, 8, 3, 7, 128), (1500, 512, 96, 3, 20, 128),
    (33, 384, 24, 4, 1, 128), (300, 256, 40, 4, 20, 32), (1500, 512, 96, 3, 20, 64),
    (700, 384, 136, 4, 7, 32), (64, 128, 8, 4, 20, 64)])
def test_search_clip_parity(T, inn, out, w_bit, n_clip, group):
    """The clip search at groups of 128 (the pages' g) and of 64 and 32 ("AWQ
    and Activation-Aware Scaling", When it breaks, contrasts g = 32)."""
    X, W = random_layer(T, inn, out, seed=T + out + n_clip + group)
    Xn, Wn = X.numpy(), W.numpy()
    s = O.scale_grid(O.act_stats(Xn), O.alpha_grid(20))[10]
    cfg = awq.AwqConfig.make(w_bit=w_bit, n_clip=n_clip, group_size=group)
    idx, err = _gpu_clip(X, W, s, cfg)
    idx_o, E = O.search_clip(Xn, Wn, s, w_bit, group, n_clip, 0.5)
    rel = np.abs(err - E) / np.maximum(np.abs(E), 1e-30)
    assert rel.max() <= MSE_RTOL, rel.max()
    for o, k in zip(*np.nonzero(idx != idx_o)):
        check_selection(int(idx[o, k]), E[o, k], f"clip row {o} group {k}")
    # s = None means s = 1
    idx1, _ = _gpu_clip(X, W, None, cfg, with_err=False)
    idx1_o, E1 = O.search_clip(Xn, Wn, None, w_bit, group, n_clip, 0.5)
    for o, k in zip(*np.nonzero(idx1 != idx1_o)):
        check_selection(int(idx1[o, k]), E1[o, k], f"clip row {o} group {k}")


@pytest.mark.parametrize("name", ["quant_group_clip.txt", "quant_group_clip_interior.txt"])
def test_clip_hand_worked(golden, name):
    """The hand-worked clip examples (ratio index 19, and the interior index 8
    whose codes are all round-half-even ties), through the pack kernel."""
    hdr, rows = golden(name)
    W = np.zeros((8, 128), dtype=np.float16)
    for r in rows:
        W[:, int(r[0])] = float(r[1])
    idx = np.full((8, 1), int(hdr["clip_index"]), dtype=np.uint8)
    qw, qz, sc = _gpu_pack(torch.from_numpy(W), None, idx, awq.AwqConfig.make(n_clip=int(hdr["n_clip"])))
    q = O.unpack_nibbles(qw)
    assert np.all(sc == np.float16(float(hdr["delta"])))
    assert np.all(O.unpack_nibbles(qz) == int(hdr["zero"]))
    for r in rows:
        assert np.all(q[:, int(r[0])] == int(r[2]))


# ------------------------------------------------------------------ full sizes
def test_full_q_proj_4096_workload():
    """The Llama-7B-shaped q_proj workload at full size: X [65536 x 4096],
    W [4096 x 4096], INT4 g128, 20 alphas, 20 clip ratios, packed."""
    d = workload_inputs(1)
    _, X, W = d["groups"][0]
    layer_parity(X, W, 4, 20, 20)


# ------------------------------------------------------------------ K8
@pytest.mark.parametrize("rows,cols", [(4096, 1), (5120, 1), (4096, 4096), (136, 24)])
def test_fold_inv_scale_bitwise(rows, cols):
    """Folding 1/s into the preceding norm's gamma (cols = 1) or the preceding
    linear's rows: RN16(RN32(v) / s), bit-exact."""
    rng = np.random.default_rng(rows + cols)
    v = rng.normal(0, 0.05 if cols > 1 else 1.0, (rows, cols)).astype(np.float16)
    s = O.scale_grid(np.exp(rng.normal(0, 1.5, rows)), O.alpha_grid(20))[13]
    vd = torch.from_numpy(v).cuda()
    awq.awq_fold_inv_scale(vd, torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    want = O.fold_inv_scale(v[:, 0] if cols == 1 else v, s)
    got = vd.cpu().numpy()
    got = got[:, 0] if cols == 1 else got
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_fold_rounding_chain_hand_worked(golden):
    """The fixture where RN16(RN32(v)/s) lands on an fp16 tie (two roundings)
    and the single rounding or the reciprocal product would give the other
    neighbour: the fold kernel gives the fixture's bits."""
    hdr, _ = golden("fold_rounding.txt")
    v = np.full((8, 4), int(hdr["v_hex"], 16), dtype=np.uint16).view(np.float16)
    s = np.full(8, int(hdr["s_hex"], 16), dtype=np.uint32).view(np.float32)
    vd = torch.from_numpy(v).cuda()
    awq.awq_fold_inv_scale(vd, torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    assert np.all(vd.cpu().numpy().view(np.uint16) == int(hdr["folded_hex"], 16))


# ------------------------------------------------------------------ Gram form
@pytest.mark.parametrize("T,inn,out,w_bit", [(64, 128, 16, 4), (200, 384, 264, 3), (256, 512, 512, 4),
                                             (2125, 1024, 768, 4)])
def test_search_scale_gram_form_parity(T, inn, out, w_bit):
    """The Gram-form search (sum_o dW_o^T X^T X dW_o, normalised G in fp16
    hi + lo) against the oracle's MSE curve and selection."""
    X, W = random_layer(T, inn, out, seed=T * 7 + inn + out)
    cfg = awq.AwqConfig.make(w_bit=w_bit, search_form=awq.abi.SEARCH_GRAM)
    g = gpu_search(X, W, cfg)
    Xn, Wn = X.numpy(), W.numpy()
    mse, _, _, S = O.search_scale(Xn, Wn, O.act_stats(Xn), w_bit, 128, 20)
    check_mse(g["mse"], mse)
    check_selection(g["best"], mse, "alpha (Gram form)")
    assert np.array_equal(g["s_best"], S[g["best"]])


def test_gram_form_matches_direct_form_full_q_proj():
    """Both scoring forms on the full q_proj workload agree within the MSE bar
    and pick the same alpha (unless tied within 1e-4)."""
    d = workload_inputs(1)
    _, X, W = d["groups"][0]
    a = gpu_search(X, W, awq.AwqConfig.make())
    b = gpu_search(X, W, awq.AwqConfig.make(search_form=awq.abi.SEARCH_GRAM))
    rel = np.abs(a["mse"] - b["mse"]) / a["mse"]
    assert rel.max() <= MSE_RTOL, rel.max()
    check_selection(b["best"], a["mse"], "alpha (Gram vs direct)")


# ------------------------------------------------------------------ group sizes 32 / 64
@pytest.mark.parametrize("T,inn,out,w_bit,group,form", [
    (300, 256, 72, 4, 32, 0), (1200, 640, 264, 3, 64, 0), (500, 384, 136, 4, 32, 1), (257, 512, 512, 4, 64, 1),
    (300, 64, 72, 4, 32, 0), (1, 64, 8, 4, 32, 0), (90, 192, 264, 3, 64, 0)])
def test_search_scale_other_group_sizes(T, inn, out, w_bit, group, form):
    """Groups of 32 and 64 input channels ("AWQ and Activation-Aware Scaling",
    When it breaks: the gain narrows at g = 32), both scoring forms; in = 64
    and 192 give the scored GEMM one and three K blocks."""
    X, W = random_layer(T, inn, out, seed=T + inn + group)
    cfg = awq.AwqConfig.make(w_bit=w_bit, group_size=group, search_form=form)
    g = gpu_search(X, W, cfg)
    Xn, Wn = X.numpy(), W.numpy()
    mse, _, _, S = O.search_scale(Xn, Wn, O.act_stats(Xn), w_bit, group, 20)
    check_mse(g["mse"], mse)
    check_selection(g["best"], mse, f"alpha g={group}")
    assert np.array_equal(g["s_best"], S[g["best"]])


@pytest.mark.parametrize("out,inn,w_bit,group,n_clip", [
    (72, 96, 4, 32, 0), (136, 320, 3, 64, 0), (512, 4096, 4, 32, 0), (64, 192, 4, 64, 0),
    (72, 96, 4, 32, 20), (136, 320, 3, 64, 7), (520, 1024, 4, 32, 20), (264, 640, 4, 64, 20)])
def test_quant_pack_other_group_sizes(out, inn, w_bit, group, n_clip):
    """Groups of 32 and 64 channels, with and without clip indices; widths
    that leave a partial 128-channel tile (96, 320, 640) and row counts that
    leave a partial 64-row block (72, 136, 264, 520)."""
    X, W = random_layer(16, inn, out, seed=out + inn + n_clip)
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[11]
    cfg = awq.AwqConfig.make(w_bit=w_bit, group_size=group, n_clip=n_clip)
    clip_idx = (np.random.default_rng(out + group).integers(0, n_clip, size=(out, inn // group))
                .astype(np.uint8) if n_clip else None)
    qw = torch.empty((inn, out // 8), dtype=torch.int32, device="cuda")
    qz = torch.empty((inn // group, out // 8), dtype=torch.int32, device="cuda")
    sc = torch.empty((inn // group, out), dtype=torch.float16, device="cuda")
    awq.awq_quant_pack(to_dev(W), torch.from_numpy(s).cuda(),
                       None if clip_idx is None else torch.from_numpy(clip_idx).cuda(), cfg, qw, qz, sc)
    torch.cuda.synchronize()
    awq.awq_device_status(None)
    want = O.quant_pack(W.numpy(), s, clip_idx, w_bit, group, max(n_clip, 1), 0.5)
    for g_, w_, name in zip((qw.cpu().numpy(), qz.cpu().numpy(), sc.cpu().numpy()), want,
                            ("qweight", "qzeros", "scales")):
        assert np.array_equal(g_.view(np.uint8), w_.view(np.uint8)), name


# ------------------------------------------------------------------ candidates in chunks
def _search_with_ws_bytes(X, W, cfg, nbytes):
    Xd, Wd = to_dev(X), to_dev(W)
    T, inn = Xd.shape
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    abar = torch.empty(inn, dtype=torch.float64, device="cuda")
    mse = torch.empty(cfg.n_alpha, dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")
    s_best = torch.empty(inn, dtype=torch.float32, device="cuda")
    awq.awq_act_stats(Xd, abar)
    awq.awq_search_scale(Xd, Wd, abar, cfg, ws, s_best, mse, best)
    awq.awq_device_status(ws)
    return mse.cpu().numpy(), int(best.item()), s_best.cpu().numpy()


@pytest.mark.parametrize("form", [0, 1, 2])
def test_search_scale_in_chunks_is_bitwise_the_same(form):
    """A workspace below awq_workspace_size() runs the candidates in chunks
    (one at a time at awq_workspace_size_min()); every score comes from the
    same tiles, so MSE, selection and s are the same bits."""
    X, W = random_layer(2125, 1024, 520, seed=31)
    cfg = awq.AwqConfig.make(search_form=form)
    full = awq.awq_workspace_size(2125, 1024, 520, cfg)
    low = awq.awq_workspace_size_min(2125, 1024, 520, cfg)
    assert low < full
    ref = _search_with_ws_bytes(X, W, cfg, full)
    for nbytes in (low, low + (full - low) // 3):
        got = _search_with_ws_bytes(X, W, cfg, nbytes)
        assert np.array_equal(got[0], ref[0]) and got[1] == ref[1]
        assert np.array_equal(got[2], ref[2])
    mse_o, _, _, _ = O.search_scale(X.numpy(), W.numpy(), O.act_stats(X.numpy()), 4, 128, 20,
                                    form="fp16_output" if form == 2 else "gram")
    check_mse(ref[0], mse_o)
