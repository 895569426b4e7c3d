"""GPU parity on the method's degenerate cases, with a zero point (the default)
and without: synthetic.edge_layer gives one-signed narrow groups (the exact
division decides, the zero point clamps), constant and all-zero groups (the
1e-5 range floor), fp16-subnormal weights, and dead input channels (mean |x|
of 0 and below 1e-4: s at its floor, r = sqrt(G_jj) = 0 in the Gram form and in
the clip search's normalisation).  Every scoring form, the clip search and the
packing run on them; bars as in the other parity tests (codes and packing
bit-exact, MSE and clip errors within 1e-3, selections equal unless tied
within 1e-4).  Also: the non-finite score check, and the packing's check of
its clip indices."""

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O
from synthetic import edge_layer

from gpu_helpers import MSE_RTOL, check_mse, check_selection, gpu_search, need_cuda, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


FORMS = {0: "direct", 1: "gram", 2: "fp16_output"}


@pytest.mark.parametrize("form", [0, 1, 2])
@pytest.mark.parametrize("T,inn,out,w_bit,group,zp", [
    (300, 512, 264, 4, 128, 1), (700, 768, 136, 3, 128, 1), (257, 512, 72, 4, 32, 1),
    (400, 512, 264, 4, 128, 0), (300, 384, 136, 4, 64, 0)])
def test_search_scale_edge_layer(form, T, inn, out, w_bit, group, zp):
    X, W = edge_layer(T, inn, out, seed=T + inn + out + group, group=group)
    cfg = awq.AwqConfig.make(w_bit=w_bit, group_size=group, zero_point=zp, search_form=form)
    g = gpu_search(X, W, cfg)
    Xn, Wn = X.numpy(), W.numpy()
    abar = O.act_stats(Xn)
    assert np.array_equal(g["abar"], abar)
    assert abar[0] == 0.0
    mse, _, _, S = O.search_scale(Xn, Wn, abar, w_bit, group, 20, form=FORMS[form],
                                  zero_point=bool(zp))
    check_mse(g["mse"], mse)
    check_selection(g["best"], mse, f"alpha ({FORMS[form]})")
    assert np.array_equal(g["s_best"], S[g["best"]])


def _clip(X, W, s, cfg):
    Xd, Wd = to_dev(X), to_dev(W)
    T, inn = Xd.shape
    out = Wd.shape[0]
    ws = awq.alloc_workspace(T, inn, out, cfg)
    idx = torch.empty((out, inn // 128), dtype=torch.uint8, device="cuda")
    err = torch.empty((out, inn // 128, cfg.n_clip), dtype=torch.float32, device="cuda")
    awq.awq_search_clip(Xd, Wd, torch.from_numpy(s).cuda(), cfg, ws, idx, err)
    awq.awq_device_status(ws)
    return idx.cpu().numpy(), err.cpu().numpy()


@pytest.mark.parametrize("w_bit,zp", [(4, 1), (3, 1), (4, 0)])
def test_search_clip_and_pack_edge_layer(w_bit, zp):
    X, W = edge_layer(600, 512, 264, seed=70 + w_bit + zp)
    Xn, Wn = X.numpy(), W.numpy()
    s = O.scale_grid(O.act_stats(Xn), O.alpha_grid(20))[17]
    cfg = awq.AwqConfig.make(w_bit=w_bit, n_clip=20, zero_point=zp)
    idx, err = _clip(X, W, s, cfg)
    idx_o, E = O.search_clip(Xn, Wn, s, w_bit, 128, 20, 0.5, zero_point=bool(zp))
    # groups whose error is exactly zero (dead inputs, zero weights) must be
    # zero on the GPU too; the rest within the bar
    zero = E == 0
    assert np.all(err[zero] == 0)
    rel = np.abs(err[~zero] - E[~zero]) / np.abs(E[~zero])
    assert rel.max() <= MSE_RTOL, rel.max()
    for o, k in zip(*np.nonzero(idx != idx_o)):
        check_selection(int(idx[o, k]), E[o, k], f"clip row {o} group {k}")
    qw = torch.empty((512, 264 // 8), dtype=torch.int32, device="cuda")
    qz = torch.empty((4, 264 // 8), dtype=torch.int32, device="cuda")
    sc = torch.empty((4, 264), dtype=torch.float16, device="cuda")
    awq.awq_quant_pack(to_dev(W), torch.from_numpy(s).cuda(), torch.from_numpy(idx).cuda(), cfg,
                       qw, qz, sc)
    awq.awq_device_status(None)
    want = O.quant_pack(Wn, s, idx, w_bit, 128, 20, 0.5, zero_point=bool(zp))
    for got, ref, name in zip((qw, qz, sc), want, ("qweight", "qzeros", "scales")):
        assert np.array_equal(got.cpu().numpy().view(np.uint8), ref.view(np.uint8)), name


def test_whole_path_edge_layer_all_forms_agree():
    """quantize_layer on the edge layer with each scoring form: all three
    pack the same bits when they select the same alpha."""
    X, W = edge_layer(1000, 1024, 520, seed=91)
    outs = []
    for form in (0, 1, 2):
        cfg = awq.AwqConfig.make(n_clip=20, search_form=form)
        res = awq.quantize_layer(to_dev(X), to_dev(W), cfg)
        torch.cuda.synchronize()
        outs.append(res)
    for r in outs[1:]:
        if int(r.best_idx.item()) == int(outs[0].best_idx.item()):
            assert torch.equal(r.qweight, outs[0].qweight)
            assert torch.equal(r.scales.view(torch.int16), outs[0].scales.view(torch.int16))


# ------------------------------------------------------------------ status paths
def test_nonfinite_weight_is_reported():
    """An infinite weight makes every candidate's score non-finite: the search
    reports AWQ_ERR_NONFINITE, and the next call on valid input is clean."""
    X, W = edge_layer(256, 512, 264, seed=5)
    W[7, 300] = float("inf")
    cfg = awq.AwqConfig.make()
    Xd, Wd = to_dev(X), to_dev(W)
    ws = awq.alloc_workspace(256, 512, 264, cfg)
    abar = torch.empty(512, dtype=torch.float64, device="cuda")
    mse = torch.empty(20, dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")
    s_best = torch.empty(512, dtype=torch.float32, device="cuda")
    awq.awq_act_stats(Xd, abar)
    awq.awq_search_scale(Xd, Wd, abar, cfg, ws, s_best, mse, best)
    with pytest.raises(awq.AwqError) as ei:
        awq.awq_device_status(ws)
    assert ei.value.status_name == "AWQ_ERR_NONFINITE"
    assert not np.all(np.isfinite(mse.cpu().numpy()))
    Wd[7, 300] = 0.0
    awq.awq_search_scale(Xd, Wd, abar, cfg, ws, s_best, mse, best)
    awq.awq_device_status(ws)
    assert np.all(np.isfinite(mse.cpu().numpy()))


@pytest.mark.parametrize("form", [0, 1, 2])
def test_injected_nonfinite_is_reported(monkeypatch, form):
    X, W = edge_layer(256, 512, 264, seed=6)
    cfg = awq.AwqConfig.make(search_form=form)
    monkeypatch.setenv("AWQ_FAULT", "nonfinite")
    g = None
    with pytest.raises(awq.AwqError) as ei:
        gpu_search(X, W, cfg)
    assert ei.value.status_name == "AWQ_ERR_NONFINITE"
    monkeypatch.delenv("AWQ_FAULT")
    g = gpu_search(X, W, cfg)
    assert np.all(np.isfinite(g["mse"]))


def test_injected_nonfinite_in_token_sharded_selection(monkeypatch):
    cfg = awq.AwqConfig.make()
    sse = torch.rand(20, dtype=torch.float64, device="cuda") + 1.0
    abar = torch.rand(512, dtype=torch.float64, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    s_best = torch.empty(512, dtype=torch.float32, device="cuda")
    mse = torch.empty(20, dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("AWQ_FAULT", "nonfinite")
    awq.awq_select_scale(sse, 1000, 264, abar, cfg, ws, s_best, mse, best)
    with pytest.raises(awq.AwqError) as ei:
        awq.awq_device_status(ws)
    assert ei.value.status_name == "AWQ_ERR_NONFINITE"
    monkeypatch.delenv("AWQ_FAULT")
    awq.awq_select_scale(sse, 1000, 264, abar, cfg, ws, s_best, mse, best)
    awq.awq_device_status(ws)


@pytest.mark.parametrize("bad", [20, 63, 64, 255])
def test_pack_rejects_clip_index_past_the_grid(monkeypatch, bad):
    """A clip index >= n_clip marks its group (codes and zero 0, NaN scale),
    leaves the other groups exact, and is reported by the library status
    word; with AWQ_SYNC_CHECK the call reports it itself."""
    X, W = edge_layer(64, 512, 136, seed=8)
    Wn = W.numpy()
    rng = np.random.default_rng(bad)
    idx = rng.integers(0, 20, size=(136, 4)).astype(np.uint8)
    idx[5, 2] = bad
    idx[100, 0] = bad
    cfg = awq.AwqConfig.make(n_clip=20)
    qw = torch.empty((512, 17), dtype=torch.int32, device="cuda")
    qz = torch.empty((4, 17), dtype=torch.int32, device="cuda")
    sc = torch.empty((4, 136), dtype=torch.float16, device="cuda")
    awq.awq_device_status(None)  # start clean
    awq.awq_quant_pack(to_dev(W), None, torch.from_numpy(idx).cuda(), cfg, qw, qz, sc)
    with pytest.raises(awq.AwqError) as ei:
        awq.awq_device_status(None)
    assert ei.value.status_name == "AWQ_ERR_INVALID_ARG"
    awq.awq_device_status(None)  # read clears it
    ok = idx.copy()
    ok[5, 2] = 0
    ok[100, 0] = 0
    want_qw, want_qz, want_sc = O.quant_pack(Wn, None, ok, 4, 128, 20, 0.5)
    q, qo = O.unpack_nibbles(qw.cpu().numpy()), O.unpack_nibbles(want_qw)
    z, zo = O.unpack_nibbles(qz.cpu().numpy()), O.unpack_nibbles(want_qz)
    scn = sc.cpu().numpy()
    for (o, k) in ((5, 2), (100, 0)):
        assert np.all(q[o, 128 * k:128 * (k + 1)] == 0) and z[o, k] == 0 and np.isnan(scn[k, o])
        q[o, 128 * k:128 * (k + 1)] = qo[o, 128 * k:128 * (k + 1)]
        z[o, k] = zo[o, k]
        scn[k, o] = want_sc[k, o]
    assert np.array_equal(q, qo) and np.array_equal(z, zo)
    assert np.array_equal(scn.view(np.uint16), want_sc.view(np.uint16))
    monkeypatch.setenv("AWQ_SYNC_CHECK", "1")
    with pytest.raises(awq.AwqError) as ei:
        awq.awq_quant_pack(to_dev(W), None, torch.from_numpy(idx).cuda(), cfg, qw, qz, sc)
    assert ei.value.status_name == "AWQ_ERR_INVALID_ARG"
    awq.awq_quant_pack(to_dev(W), None, torch.from_numpy(ok).cuda(), cfg, qw, qz, sc)
