"""GPU parity without a zero point (the symmetric scheme of "05 — AWQ: Activation-
Aware Weight Scaling" §3, selected by quant_config's zero_point switch, §9):
step = max|s w| / (2^(b-1) - 1), codes centred on z = 2^(b-1).  Same bars as the
asymmetric path: codes, zeros and packing bit-exact; per-alpha MSE within 1e-3;
selections equal unless tied within 1e-4."""

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O
from synthetic import random_layer, workload_inputs

from gpu_helpers import MSE_RTOL, check_mse, check_selection, gpu_search, need_cuda, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


def _pack(W, s, clip_idx, cfg):
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


@pytest.mark.parametrize("out,inn,w_bit,group,use_s,use_clip", [
    (8, 128, 4, 128, False, False), (136, 256, 3, 128, True, True), (512, 512, 4, 128, True, True),
    (72, 96, 4, 32, True, False), (1000, 1024, 3, 64, False, False)])
def test_quant_pack_symmetric_bitwise(out, inn, w_bit, group, use_s, use_clip):
    X, W = random_layer(64, inn, out, seed=out + inn + 3 * w_bit)
    Wn = W.numpy().copy()
    Wn[:8] = np.abs(Wn[:8])  # one-signed rows
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[13] if use_s else None
    n_clip = 20 if use_clip else 0
    clip_idx = (np.random.default_rng(out).integers(0, 20, size=(out, inn // group)).astype(np.uint8)
                if use_clip else None)
    cfg = awq.AwqConfig.make(w_bit=w_bit, group_size=group, zero_point=0, n_clip=n_clip)
    got = _pack(torch.from_numpy(Wn), s, clip_idx, cfg)
    want = O.quant_pack(Wn, s, clip_idx, w_bit, group, max(n_clip, 1), 0.5, zero_point=False)
    for g_, w_, name in zip(got, want, ("qweight", "qzeros", "scales")):
        assert np.array_equal(g_.view(np.uint8), w_.view(np.uint8)), name
    assert np.all(O.unpack_nibbles(got[1]) == 2 ** (w_bit - 1))


@pytest.mark.parametrize("name", ["quant_group_sym_int4.txt", "quant_group_sym_int3.txt",
                                  "quant_group_sym_clip.txt"])
def test_symmetric_hand_worked_through_pack(golden, name):
    """The hand-worked symmetric groups, through the packing kernel (8 equal
    rows): every code, the zero nibble and the fp16 step as derived by hand."""
    hdr, rows = golden(name)
    b = int(hdr["w_bit"])
    W = np.zeros((8, 128), dtype=np.float16)
    for r in rows:
        W[:, int(r[0])] = float(r[1])
    n_clip = int(hdr.get("n_clip", 0))
    idx = np.full((8, 1), int(hdr["clip_index"]), dtype=np.uint8) if "clip_index" in hdr else None
    qw, qz, sc = _pack(torch.from_numpy(W), None, idx, awq.AwqConfig.make(w_bit=b, zero_point=0,
                                                                           n_clip=n_clip))
    q = O.unpack_nibbles(qw)
    assert np.all(sc == np.float16(float(hdr["delta"])))
    assert np.all(O.unpack_nibbles(qz) == int(hdr["zero"]))
    listed = {int(r[0]) for r in rows}
    for r in rows:
        assert np.all(q[:, int(r[0])] == int(r[2])), r
    for j in range(128):
        if j not in listed:
            assert np.all(q[:, j] == int(hdr["zero"]))


@pytest.mark.parametrize("T,inn,out,w_bit,group,form", [
    (64, 128, 16, 4, 128, 0), (200, 384, 264, 3, 128, 0), (2125, 1024, 768, 4, 128, 0),
    (256, 512, 512, 4, 128, 1), (500, 384, 136, 3, 64, 1), (300, 256, 72, 4, 32, 0)])
def test_search_scale_symmetric(T, inn, out, w_bit, group, form):
    X, W = random_layer(T, inn, out, seed=T * 5 + inn + out)
    cfg = awq.AwqConfig.make(w_bit=w_bit, group_size=group, zero_point=0, search_form=form)
    g = gpu_search(X, W, cfg)
    Xn, Wn = X.numpy(), W.numpy()
    mse, _, _, S = O.search_scale(Xn, Wn, O.act_stats(Xn), w_bit, group, 20, zero_point=False)
    check_mse(g["mse"], mse)
    check_selection(g["best"], mse, "alpha (symmetric)")
    assert np.array_equal(g["s_best"], S[g["best"]])


def _gpu_clip(X, W, s, cfg):
    Xd, Wd = to_dev(X), to_dev(W)
    T, inn = Xd.shape
    out = Wd.shape[0]
    ws = awq.alloc_workspace(T, inn, out, cfg)
    idx = torch.empty((out, inn // 128), dtype=torch.uint8, device="cuda")
    err = torch.empty((out, inn // 128, cfg.n_clip), dtype=torch.float32, device="cuda")
    awq.awq_search_clip(Xd, Wd, torch.from_numpy(s).cuda(), cfg, ws, idx, err)
    awq.awq_device_status(ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), err.cpu().numpy()


@pytest.mark.parametrize("T,inn,out,w_bit,n_clip", [(300, 256, 40, 4, 20), (1500, 512, 96, 3, 20),
                                                     (64, 128, 8, 4, 7)])
def test_search_clip_symmetric(T, inn, out, w_bit, n_clip):
    X, W = random_layer(T, inn, out, seed=T + out + 2 * n_clip)
    Xn, Wn = X.numpy(), W.numpy()
    s = O.scale_grid(O.act_stats(Xn), O.alpha_grid(20))[10]
    cfg = awq.AwqConfig.make(w_bit=w_bit, zero_point=0, n_clip=n_clip)
    idx, err = _gpu_clip(X, W, s, cfg)
    idx_o, E = O.search_clip(Xn, Wn, s, w_bit, 128, n_clip, 0.5, zero_point=False)
    rel = np.abs(err - E) / np.maximum(np.abs(E), 1e-30)
    assert rel.max() <= MSE_RTOL, rel.max()
    for o, k in zip(*np.nonzero(idx != idx_o)):
        check_selection(int(idx[o, k]), E[o, k], f"clip row {o} group {k}")


def test_q_proj_workload_symmetric_sampled_rows():
    """Full T = 65536 and in = 4096 of the q_proj workload, 256 sampled output
    rows (same launch shapes along T and in): the whole layer without a zero
    point -- search, clip, packing -- against the oracle."""
    d = workload_inputs(1)
    _, X, W = d["groups"][0]
    rows = np.sort(np.random.default_rng(3).choice(W.shape[0], 256, replace=False))
    Ws = W[torch.from_numpy(rows)]
    cfg = awq.AwqConfig.make(w_bit=4, zero_point=0, n_alpha=20, n_clip=20)
    Xd, Wd = to_dev(X), to_dev(Ws)
    ws = awq.alloc_workspace(Xd.shape[0], Xd.shape[1], Wd.shape[0], cfg)
    res = awq.quantize_layer(Xd, Wd, cfg, ws=ws)
    awq.awq_device_status(ws)
    torch.cuda.synchronize()
    Xn, Wn = X.numpy(), Ws.numpy()
    abar = O.act_stats(Xn)
    G = O.gram(Xn)
    mse, _, _, S = O.search_scale(Xn, Wn, abar, 4, 128, 20, G=G, zero_point=False)
    check_mse(res.mse.cpu().numpy(), mse)
    best = int(res.best_idx.item())
    check_selection(best, mse, "alpha")
    s = S[best]
    assert np.array_equal(res.s_best.cpu().numpy(), s)
    Gk = [G[128 * k:128 * (k + 1), 128 * k:128 * (k + 1)] for k in range(Wn.shape[1] // 128)]
    clip = res.clip_idx.cpu().numpy()
    idx_o, E = O.search_clip(Xn, Wn, s, 4, 128, 20, 0.5, Gk=Gk, zero_point=False)
    for o, k in zip(*np.nonzero(clip != idx_o)):
        check_selection(int(clip[o, k]), E[o, k], f"clip row {o} group {k}")
    qw, qz, sc = O.quant_pack(Wn, s, clip, 4, 128, 20, 0.5, zero_point=False)
    assert np.array_equal(res.qweight.cpu().numpy(), qw)
    assert np.array_equal(res.qzeros.cpu().numpy(), qz)
    assert np.array_equal(res.scales.cpu().numpy().view(np.uint16), sc.view(np.uint16))
