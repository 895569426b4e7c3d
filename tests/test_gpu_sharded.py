"""GPU side of the token-sharded layer (post_weight_quantization_awq_b200.sharded):
the library's per-shard calls on slices of the tokens, their parts added on the
device as an all-reduce would, and the finishing calls, against the oracle on
all tokens; and the sharded path on one process, which must reproduce
quantize_layer bit for bit (same kernels, same sums)."""

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from post_weight_quantization_awq_b200.sharded import LibraryShardOps, quantize_layer_sharded
from oracle import awq_oracle as O
from synthetic import random_layer

from gpu_helpers import check_mse, check_selection, need_cuda, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


@pytest.mark.parametrize("T,inn,out,w_bit,cuts,form", [
    (2125, 1024, 264, 4, (1000,), 0), (600, 512, 136, 3, (129, 300), 0), (900, 512, 256, 4, (450,), 2),
    (700, 384, 128, 4, (350,), 1), (1100, 512, 264, 4, (400, 700), 3)])
def test_shards_summed_on_device_match_oracle(T, inn, out, w_bit, cuts, form):
    X, W = random_layer(T, inn, out, seed=T + inn + out)
    cfg = awq.AwqConfig.make(w_bit=w_bit, n_alpha=20, n_clip=20, search_form=form)
    Xd, Wd = to_dev(X), to_dev(W)
    ops = LibraryShardOps()
    bounds = (0,) + tuple(cuts) + (T,)
    shards = [Xd[a:b] for a, b in zip(bounds[:-1], bounds[1:])]
    ws = ops.workspace(max(x.shape[0] for x in shards), inn, out, cfg)
    sums = sum(ops.act_sums(x, inn) for x in shards)
    abar = ops.act_finish(sums, T)
    full = torch.empty(inn, dtype=torch.float64, device="cuda")
    awq.awq_act_stats(Xd, full)
    assert torch.equal(abar, full)  # exact sums: bit for bit
    sse = sum(ops.search_sse(x, Wd, abar, cfg, ws) for x in shards)
    s_best, mse, best = ops.select(sse, T, out, abar, cfg, ws)
    G = sum(ops.block_grams(x, inn, cfg, ws) for x in shards)
    clip = ops.clip_from_grams(Wd, s_best, G, cfg, ws)
    qw, qz, sc = ops.pack(Wd, s_best, clip, cfg)
    torch.cuda.synchronize()

    Xn, Wn = X.numpy(), W.numpy()
    abar_o = O.act_stats(Xn)
    assert np.array_equal(abar.cpu().numpy(), abar_o)
    form_o = "fp16_output" if form == awq.abi.SEARCH_CACHED_Y else "direct"
    mse_o, _, _, S = O.search_scale(Xn, Wn, abar_o, w_bit, 128, 20, form=form_o)
    check_mse(mse.cpu().numpy(), mse_o)
    b = int(best.item())
    check_selection(b, mse_o, "alpha (sharded)")
    s = S[b]
    assert np.array_equal(s_best.cpu().numpy(), s)
    idx_o, E = O.search_clip(Xn, Wn, s, w_bit, 128, 20, 0.5)
    got = clip.cpu().numpy()
    for o, k in zip(*np.nonzero(got != idx_o)):
        check_selection(int(got[o, k]), E[o, k], f"clip row {o} group {k}")
    want = O.quant_pack(Wn, s, got, w_bit, 128, 20, 0.5)
    for g_, w_, name in zip((qw.cpu().numpy(), qz.cpu().numpy(), sc.cpu().numpy()), want,
                            ("qweight", "qzeros", "scales")):
        assert np.array_equal(g_.view(np.uint8), w_.view(np.uint8)), name


def test_single_process_sharded_path_is_quantize_layer():
    X, W = random_layer(1500, 1024, 512, seed=41)
    cfg = awq.AwqConfig.make(w_bit=4, n_alpha=20, n_clip=20)
    Xd, Wd = to_dev(X), to_dev(W)
    a = awq.quantize_layer(Xd, Wd, cfg)
    b = quantize_layer_sharded(Xd, Wd, cfg)
    torch.cuda.synchronize()
    for name in ("abar", "mse", "best_idx", "s_best", "clip_idx", "qweight", "qzeros", "scales"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
