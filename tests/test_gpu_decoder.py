"""The 32-layer Llama-2-7B-architecture decoder workload: layer-by-layer AWQ
(four groups per layer, INT4 g128, 20 alphas + 20 clip ratios, folds, packing)
with the calibration hidden states propagated through the fp16 layers, at
the workload's 128 x 512 = 65536 calibration tokens.  On sampled layers every output is checked
against the CPU oracle: abar, s, folds and packing bit-exact on the whole
layer; clip choices on sampled rows; and the alpha search, run through the
same C ABI on sampled rows of the same captured inputs, against the oracle's
MSE curve."""

import os

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from post_weight_quantization_awq_b200 import decoder
from oracle import awq_oracle as O
from synthetic import DecoderSpec, decoder_embeddings, decoder_layer_forward, decoder_layer_weights

from gpu_helpers import check_mse, check_selection, gpu_search, need_cuda

pytestmark = pytest.mark.gpu

SAMPLED_LAYERS = (0, 1, 15, 31)


def _check_layer(caps, w_orig, w_folded, res, cfg, rng):
    for g, names in decoder.GROUPS:
        X = caps[g].cpu().numpy()
        W = np.concatenate([w_orig[n] for n in names], 0)
        r = res[g]
        abar = O.act_stats(X)
        assert np.array_equal(r["abar"].cpu().numpy(), abar), g
        S = O.scale_grid(abar, O.alpha_grid(cfg.n_alpha))
        best = int(r["best_idx"].item())
        s = S[best]
        assert np.array_equal(r["s"].cpu().numpy(), s), g
        # alpha search on sampled rows, same X, same launch shape along T and in
        rows = np.sort(rng.choice(W.shape[0], 256, replace=False))
        gs = gpu_search(torch.from_numpy(X), torch.from_numpy(W[rows]), cfg)
        mse_o, best_o, _, _ = O.search_scale(X, W[rows], abar, cfg.w_bit, 128, cfg.n_alpha)
        check_mse(gs["mse"], mse_o)
        check_selection(gs["best"], mse_o, f"{g} alpha")
        # packing of the folded weights, whole group, bit-exact
        Wf = np.concatenate([w_folded[n] for n in names], 0)
        clip = r["clip_idx"].cpu().numpy()
        qw, qz, sc = O.quant_pack(Wf, s, clip, cfg.w_bit, 128, cfg.n_clip, cfg.clip_min)
        assert np.array_equal(r["qweight"].cpu().numpy(), qw), g
        assert np.array_equal(r["qzeros"].cpu().numpy(), qz), g
        assert np.array_equal(r["scales"].cpu().numpy().view(np.uint16), sc.view(np.uint16)), g
        # clip choices on sampled rows
        crow = np.sort(rng.choice(W.shape[0], 64, replace=False))
        idx_o, E = O.search_clip(X, Wf[crow], s, cfg.w_bit, 128, cfg.n_clip, cfg.clip_min)
        got = clip[crow]
        for o, k in zip(*np.nonzero(got != idx_o)):
            check_selection(int(got[o, k]), E[o, k], f"{g} clip")


def test_llama7b_decoder_layer_by_layer(tmp_path):
    need_cuda()
    spec = DecoderSpec()  # 128 sequences x 512 tokens
    cfg = awq.AwqConfig.make(w_bit=4, n_alpha=20, n_clip=20, clip_min=0.5)
    rng = np.random.default_rng(5)
    x = decoder_embeddings(spec, device="cuda")
    ws = None
    for layer in range(spec.layers):
        w = decoder_layer_weights(spec, layer, device="cuda")
        caps, x_next = decoder_layer_forward(x, w, spec)
        keep = layer in SAMPLED_LAYERS
        w_orig = {n: t.cpu().numpy() for n, t in w.items()} if keep else None
        if ws is None:
            ws = decoder.workspace_for_layer(caps, w, cfg)
        res = decoder.quantize_layer_groups(caps, w, cfg, ws)
        torch.cuda.synchronize()
        if keep:
            w_folded = {n: t.cpu().numpy() for n, t in w.items()}
            # the folds, bit-exact: gamma1 <- qkv's s, v rows <- o's s,
            # gamma2 <- gate|up's s, up rows <- down's s
            for g, target in decoder.FOLDS:
                want = O.fold_inv_scale(w_orig[target], res[g]["s"].cpu().numpy())
                assert np.array_equal(w_folded[target].view(np.uint16), want.view(np.uint16)), target
            _check_layer(caps, w_orig, w_folded, res, cfg, rng)
            path = os.path.join(tmp_path, f"layer{layer:02d}.pt")
            decoder.save_layer_checkpoint(path, layer, res)
            state = torch.load(path)
            assert state["layer"] == layer and torch.equal(state["qkv"]["qweight"], res["qkv"]["qweight"].cpu())
        x = x_next
        assert torch.isfinite(x.float()).all()
