"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the CPU oracle on the same seeded inputs, and compare."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O

MSE_RTOL = 1e-3      # per-alpha MSE, fp32 tensor-core accumulation vs fp64
TIE_RTOL = 1e-4      # selections may differ only between near-tied candidates


def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def to_dev(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().cuda()


def gpu_search(X: torch.Tensor, W: torch.Tensor, cfg: awq.AwqConfig):
    """act_stats + search_scale on the GPU; returns numpy results."""
    Xd, Wd = to_dev(X), to_dev(W)
    T, inn = Xd.shape
    out = Wd.shape[0]
    ws = awq.alloc_workspace(T, inn, out, cfg)
    abar = torch.empty(inn, dtype=torch.float64, device="cuda")
    mse = torch.empty(cfg.n_alpha, dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")
    s_best = torch.empty(inn, dtype=torch.float32, device="cuda")
    awq.awq_act_stats(Xd, abar)
    awq.awq_search_scale(Xd, Wd, abar, cfg, ws, s_best, mse, best)
    awq.awq_device_status(ws)
    torch.cuda.synchronize()
    return {"abar": abar.cpu().numpy(), "mse": mse.cpu().numpy(), "best": int(best.item()),
            "s_best": s_best.cpu().numpy(), "ws": ws}


def check_selection(gpu_idx: int, oracle_scores: np.ndarray, what: str):
    """Same index as the oracle, unless the oracle's scores of the two indices
    are within TIE_RTOL of each other."""
    o_idx = int(np.argmin(oracle_scores))
    if gpu_idx == o_idx:
        return
    a, b = oracle_scores[gpu_idx], oracle_scores[o_idx]
    assert abs(a - b) <= TIE_RTOL * abs(b), (what, gpu_idx, o_idx, a, b)


def check_mse(gpu_mse: np.ndarray, oracle_mse: np.ndarray):
    rel = np.abs(gpu_mse - oracle_mse) / np.abs(oracle_mse)
    assert np.all(rel <= MSE_RTOL), (rel.max(), gpu_mse, oracle_mse)
    return float(rel.max())


def midpoint_report(abar: np.ndarray, alphas: np.ndarray, s_gpu: np.ndarray, s_ref: np.ndarray) -> str:
    """For s-grid mismatches: how far the double pow result sits from the
    fp32 rounding midpoint (a 1-ulp difference between two libm pows can only
    flip values that sit on a midpoint)."""
    bad = np.argwhere(s_gpu != s_ref)
    lines = []
    for i, j in bad[:10]:
        x = max(float(abar[j]), 1e-4)
        v = x ** float(alphas[i])
        lo, hi = sorted((float(s_gpu[i, j]), float(s_ref[i, j])))
        mid = (lo + hi) / 2
        lines.append(f"alpha[{i}] ch {j}: pow={v!r} fp32 gpu={s_gpu[i, j]!r} ref={s_ref[i, j]!r} "
                     f"|pow-mid|/ulp={abs(v - mid) / (hi - lo):.3e}")
    return "\n".join(lines)


def layer_parity(X, W, w_bit, n_alpha, n_clip, rows=None):
    """The whole path at full T and in; with `rows`, on that sample of output
    rows (the same launch configuration with a smaller N)."""
    if rows is not None:
        W = W[rows]
    cfg = awq.AwqConfig.make(w_bit=w_bit, n_alpha=n_alpha, n_clip=n_clip)
    Xd, Wd = to_dev(X), to_dev(W)
    ws = awq.alloc_workspace(Xd.shape[0], Xd.shape[1], Wd.shape[0], cfg)
    res = awq.quantize_layer(Xd, Wd, cfg, ws=ws)
    awq.awq_device_status(ws)
    torch.cuda.synchronize()
    Xn, Wn = X.numpy(), W.numpy()
    abar = O.act_stats(Xn)
    assert np.array_equal(res.abar.cpu().numpy(), abar)
    mse, best, s_best, S = O.search_scale(Xn, Wn, abar, w_bit, 128, n_alpha)
    g_mse = res.mse.cpu().numpy()
    check_mse(g_mse, mse)
    g_best = int(res.best_idx.item())
    check_selection(g_best, mse, "alpha")
    s = S[g_best]
    assert np.array_equal(res.s_best.cpu().numpy(), s)
    clip_idx = None
    if n_clip:
        clip_idx = res.clip_idx.cpu().numpy()
        idx_o, E = O.search_clip(Xn, Wn, s, w_bit, 128, n_clip, 0.5)
        for o, k in zip(*np.nonzero(clip_idx != idx_o)):
            check_selection(int(clip_idx[o, k]), E[o, k], f"clip row {o} group {k}")
    qw, qz, sc = O.quant_pack(Wn, s, clip_idx, w_bit, 128, max(n_clip, 1), 0.5)
    assert np.array_equal(res.qweight.cpu().numpy(), qw)
    assert np.array_equal(res.qzeros.cpu().numpy(), qz)
    assert np.array_equal(res.scales.cpu().numpy().view(np.uint16), sc.view(np.uint16))
    return g_mse, mse
