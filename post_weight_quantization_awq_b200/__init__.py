"""AWQ per-layer activation-aware scale search on B200 (sm_100a).

Public API: the C-ABI calls of include/awq.h under the same names
(``awq_act_stats``, ``awq_search_scale``, ``awq_search_clip``,
``awq_quant_pack``, ...) taking torch CUDA tensors, plus ``quantize_layer``,
which runs the four calls for one linear (or one group of linears that share
an input) and returns the packed result.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

from .abi import (  # noqa: F401
    AwqConfig,
    AwqError,
    awq_act_stats,
    awq_act_stats_finish,
    awq_act_sums,
    awq_block_grams,
    awq_bounds_checks_enabled,
    awq_bounds_status,
    awq_candidate_codes,
    awq_clip_candidate_codes,
    awq_device_status,
    awq_fold_inv_scale,
    awq_quant_pack,
    awq_scale_grid,
    awq_search_clip,
    awq_search_clip_grams,
    awq_search_clip_noalloc,
    awq_search_scale,
    awq_search_scale_sse,
    awq_select_scale,
    awq_w4a16_gemm,
    awq_w4a16_workspace_size,
    awq_workspace_size,
    awq_workspace_size_min,
    header_functions,
    last_error,
    profile_enable,
    profile_read,
    profile_reset,
    version,
)


@dataclasses.dataclass
class LayerResult:
    """Output of one layer's search (all CUDA tensors)."""

    abar: "torch.Tensor"       # fp64 [in]
    mse: "torch.Tensor"        # fp64 [n_alpha]
    best_idx: "torch.Tensor"   # int32 [1]
    s_best: "torch.Tensor"     # fp32 [in]
    clip_idx: Optional["torch.Tensor"]  # uint8 [out, in/g] or None
    qweight: "torch.Tensor"    # int32 [in, out/8]
    qzeros: "torch.Tensor"     # int32 [in/g, out/8]
    scales: "torch.Tensor"     # fp16 [in/g, out]


def alloc_workspace(T: int, inn: int, out: int, cfg: AwqConfig, device="cuda"):
    import torch
    n = awq_workspace_size(T, inn, out, cfg)
    return torch.empty(n, dtype=torch.uint8, device=device)


def quantize_layer(X, W, cfg: AwqConfig, ws=None, stream=None) -> LayerResult:
    """act stats -> alpha search -> [clip search] -> quantise + pack, all on
    the current CUDA stream.  X: fp16 [T, in]; W: fp16 [out, in] (linears that
    share X and one scale concatenated along out)."""
    import torch
    T, inn = X.shape
    out = W.shape[0]
    dev = X.device
    g = cfg.group_size
    if ws is None:
        ws = alloc_workspace(T, inn, out, cfg, dev)
    abar = torch.empty(inn, dtype=torch.float64, device=dev)
    mse = torch.empty(cfg.n_alpha, dtype=torch.float64, device=dev)
    best = torch.empty(1, dtype=torch.int32, device=dev)
    s_best = torch.empty(inn, dtype=torch.float32, device=dev)
    awq_act_stats(X, abar, stream)
    awq_search_scale(X, W, abar, cfg, ws, s_best, mse, best, stream)
    clip_idx = None
    if cfg.n_clip > 0:
        clip_idx = torch.empty((out, inn // g), dtype=torch.uint8, device=dev)
        awq_search_clip(X, W, s_best, cfg, ws, clip_idx, None, stream)
    qweight = torch.empty((inn, out // 8), dtype=torch.int32, device=dev)
    qzeros = torch.empty((inn // g, out // 8), dtype=torch.int32, device=dev)
    scales = torch.empty((inn // g, out), dtype=torch.float16, device=dev)
    awq_quant_pack(W, s_best, clip_idx, cfg, qweight, qzeros, scales, stream)
    return LayerResult(abar, mse, best, s_best, clip_idx, qweight, qzeros, scales)
