"""Token sharding of one layer's AWQ search over several GPUs.

Every statistic the search needs is a sum over calibration tokens: the exact
|x| sums behind abar ("AWQ and Activation-Aware Scaling", Scaling instead of
protecting), each alpha's squared output error ("05 — AWQ: Activation-Aware
Weight Scaling" §4), and the block Grams X_k^T X_k that score the clip ratios.
Each rank holds a slice of the tokens and the full W; it computes its slice's
part of each sum with the library, the parts are added by an all-reduce
(torch.distributed: NCCL over NVLink between GPUs), and the library's
finishing calls turn the sums into the same results a single GPU gives on all
the tokens.  Three all-reduces per layer: int64 [in] (exact, so abar is
bit-identical), fp64 [n_alpha], and fp32 [in/128, 128, 128] when clipping.

The per-shard work goes through an ``ops`` object so that the order and
content of the collectives can be exercised with other implementations of the
same calls; the default, ``LibraryShardOps``, is the CUDA library.
"""

from __future__ import annotations

from typing import Optional

from . import LayerResult, abi


class LibraryShardOps:
    """The library's per-shard and finishing calls on CUDA tensors."""

    def __init__(self, device="cuda"):
        import torch
        self.device = torch.device(device)

    def workspace(self, T: int, inn: int, out: int, cfg: abi.AwqConfig):
        import torch
        n = abi.awq_workspace_size(max(T, 1), inn, out, cfg)
        return torch.empty(n, dtype=torch.uint8, device=self.device)

    def act_sums(self, X, inn: int):
        import torch
        sums = torch.zeros(inn, dtype=torch.int64, device=self.device)
        if X.shape[0] > 0:
            abi.awq_act_sums(X, sums)
        return sums

    def act_finish(self, sums, T_total: int):
        import torch
        abar = torch.empty(sums.shape[0], dtype=torch.float64, device=self.device)
        abi.awq_act_stats_finish(sums, T_total, abar)
        return abar

    def search_sse(self, X, W, abar, cfg, ws):
        import torch
        sse = torch.zeros(cfg.n_alpha, dtype=torch.float64, device=self.device)
        if X.shape[0] > 0:
            abi.awq_search_scale_sse(X, W, abar, cfg, ws, sse)
            abi.awq_device_status(ws)
        return sse

    def select(self, sse, T_total: int, out: int, abar, cfg, ws):
        import torch
        s_best = torch.empty(abar.shape[0], dtype=torch.float32, device=self.device)
        mse = torch.empty(cfg.n_alpha, dtype=torch.float64, device=self.device)
        best = torch.empty(1, dtype=torch.int32, device=self.device)
        abi.awq_select_scale(sse, T_total, out, abar, cfg, ws, s_best, mse, best)
        return s_best, mse, best

    def block_grams(self, X, inn: int, cfg, ws):
        import torch
        G = torch.zeros((inn // 128, 128, 128), dtype=torch.float32, device=self.device)
        if X.shape[0] > 0:
            abi.awq_block_grams(X, cfg, ws, G)
            abi.awq_device_status(ws)
        return G

    def clip_from_grams(self, W, s_best, G, cfg, ws):
        import torch
        out, inn = W.shape
        clip_idx = torch.empty((out, inn // cfg.group_size), dtype=torch.uint8, device=self.device)
        abi.awq_search_clip_grams(W, s_best, G, cfg, ws, clip_idx)
        abi.awq_device_status(ws)
        return clip_idx

    def pack(self, W, s_best, clip_idx, cfg):
        import torch
        out, inn = W.shape
        g = cfg.group_size
        qweight = torch.empty((inn, out // 8), dtype=torch.int32, device=self.device)
        qzeros = torch.empty((inn // g, out // 8), dtype=torch.int32, device=self.device)
        scales = torch.empty((inn // g, out), dtype=torch.float16, device=self.device)
        abi.awq_quant_pack(W, s_best, clip_idx, cfg, qweight, qzeros, scales)
        return qweight, qzeros, scales


def quantize_layer_sharded(X_local, W, cfg: abi.AwqConfig, group=None, ops=None, ws=None,
                           T_total: Optional[int] = None) -> LayerResult:
    """AWQ of one layer whose calibration tokens are split over the ranks of
    ``group`` (torch.distributed; a single process if it is not initialised).

    X_local: this rank's tokens, fp16 [T_local, in] (T_local may be 0);
    W: the full weights, fp16 [out, in], the same on every rank.  Every rank
    returns the same result, equal to ``quantize_layer`` on all the tokens
    (abar and the packing bit for bit; the MSE up to the order of the sums)."""
    import torch
    import torch.distributed as dist

    ops = ops or LibraryShardOps()
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1

    def all_sum(t):
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        return t

    T_local, inn = int(X_local.shape[0]), int(X_local.shape[1])
    out = int(W.shape[0])
    if T_total is None:
        T_total = int(all_sum(torch.tensor([T_local], dtype=torch.int64, device=ops.device)).item())
    if ws is None:
        ws = ops.workspace(T_local, inn, out, cfg)

    sums = all_sum(ops.act_sums(X_local, inn))
    abar = ops.act_finish(sums, T_total)
    sse = all_sum(ops.search_sse(X_local, W, abar, cfg, ws))
    s_best, mse, best = ops.select(sse, T_total, out, abar, cfg, ws)
    clip_idx = None
    if cfg.n_clip > 0:
        G = all_sum(ops.block_grams(X_local, inn, cfg, ws))
        clip_idx = ops.clip_from_grams(W, s_best, G, cfg, ws)
    qweight, qzeros, scales = ops.pack(W, s_best, clip_idx, cfg)
    return LayerResult(abar, mse, best, s_best, clip_idx, qweight, qzeros, scales)
