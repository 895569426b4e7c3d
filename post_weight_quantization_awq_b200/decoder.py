"""Layer-by-layer AWQ of a Llama-style decoder layer (the pages' offline
pass: "AWQ and Activation-Aware Scaling", Why this is attractive: forward
passes to collect statistics, then a small per-layer search).

Per layer, for the four groups of linears that share an input
(q|k|v, o, gate|up, down):
  1. abar and the alpha search on the captured fp16 inputs (awq_act_stats,
     awq_search_scale), all four groups before any weight changes;
  2. fold 1/s into the operation feeding each group ("Scaling instead of
     protecting": the activation-side division is absorbed by the preceding
     normalisation's scale or linear layer): RMSNorm1 gamma <- qkv's s,
     v_proj rows <- o's s, RMSNorm2 gamma <- gate|up's s, up_proj rows <-
     down's s (awq_fold_inv_scale, in fp16);
  3. clip search and packing of each group on the folded weights
     (awq_search_clip, awq_quant_pack).
Every step runs in the library's kernels; this module only orders the calls
and slices the concatenated results.
"""

from __future__ import annotations

import os
from typing import Dict, Optional

import torch

from . import abi
from .abi import AwqConfig

GROUPS = (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gate_up", ("gate", "up")), ("down", ("down",)))
FOLDS = (("qkv", "gamma1"), ("o", "v"), ("gate_up", "gamma2"), ("down", "up"))


def _search(X: torch.Tensor, W: torch.Tensor, cfg: AwqConfig, ws: torch.Tensor):
    inn = X.shape[1]
    dev = X.device
    abar = torch.empty(inn, dtype=torch.float64, device=dev)
    mse = torch.empty(cfg.n_alpha, dtype=torch.float64, device=dev)
    best = torch.empty(1, dtype=torch.int32, device=dev)
    s = torch.empty(inn, dtype=torch.float32, device=dev)
    abi.awq_act_stats(X, abar)
    abi.awq_search_scale(X, W, abar, cfg, ws, s, mse, best)
    return {"abar": abar, "mse": mse, "best_idx": best, "s": s}


def workspace_for_layer(captures: Dict[str, torch.Tensor], weights: Dict[str, torch.Tensor],
                        cfg: AwqConfig) -> torch.Tensor:
    need = 0
    for g, names in GROUPS:
        X = captures[g]
        out = sum(weights[n].shape[0] for n in names)
        need = max(need, abi.awq_workspace_size(X.shape[0], X.shape[1], out, cfg))
    return torch.empty(need, dtype=torch.uint8, device=captures["qkv"].device)


def quantize_layer_groups(captures: Dict[str, torch.Tensor], weights: Dict[str, torch.Tensor],
                          cfg: AwqConfig, ws: Optional[torch.Tensor] = None) -> dict:
    """AWQ of one decoder layer.  `weights` (fp16, [out, in]; gammas [hidden])
    are modified in place by the folds.  Returns per group: abar, mse,
    best_idx, s, clip_idx, qweight, qzeros, scales (concatenated along out for
    joint groups) and per linear the (first, last) output rows."""
    if ws is None:
        ws = workspace_for_layer(captures, weights, cfg)
    res = {}
    cat = {g: (torch.cat([weights[n] for n in names], 0) if len(names) > 1 else weights[names[0]])
           for g, names in GROUPS}
    for g, _ in GROUPS:
        res[g] = _search(captures[g], cat[g], cfg, ws)
        abi.awq_device_status(ws)
    for g, target in FOLDS:
        abi.awq_fold_inv_scale(weights[target], res[g]["s"])
    for g, names in GROUPS:
        W = torch.cat([weights[n] for n in names], 0) if len(names) > 1 else weights[names[0]]
        X = captures[g]
        out, inn = W.shape
        gsz = cfg.group_size
        clip_idx = None
        if cfg.n_clip > 0:
            clip_idx = torch.empty((out, inn // gsz), dtype=torch.uint8, device=W.device)
            abi.awq_search_clip(X, W, res[g]["s"], cfg, ws, clip_idx)
            abi.awq_device_status(ws)
        qweight = torch.empty((inn, out // 8), dtype=torch.int32, device=W.device)
        qzeros = torch.empty((inn // gsz, out // 8), dtype=torch.int32, device=W.device)
        scales = torch.empty((inn // gsz, out), dtype=torch.float16, device=W.device)
        abi.awq_quant_pack(W, res[g]["s"], clip_idx, cfg, qweight, qzeros, scales)
        rows, r0 = {}, 0
        for n in names:
            rows[n] = (r0, r0 + weights[n].shape[0])
            r0 += weights[n].shape[0]
        res[g].update({"clip_idx": clip_idx, "qweight": qweight, "qzeros": qzeros, "scales": scales,
                       "rows": rows, "weights_folded": W})
    return res


def save_layer_checkpoint(path: str, layer: int, res: dict) -> None:
    """Writes one layer's results atomically (temporary file, then rename)."""
    state = {"layer": layer}
    for g, _ in GROUPS:
        r = res[g]
        state[g] = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in r.items()
                    if k not in ("weights_folded", "abar")}
    _save_atomic(state, path)


def layer_checkpoint_path(ckpt_dir: str, layer: int) -> str:
    return os.path.join(ckpt_dir, f"layer_{layer:03d}.pt")


def state_checkpoint_path(ckpt_dir: str, layer: int) -> str:
    """The fp16 hidden state entering `layer`."""
    return os.path.join(ckpt_dir, f"hidden_{layer:03d}.pt")


def _save_atomic(obj, path: str) -> None:
    tmp = path + ".tmp"
    torch.save(obj, tmp)
    os.replace(tmp, path)


def finished_layers(ckpt_dir: str, layers) -> int:
    """How many of `layers` (in order) have a checkpoint: the driver resumes
    at the first one without."""
    n = 0
    for layer in layers:
        if not os.path.exists(layer_checkpoint_path(ckpt_dir, layer)):
            break
        n += 1
    return n


def quantize_layers(layers, get_weights, forward, x0: torch.Tensor, cfg: AwqConfig,
                    ckpt_dir: Optional[str] = None, resume: bool = False,
                    ws: Optional[torch.Tensor] = None) -> list:
    """Layer-by-layer AWQ of a decoder (the offline pass of "AWQ and
    Activation-Aware Scaling", Why this is attractive).  For each layer l of
    `layers` (consecutive, ascending): w = get_weights(l); caps, x_next =
    forward(x, w) captures the inputs of the four groups from the fp16 layer
    (the calibration states propagate through the unquantised model);
    quantize_layer_groups(caps, w, cfg) then searches, folds (w changes in
    place) and packs.  With ckpt_dir, after each layer the hidden state
    entering the next layer and then the layer's results are written, each
    atomically, so a layer's checkpoint implies the state after it.
    resume=True skips the layers that already have a checkpoint (from the
    first, consecutively) and restarts from the saved state after the last
    of them.  Returns one layer_summary per layer, the skipped ones read back
    from their checkpoints."""
    layers = list(layers)
    if any(b != a + 1 for a, b in zip(layers, layers[1:])):
        raise ValueError("layers must be consecutive and ascending")
    summaries = []
    start = 0
    x = x0
    if ckpt_dir is not None:
        os.makedirs(ckpt_dir, exist_ok=True)
        if resume:
            start = finished_layers(ckpt_dir, layers)
            for layer in layers[:start]:
                state = torch.load(layer_checkpoint_path(ckpt_dir, layer), weights_only=False)
                summaries.append(layer_summary(layer, state))
            if start == len(layers):
                return summaries
            if start > 0:
                x = torch.load(state_checkpoint_path(ckpt_dir, layers[start]),
                               weights_only=False).to(x0.device)
    for layer in layers[start:]:
        w = get_weights(layer)
        caps, x_next = forward(x, w)
        if ws is None:
            ws = workspace_for_layer(caps, w, cfg)
        res = quantize_layer_groups(caps, w, cfg, ws)
        summaries.append(layer_summary(layer, res))
        if ckpt_dir is not None:
            _save_atomic(x_next.cpu(), state_checkpoint_path(ckpt_dir, layer + 1))
            save_layer_checkpoint(layer_checkpoint_path(ckpt_dir, layer), layer, res)
        x = x_next
    return summaries


# ---------------------------------------------------------------------------
# Several GPUs: every layer's search is independent once its fp16 inputs are
# known (the calibration states propagate through the unmodified layers), so
# the layers split into contiguous blocks, one per rank, with no collective on
# the data path.  A rank computes the fp16 forward up to its first layer
# (input synthesis), then quantises its block.
# ---------------------------------------------------------------------------
def layer_block(rank: int, world: int, n_layers: int) -> range:
    """Contiguous block of layers of `rank` out of `world`: the first
    n_layers % world ranks take one layer more.  Blocks are disjoint, in
    order, and cover range(n_layers)."""
    if world < 1 or not 0 <= rank < world or n_layers < 0:
        raise ValueError(f"rank {rank} of {world}, {n_layers} layers")
    base, extra = divmod(n_layers, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def layer_summary(layer: int, res: dict) -> dict:
    """What a rank reports about one quantised layer: per group the selected
    alpha index, the smallest MSE and a checksum of the packed weights."""
    out = {"layer": layer}
    for g, _ in GROUPS:
        r = res[g]
        out[g] = {"best_idx": int(r["best_idx"].item()), "mse": float(r["mse"].min().item()),
                  "qweight_sum": int(r["qweight"].to(torch.int64).sum().item())}
    return out


def gather_summaries(summaries: list, dist=None) -> list:
    """All ranks' layer summaries, ordered by layer (an all_gather of Python
    objects over the process group; a single process returns its own)."""
    if dist is None:
        return sorted(summaries, key=lambda d: d["layer"])
    parts = [None] * dist.get_world_size()
    dist.all_gather_object(parts, summaries)
    return sorted((s for p in parts for s in p), key=lambda d: d["layer"])

