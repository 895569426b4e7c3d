"""Runs one call of the library on a seeded synthetic layer, for profiling
(ncu) and quick timing.

    python -m post_weight_quantization_awq_b200.run_case --op search --tokens 16384 \
        --in 4096 --out 4096 [--alphas 20] [--clips 20] [--bits 4] [--repeat 3] [--form gram|cached_y|fused]

--op is one of: stats, search, clip, pack, layer (all four calls), w4a16 (the
GEMM on the packed output, Y = X Wd^T with Wd = RN16((q - z) scale); with
--w4a16-form fused the weights are dequantised tile by tile inside the GEMM).  Inputs
follow the heavy-tailed recipe of the synthetic module (1% outlier channels
x U[20, 50], W ~ N(0, 0.02)).  Prints the CUDA-event time of the last repeat.
"""

from __future__ import annotations

import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None) -> int:
    import torch

    import post_weight_quantization_awq_b200 as awq
    from synthetic import OutlierSpec, gaussian_weight, heavy_tailed_activations

    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=("stats", "search", "clip", "pack", "layer", "w4a16"), required=True)
    ap.add_argument("--tokens", type=int, default=16384)
    ap.add_argument("--in", dest="inn", type=int, default=4096)
    ap.add_argument("--out", type=int, default=4096)
    ap.add_argument("--alphas", type=int, default=20)
    ap.add_argument("--clips", type=int, default=20)
    ap.add_argument("--bits", type=int, default=4)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--form", choices=("direct", "gram", "cached_y", "fused"), default="direct",
                    help="alpha-search scoring form")
    ap.add_argument("--w4a16-form", choices=("auto", "fused"), default="auto",
                    help="auto: the workspace awq_w4a16_workspace_size asks for (dequantise once "
                         "for many tokens, split-K for few); fused: 256 bytes (dequantise per tile)")
    a = ap.parse_args(argv)

    X = heavy_tailed_activations(a.tokens, a.inn, OutlierSpec(0.01, 20.0, 50.0), a.seed).cuda()
    W = gaussian_weight(a.out, a.inn, a.seed).cuda()
    cfg = awq.AwqConfig.make(w_bit=a.bits, n_alpha=a.alphas, n_clip=a.clips,
                             search_form={"direct": awq.abi.SEARCH_DIRECT, "gram": awq.abi.SEARCH_GRAM,
                                          "cached_y": awq.abi.SEARCH_CACHED_Y,
                                          "fused": awq.abi.SEARCH_FUSED}[a.form])
    ws = awq.alloc_workspace(a.tokens, a.inn, a.out, cfg)
    abar = torch.empty(a.inn, dtype=torch.float64, device="cuda")
    mse = torch.empty(a.alphas, dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")
    s_best = torch.ones(a.inn, dtype=torch.float32, device="cuda")
    clip_idx = torch.zeros((a.out, a.inn // 128), dtype=torch.uint8, device="cuda")
    g = 128
    qw = torch.empty((a.inn, a.out // 8), dtype=torch.int32, device="cuda")
    qz = torch.empty((a.inn // g, a.out // 8), dtype=torch.int32, device="cuda")
    sc = torch.empty((a.inn // g, a.out), dtype=torch.float16, device="cuda")
    awq.awq_act_stats(X, abar)
    if a.op == "w4a16":
        awq.awq_quant_pack(W, s_best, None, cfg, qw, qz, sc)
        Y = torch.empty((a.tokens, a.out), dtype=torch.float16, device="cuda")
        nws = 256 if a.w4a16_form == "fused" else awq.awq_w4a16_workspace_size(a.tokens, a.inn, a.out, cfg)
        ws16 = torch.empty(nws, dtype=torch.uint8, device="cuda")

    def once():
        if a.op == "stats":
            awq.awq_act_stats(X, abar)
        elif a.op == "search":
            awq.awq_search_scale(X, W, abar, cfg, ws, s_best, mse, best)
        elif a.op == "clip":
            awq.awq_search_clip(X, W, s_best, cfg, ws, clip_idx)
        elif a.op == "pack":
            awq.awq_quant_pack(W, s_best, clip_idx if a.clips else None, cfg, qw, qz, sc)
        elif a.op == "w4a16":
            awq.awq_w4a16_gemm(X, qw, qz, sc, cfg, Y, ws16)
        else:
            awq.quantize_layer(X, W, cfg, ws=ws)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(a.repeat):
        e0.record()
        once()
        e1.record()
    torch.cuda.synchronize()
    awq.awq_device_status(ws)
    ms = e0.elapsed_time(e1)
    extra = ""
    if a.op == "w4a16":
        extra = f", {2.0 * a.tokens * a.inn * a.out / (ms * 1e-3) / 1e12:.1f} TFLOP/s"
    print(f"{a.op}: T={a.tokens} in={a.inn} out={a.out} last call {ms:.3f} ms{extra}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
