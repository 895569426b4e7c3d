"""Runs every C-ABI call of the library on ragged shapes and saves the results
(imported by test_gpu_debug_bounds.py, which runs it once with the debug
library, AWQ_LIB=debug, and once with the release library in child
processes).  Usage: python tests/debug_bounds_battery.py OUT.pt"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import post_weight_quantization_awq_b200 as awq  # noqa: E402
from synthetic import edge_layer, random_layer  # noqa: E402


def _packed(rng_seed, inn, out, group):
    g = torch.Generator().manual_seed(rng_seed)
    qw = torch.randint(-2 ** 31, 2 ** 31 - 1, (inn, out // 8), generator=g, dtype=torch.int64).to(torch.int32)
    qz = torch.randint(-2 ** 31, 2 ** 31 - 1, (inn // group, out // 8), generator=g,
                       dtype=torch.int64).to(torch.int32)
    sc = (torch.rand((inn // group, out), generator=g) * 0.1 + 0.01).half()
    return qw.cuda(), qz.cuda(), sc.cuda()


def run(out_path: str) -> None:
    res = {}
    # the whole path (stats, alpha search, clip search, packing) in every scoring
    # form (direct, Gram, cached output, fused), with and without a zero point,
    # at the three group sizes
    cases = [(300, 384, 136, 4, 128, 1, 0), (4173, 512, 264, 3, 128, 1, 1), (257, 256, 72, 4, 32, 1, 2),
             (1000, 640, 520, 4, 64, 0, 0), (600, 512, 264, 4, 128, 1, 1), (700, 512, 136, 4, 32, 1, 3)]
    for i, (T, inn, out, w_bit, group, zp, form) in enumerate(cases):
        X, W = (edge_layer if i == 4 else random_layer)(T, inn, out, seed=100 + i, **(
            {"group": group} if i == 4 else {}))
        cfg = awq.AwqConfig.make(w_bit=w_bit, group_size=group, zero_point=zp, n_clip=20,
                                 search_form=form)
        r = awq.quantize_layer(X.cuda(), W.cuda(), cfg)
        torch.cuda.synchronize()
        res[f"layer{i}"] = {k: getattr(r, k).cpu() for k in
                            ("abar", "mse", "best_idx", "s_best", "clip_idx", "qweight", "qzeros", "scales")}
        # the allocation-free clip search and the inspection forms on the same layer
        Xd, Wd = X.cuda(), W.cuda()
        idx = torch.empty_like(r.clip_idx)
        awq.awq_search_clip_noalloc(Xd, Wd, r.s_best, cfg, idx)
        awq.awq_device_status(None)
        res[f"noalloc{i}"] = idx.cpu()
    # the alpha search in the smallest workspace (candidates one at a time)
    X, W = random_layer(2125, 512, 264, seed=7)
    cfg = awq.AwqConfig.make()
    ws = torch.empty(awq.awq_workspace_size_min(2125, 512, 264, cfg), dtype=torch.uint8, device="cuda")
    r = awq.quantize_layer(X.cuda(), W.cuda(), cfg, ws=ws)
    res["small_ws"] = {"mse": r.mse.cpu(), "qweight": r.qweight.cpu()}
    # token-sharded parts on one GPU
    sums = torch.zeros(512, dtype=torch.int64, device="cuda")
    awq.awq_act_sums(X.cuda()[:1000], sums)
    abar = torch.empty(512, dtype=torch.float64, device="cuda")
    awq.awq_act_stats_finish(sums, 1000, abar)
    ws = awq.alloc_workspace(1000, 512, 264, cfg)
    sse = torch.empty(20, dtype=torch.float64, device="cuda")
    awq.awq_search_scale_sse(X.cuda()[:1000], W.cuda(), abar, cfg, ws, sse)
    G = torch.empty((4, 128, 128), dtype=torch.float32, device="cuda")
    awq.awq_block_grams(X.cuda()[:1000], cfg, ws, G)
    awq.awq_device_status(ws)
    res["sharded"] = {"sums": sums.cpu(), "sse": sse.cpu(), "G": G.cpu()}
    # the W4A16 product in every form: decode (1, 5 tokens), split-K (100),
    # dequantise once (1100), fused (100 with a 256-byte workspace)
    for (T, inn, out, group) in [(1, 512, 288, 128), (5, 1024, 544, 32), (100, 512, 288, 64),
                                 (1100, 512, 544, 128)]:
        qw, qz, sc = _packed(T + inn, inn, out, group)
        Xh = (torch.randn(T, inn, generator=torch.Generator().manual_seed(T)) * 0.5).half().cuda()
        cfg = awq.AwqConfig.make(group_size=group)
        for name, n in (("auto", awq.awq_w4a16_workspace_size(T, inn, out, cfg)), ("fused", 256)):
            Y = torch.empty((T, out), dtype=torch.float16, device="cuda")
            wsq = torch.empty(n, dtype=torch.uint8, device="cuda")
            awq.awq_w4a16_gemm(Xh, qw, qz, sc, cfg, Y, wsq)
            awq.awq_device_status(wsq)
            res[f"w4a16_{T}_{name}"] = Y.cpu()
    # the fold
    gen = torch.Generator().manual_seed(3)
    v = (torch.randn(264, 512, generator=gen) * 0.02).half().cuda()
    awq.awq_fold_inv_scale(v, (torch.rand(264, generator=gen) + 0.5).cuda())
    res["fold"] = v.cpu()
    torch.cuda.synchronize()
    bounds_ok = True
    message = ""
    try:
        awq.awq_bounds_status()
    except awq.AwqError as e:
        bounds_ok, message = False, str(e)
    res["bounds"] = {"enabled": awq.awq_bounds_checks_enabled(), "ok": bounds_ok, "message": message}
    torch.save(res, out_path)


if __name__ == "__main__":
    run(sys.argv[1])
