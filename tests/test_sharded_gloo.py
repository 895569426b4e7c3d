"""Token sharding of one layer (post_weight_quantization_awq_b200.sharded) on
CPU: gloo ranks each hold a slice of the tokens (uneven, one rank possibly
empty) and the full W.  The per-shard calls are stand-ins written from the
oracle (the library's kernels need a GPU); the collectives and their order
are the product's.  Every rank must end with the single-process oracle
result: abar bit for bit, the same alpha, clip choices and packing."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

T, IN, OUT, N_ALPHA, N_CLIP = 90, 256, 16, 20, 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleShardOps:
    """The per-shard calls of sharded.LibraryShardOps, computed by the oracle
    in fp64 on CPU tensors."""

    device = torch.device("cpu")

    def workspace(self, T_local, inn, out, cfg):
        return None

    def act_sums(self, X, inn):
        units = np.abs(X.numpy().astype(np.float64)) * 2.0 ** 24  # integers (fp16 grid)
        return torch.from_numpy(units.astype(np.int64).sum(axis=0, dtype=np.int64))

    def act_finish(self, sums, T_total):
        return torch.from_numpy(sums.numpy().astype(np.float64) * 2.0 ** -24 / T_total)

    def search_sse(self, X, W, abar, cfg, ws):
        from oracle import awq_oracle as O
        Xn, Wn = X.numpy().astype(np.float64), W.numpy()
        S = O.scale_grid(abar.numpy(), O.alpha_grid(cfg.n_alpha))
        sse = np.zeros(cfg.n_alpha)
        for i in range(cfg.n_alpha):
            d = O.effective_error(Wn, S[i], O.quantize_groups(Wn, S[i], cfg.group_size, cfg.w_bit)["deq"])
            sse[i] = float(np.sum((Xn @ d.T) ** 2))
        return torch.from_numpy(sse)

    def select(self, sse, T_total, out, abar, cfg, ws):
        from oracle import awq_oracle as O
        mse = sse.numpy() / (T_total * out)
        best = int(np.argmin(mse))
        s = O.scale_grid(abar.numpy(), O.alpha_grid(cfg.n_alpha))[best]
        return torch.from_numpy(s.copy()), torch.from_numpy(mse), torch.tensor([best], dtype=torch.int32)

    def block_grams(self, X, inn, cfg, ws):
        from oracle import awq_oracle as O
        if X.shape[0] == 0:
            return torch.zeros((inn // 128, 128, 128), dtype=torch.float64)
        return torch.from_numpy(np.stack(O.block_grams(X.numpy(), 128)))

    def clip_from_grams(self, W, s, G, cfg, ws):
        from oracle import awq_oracle as O
        idx, _ = O.search_clip(None, W.numpy(), s.numpy(), cfg.w_bit, 128, cfg.n_clip, cfg.clip_min,
                               Gk=list(G.numpy()))
        return torch.from_numpy(idx)

    def pack(self, W, s, clip_idx, cfg):
        from oracle import awq_oracle as O
        qw, qz, sc = O.quant_pack(W.numpy(), s.numpy(), None if clip_idx is None else clip_idx.numpy(),
                                  cfg.w_bit, cfg.group_size, max(cfg.n_clip, 1), cfg.clip_min)
        return torch.from_numpy(qw), torch.from_numpy(qz), torch.from_numpy(sc)


def _layer():
    sys.path.insert(0, ROOT)
    from synthetic import random_layer
    return random_layer(T, IN, OUT, seed=31)


def _rank_main(rank, world, port, bounds, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    from post_weight_quantization_awq_b200 import AwqConfig
    from post_weight_quantization_awq_b200.sharded import quantize_layer_sharded
    from test_sharded_gloo import OracleShardOps

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    X, W = _layer()
    lo, hi = bounds[rank], bounds[rank + 1]
    cfg = AwqConfig.make(w_bit=4, n_alpha=N_ALPHA, n_clip=N_CLIP)
    r = quantize_layer_sharded(X[lo:hi], W, cfg, ops=OracleShardOps())
    dist.destroy_process_group()
    q.put((rank, r.abar.numpy(), r.mse.numpy(), int(r.best_idx[0]), r.s_best.numpy(),
           r.clip_idx.numpy(), r.qweight.numpy(), r.qzeros.numpy(), r.scales.numpy()))


@pytest.mark.parametrize("bounds", [(0, 37, T), (0, 50, 50, T)])
def test_token_sharded_layer_matches_single_process_oracle(bounds):
    from oracle import awq_oracle as O
    world = len(bounds) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, bounds, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    X, W = _layer()
    Xn, Wn = X.numpy(), W.numpy()
    abar = O.act_stats(Xn)
    mse, best, s, _ = O.search_scale(Xn, Wn, abar, 4, 128, N_ALPHA, form="direct")
    idx, _ = O.search_clip(Xn, Wn, s, 4, 128, N_CLIP, 0.5)
    qw, qz, sc = O.quant_pack(Wn, s, idx, 4, 128, N_CLIP, 0.5)
    for rank, g_abar, g_mse, g_best, g_s, g_idx, g_qw, g_qz, g_sc in res:
        assert np.array_equal(g_abar, abar), rank
        assert np.allclose(g_mse, mse, rtol=1e-12, atol=0), rank
        assert g_best == best and np.array_equal(g_s, s), rank
        assert np.array_equal(g_idx, idx), rank
        assert np.array_equal(g_qw, qw) and np.array_equal(g_qz, qz), rank
        assert np.array_equal(g_sc.view(np.uint16), sc.view(np.uint16)), rank
