"""Host logic of the decoder's layer sharding on CPU: the 32 layers split into
contiguous per-rank blocks (every layer's search is independent once its fp16
inputs are known), and the per-layer summaries of world-size-2 and -3 gloo
ranks gather into one ordered list on every rank."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from post_weight_quantization_awq_b200 import decoder  # noqa: E402


@pytest.mark.parametrize("n_layers", [0, 1, 5, 32, 33])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8, 40])
def test_layer_blocks_partition_the_layers(n_layers, world):
    blocks = [decoder.layer_block(r, world, n_layers) for r in range(world)]
    flat = [layer for b in blocks for layer in b]
    assert flat == list(range(n_layers))              # disjoint, in order, complete
    sizes = [len(b) for b in blocks]
    assert max(sizes) - min(sizes) <= 1               # balanced
    assert sizes == sorted(sizes, reverse=True)       # the larger blocks come first


def test_layer_block_rejects_bad_ranks():
    for args in ((2, 2, 32), (-1, 2, 32), (0, 0, 32), (0, 2, -1)):
        with pytest.raises(ValueError):
            decoder.layer_block(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, n_layers, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from post_weight_quantization_awq_b200 import decoder as dec
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # stand-in summaries: what a rank would report for the layers it owns
    mine = [{"layer": layer, "qkv": {"best_idx": layer % 20, "rank": rank}}
            for layer in dec.layer_block(rank, world, n_layers)]
    got = dec.gather_summaries(mine, dist)
    dist.destroy_process_group()
    q.put((rank, got))


@pytest.mark.parametrize("world", [2, 3])
def test_summaries_gather_over_gloo_ranks(world):
    n_layers = 32
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, n_layers, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        got = res[rank]
        assert [d["layer"] for d in got] == list(range(n_layers))
        for d in got:  # each layer came from the rank whose block holds it
            assert d["layer"] in decoder.layer_block(d["qkv"]["rank"], world, n_layers)
    assert all(res[r] == res[0] for r in range(world))
