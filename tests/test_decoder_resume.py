"""Host logic of the layer-by-layer driver's checkpoints (decoder.quantize_layers)
on CPU, with the GPU search replaced by a deterministic stand-in: every layer
writes the hidden state entering the next layer and then its results, each
atomically; a rerun with resume=True skips the finished layers, restarts from
the saved state, and gives the same summaries as an uninterrupted run; a run
that stopped between the two writes of a layer redoes that layer."""

import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from post_weight_quantization_awq_b200 import decoder  # noqa: E402
from post_weight_quantization_awq_b200.abi import AwqConfig  # noqa: E402


class Fake:
    """forward: x -> x + layer weight; the 'search' result depends on the
    captured input, so a wrong restart state shows in the summaries."""

    def __init__(self):
        self.forwards = []
        self.searches = []

    def weights(self, layer):
        return {"w": torch.full((4,), float(layer + 1))}

    def forward(self, x, w):
        self.forwards.append(float(w["w"][0]))
        return {"qkv": x.clone()}, x + w["w"]

    def search(self, caps, weights, cfg, ws=None):
        x = caps["qkv"]
        self.searches.append(float(x.sum()))
        res = {}
        for g, _ in decoder.GROUPS:
            res[g] = {"best_idx": torch.tensor([int(x.sum()) % 20], dtype=torch.int32),
                      "mse": torch.tensor([float(x.sum()) + 0.5], dtype=torch.float64),
                      "qweight": x.to(torch.int32).reshape(1, -1)}
        return res


@pytest.fixture
def fake(monkeypatch):
    f = Fake()
    monkeypatch.setattr(decoder, "quantize_layer_groups", f.search)
    monkeypatch.setattr(decoder, "workspace_for_layer", lambda caps, w, cfg: torch.empty(1))
    return f


def _run(f, tmp, layers, resume):
    return decoder.quantize_layers(layers, f.weights, f.forward, torch.zeros(4), AwqConfig.make(),
                                   ckpt_dir=str(tmp), resume=resume)


def test_uninterrupted_run_writes_every_checkpoint(fake, tmp_path):
    out = _run(fake, tmp_path, range(5), resume=False)
    assert [s["layer"] for s in out] == list(range(5))
    assert fake.forwards == [1.0, 2.0, 3.0, 4.0, 5.0]
    for layer in range(5):
        assert os.path.exists(decoder.layer_checkpoint_path(str(tmp_path), layer))
        assert os.path.exists(decoder.state_checkpoint_path(str(tmp_path), layer + 1))
    assert not [n for n in os.listdir(tmp_path) if n.endswith(".tmp")]
    assert decoder.finished_layers(str(tmp_path), range(5)) == 5


def test_resume_skips_finished_layers(fake, tmp_path):
    ref = _run(Fake(), tmp_path / "ref", range(5), resume=False)
    # a run that finished layers 0..2
    _run(fake, tmp_path / "ck", range(3), resume=False)
    fake.forwards.clear()
    out = _run(fake, tmp_path / "ck", range(5), resume=True)
    assert fake.forwards == [4.0, 5.0]  # layers 3 and 4 only, from the saved state
    assert out == ref
    # everything done: nothing runs again
    fake.forwards.clear()
    assert _run(fake, tmp_path / "ck", range(5), resume=True) == ref
    assert fake.forwards == []


def test_stop_between_the_two_writes_redoes_the_layer(fake, tmp_path):
    ref = _run(Fake(), tmp_path / "ref", range(4), resume=False)
    _run(fake, tmp_path / "ck", range(4), resume=False)
    # as if the run stopped after writing the state after layer 2 but before
    # layer 2's results (and never reached layer 3)
    os.remove(decoder.layer_checkpoint_path(str(tmp_path / "ck"), 2))
    os.remove(decoder.layer_checkpoint_path(str(tmp_path / "ck"), 3))
    fake.forwards.clear()
    out = _run(fake, tmp_path / "ck", range(4), resume=True)
    assert fake.forwards == [3.0, 4.0]
    assert out == ref


def test_without_resume_every_layer_runs(fake, tmp_path):
    _run(fake, tmp_path, range(3), resume=False)
    fake.forwards.clear()
    _run(fake, tmp_path, range(3), resume=False)
    assert fake.forwards == [1.0, 2.0, 3.0]


def test_layers_must_be_consecutive(fake, tmp_path):
    with pytest.raises(ValueError):
        _run(fake, tmp_path, [0, 2], resume=False)


@pytest.mark.gpu
def test_resume_on_a_small_decoder(tmp_path):
    """Three layers of a small decoder of the same architecture (hidden 512,
    4 heads, MLP 1408, 8 x 128 calibration tokens) on the GPU: a run resumed
    after layer 1 packs the same bits as an uninterrupted one."""
    from gpu_helpers import need_cuda
    need_cuda()
    from synthetic import DecoderSpec, decoder_embeddings, decoder_layer_forward, decoder_layer_weights
    spec = DecoderSpec(hidden=512, heads=4, ffn=1408, layers=3, seq=128, n_seq=8)
    cfg = AwqConfig.make(w_bit=4, n_alpha=20, n_clip=20, clip_min=0.5)
    x0 = decoder_embeddings(spec, device="cuda")

    def get_w(layer):
        return decoder_layer_weights(spec, layer, device="cuda")

    def fwd(x, w):
        with torch.no_grad():
            return decoder_layer_forward(x, w, spec)

    ref = decoder.quantize_layers(range(3), get_w, fwd, x0, cfg)
    ck = str(tmp_path / "ck")
    decoder.quantize_layers(range(2), get_w, fwd, x0, cfg, ckpt_dir=ck)
    out = decoder.quantize_layers(range(3), get_w, fwd, x0, cfg, ckpt_dir=ck, resume=True)
    assert out == ref
    assert decoder.finished_layers(ck, range(3)) == 3
