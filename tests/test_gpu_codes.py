"""GPU parity of the candidate codes, code for code.

The alpha search's candidate quantiser (awq_candidate_codes: the kernel that
builds the scored operand, in its inspection form) and the clip search's
producers (awq_clip_candidate_codes) quantise with a batched fast path: an
approximate reciprocal proposes each code, one remainder test per 8 values
proves it, a group bound sends groups with large quotients to the correctly
rounded division.  Here every candidate's codes, zero points and steps are
compared bit for bit with the oracle's quantize_groups ("05 — AWQ" §4: for each
alpha apply the scaling and quantize; §5: codes, zero points, fp16 scales),
including layers built to take the exact fallback, the one-signed clamps and
the constant-group guard (synthetic.edge_layer)."""

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O
from synthetic import edge_layer, random_layer, workload_inputs

from gpu_helpers import need_cuda, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


def gpu_candidate_codes(W, abar, cfg):
    Wd = to_dev(W)
    out, inn = Wd.shape
    g = cfg.group_size
    ws = awq.alloc_workspace(1, inn, out, cfg)
    q = torch.empty((cfg.n_alpha, out, inn), dtype=torch.uint8, device="cuda")
    z = torch.empty((cfg.n_alpha, out, inn // g), dtype=torch.uint8, device="cuda")
    d = torch.empty((cfg.n_alpha, out, inn // g), dtype=torch.float32, device="cuda")
    awq.awq_candidate_codes(Wd, torch.from_numpy(abar).cuda(), cfg, ws, q, z, d)
    awq.awq_device_status(ws)
    return q.cpu().numpy(), z.cpu().numpy(), d.cpu().numpy()


def check_candidate_codes(X, W, cfg, alphas=None):
    Xn, Wn = X.numpy(), W.numpy()
    abar = O.act_stats(Xn)
    S = O.scale_grid(abar, O.alpha_grid(cfg.n_alpha))
    q, z, d = gpu_candidate_codes(W, abar, cfg)
    for i in (range(cfg.n_alpha) if alphas is None else alphas):
        ref = O.quantize_groups(Wn, S[i], cfg.group_size, cfg.w_bit, zero_point=bool(cfg.zero_point))
        bad = np.argwhere(q[i] != ref["q"])
        assert bad.size == 0, (i, bad[:5], q[i][tuple(bad[0])], ref["q"][tuple(bad[0])])
        assert np.array_equal(z[i], ref["z"]), i
        assert np.array_equal(d[i].view(np.uint32), ref["delta"].view(np.uint32)), i


@pytest.mark.parametrize("T,inn,out,w_bit,group,zp", [
    (64, 128, 16, 4, 128, 1), (200, 384, 264, 3, 128, 1), (300, 256, 72, 4, 32, 1),
    (257, 512, 520, 4, 64, 1), (500, 640, 136, 4, 128, 0), (128, 192, 24, 3, 64, 0)])
def test_candidate_codes_bitwise(T, inn, out, w_bit, group, zp):
    X, W = random_layer(T, inn, out, seed=T + inn + out + group)
    check_candidate_codes(X, W, awq.AwqConfig.make(w_bit=w_bit, group_size=group, zero_point=zp))


@pytest.mark.parametrize("w_bit,group,zp", [(4, 128, 1), (3, 128, 1), (4, 32, 1), (4, 64, 0),
                                            (3, 128, 0)])
def test_candidate_codes_edge_layer(w_bit, group, zp):
    """One-signed narrow groups (the group bound fails, the exact division
    decides, z clamps to 0 or 2^b - 1), constant and all-zero groups (the
    1e-5 range floor, under the search's 2^k scaling), fp16-subnormal weights,
    and dead input channels (s at the 1e-4 floor)."""
    X, W = edge_layer(200, 4 * 128, 264, seed=w_bit * 10 + group + zp, group=group)
    check_candidate_codes(X, W, awq.AwqConfig.make(w_bit=w_bit, group_size=group, zero_point=zp))


def test_candidate_codes_full_q_proj():
    """All 20 candidates of the Llama-7B-shaped q_proj layer (4096 x 4096)."""
    d = workload_inputs(1)
    _, X, W = d["groups"][0]
    check_candidate_codes(X, W, awq.AwqConfig.make())


# ------------------------------------------------------------------ clip producers
def gpu_clip_codes(X, W, s, cfg):
    Xd, Wd = to_dev(X), to_dev(W)
    T, inn = Xd.shape
    out = Wd.shape[0]
    ws = awq.alloc_workspace(T, inn, out, cfg)
    G = torch.empty((inn // 128, 128, 128), dtype=torch.float32, device="cuda")
    awq.awq_block_grams(Xd, cfg, ws, G)
    g = cfg.group_size
    idx = torch.empty((out, inn // g), dtype=torch.uint8, device="cuda")
    q = torch.empty((out, cfg.n_clip, inn), dtype=torch.uint8, device="cuda")
    z = torch.empty((out, cfg.n_clip, inn // g), dtype=torch.uint8, device="cuda")
    sd = None if s is None else torch.from_numpy(s).cuda()
    awq.awq_clip_candidate_codes(Wd, sd, G, cfg, ws, idx, None, q, z)
    awq.awq_device_status(ws)
    # the plain search gives the same selection
    idx2 = torch.empty_like(idx)
    awq.awq_search_clip_grams(Wd, sd, G, cfg, ws, idx2)
    awq.awq_device_status(ws)
    assert torch.equal(idx, idx2)
    return q.cpu().numpy(), z.cpu().numpy()


def check_clip_codes(X, W, s, cfg):
    q, z = gpu_clip_codes(X, W, s, cfg)
    Wn = W.numpy()
    out, inn = Wn.shape
    g = cfg.group_size
    r = O.clip_ratios(cfg.n_clip, cfg.clip_min).astype(np.float32)
    for c in range(cfg.n_clip):
        ratio = np.full((out, inn // g), r[c], dtype=np.float32)
        ref = O.quantize_groups(Wn, s, g, cfg.w_bit, ratio, zero_point=bool(cfg.zero_point))
        bad = np.argwhere(q[:, c, :] != ref["q"])
        assert bad.size == 0, (c, bad[:5])
        assert np.array_equal(z[:, c, :], ref["z"]), c


@pytest.mark.parametrize("T,inn,out,w_bit,n_clip,zp,group", [
    (300, 256, 40, 4, 20, 1, 128), (64, 128, 8, 3, 7, 1, 128), (500, 512, 96, 3, 20, 1, 128),
    (100, 384, 24, 4, 1, 1, 128), (200, 256, 72, 4, 20, 0, 128), (300, 256, 40, 4, 20, 1, 32),
    (200, 384, 72, 3, 20, 0, 64)])
def test_clip_candidate_codes_bitwise(T, inn, out, w_bit, n_clip, zp, group):
    X, W = random_layer(T, inn, out, seed=T + out + n_clip)
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[10]
    cfg = awq.AwqConfig.make(w_bit=w_bit, n_clip=n_clip, zero_point=zp, group_size=group)
    check_clip_codes(X, W, s, cfg)
    check_clip_codes(X, W, None, cfg)


@pytest.mark.parametrize("w_bit,zp,group", [(4, 1, 128), (3, 1, 128), (4, 0, 128), (4, 1, 32),
                                            (3, 0, 64)])
def test_clip_candidate_codes_edge_layer(w_bit, zp, group):
    X, W = edge_layer(300, 4 * 128, 136, seed=40 + w_bit + zp, group=group)
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[15]
    check_clip_codes(X, W, s, awq.AwqConfig.make(w_bit=w_bit, n_clip=20, zero_point=zp,
                                                 group_size=group))


def test_clip_candidate_codes_q_proj_rows():
    """Clip candidates of the q_proj layer at full in = 4096, on 512 rows, with
    the s of its 13th alpha."""
    d = workload_inputs(1, T=8192)
    _, X, W = d["groups"][0]
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[13]
    check_clip_codes(X, W[:512].contiguous(), s, awq.AwqConfig.make(n_clip=20))
