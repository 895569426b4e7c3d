"""The fused form of the alpha search (AWQ_SEARCH_FUSED): the scored GEMM
builds each candidate's B tile in shared memory from the W rows and
per-group parameters instead of reading a stored operand.  Its tiles hold the
direct form's operand values and its epilogue and tile order are the direct
form's, so the per-alpha MSE, the selection and s* must come out bit for bit
the same as AWQ_SEARCH_DIRECT's; and against the oracle, the usual bars (MSE
within 1e-3, the same alpha unless tied within 1e-4, s* bit-exact)."""

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O
from synthetic import edge_layer, random_layer, workload_inputs

from gpu_helpers import check_mse, check_selection, gpu_search, need_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


def _both(X, W, **kw):
    d = gpu_search(X, W, awq.AwqConfig.make(**kw))
    f = gpu_search(X, W, awq.AwqConfig.make(search_form=awq.abi.SEARCH_FUSED, **kw))
    assert np.array_equal(f["mse"].view(np.uint64), d["mse"].view(np.uint64)), (f["mse"], d["mse"])
    assert f["best"] == d["best"]
    assert np.array_equal(f["s_best"].view(np.uint32), d["s_best"].view(np.uint32))
    return f


@pytest.mark.parametrize("T,inn,out,w_bit,group,zp", [
    (64, 128, 16, 4, 128, 1),      # one tile, padded rows (out_pad 256)
    (300, 384, 264, 3, 128, 1),    # ragged T and out, INT3
    (2125, 1024, 768, 4, 128, 1),  # several M and N tiles
    (1000, 512, 520, 4, 64, 1),    # groups of 64
    (700, 512, 136, 4, 32, 1),     # groups of 32: two groups per 64-channel slice
    (900, 640, 264, 4, 128, 0),    # no zero point
    (1, 128, 8, 4, 128, 1),        # a single token
])
def test_fused_form_is_bitwise_the_direct_form(T, inn, out, w_bit, group, zp):
    X, W = random_layer(T, inn, out, seed=T + inn + out)
    f = _both(X, W, w_bit=w_bit, group_size=group, zero_point=zp)
    Xn, Wn = X.numpy(), W.numpy()
    mse, _, _, S = O.search_scale(Xn, Wn, O.act_stats(Xn), w_bit, group, 20, zero_point=bool(zp))
    check_mse(f["mse"], mse)
    check_selection(f["best"], mse, "alpha (fused form)")
    assert np.array_equal(f["s_best"], S[f["best"]])


@pytest.mark.parametrize("zp", [1, 0])
def test_fused_form_on_edge_groups(zp):
    """One-signed narrow groups (the exact-division path and the clamped zero
    points), constant groups and dead channels: the fused converters take the
    same branches as the candidate kernel."""
    X, W = edge_layer(600, 512, 264, seed=77)
    _both(X, W, zero_point=zp)


def test_fused_form_full_q_proj():
    """The q_proj workload at full size (X [65536 x 4096], W [4096 x 4096], 20
    alphas): the same bits as the direct form."""
    d = workload_inputs(1)
    _, X, W = d["groups"][0]
    _both(X, W)
