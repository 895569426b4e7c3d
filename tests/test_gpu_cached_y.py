"""GPU parity of the cached-output scoring form (search_form = 2): the literal
reading of "05 — AWQ: Activation-Aware Weight Scaling" §4, which measures each
candidate's output against the fp16 output X W^T.  Y = RN16(X W^T) is computed
once; the candidate GEMM multiplies X by RN16(Qdeq/s) and its epilogue
subtracts the cached Y tile and sums the squares.

The oracle for this form is its own definition (mse_fp16_output: the same two
fp16 roundings, everything else in fp64); bars as elsewhere: per-alpha MSE
within 1e-3, the same selection unless tied within 1e-4.  Against the exact
score the roundings' cross term shrinks like 1/sqrt(T out): at the full
q_proj size the form agrees with the error form within the same bar."""

import numpy as np
import pytest

import post_weight_quantization_awq_b200 as awq
from oracle import awq_oracle as O
from synthetic import random_layer, workload_inputs

from gpu_helpers import MSE_RTOL, check_mse, check_selection, gpu_search, need_cuda

pytestmark = pytest.mark.gpu

CACHED_Y = awq.abi.SEARCH_CACHED_Y


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


@pytest.mark.parametrize("T,inn,out,w_bit,group,zp", [
    (64, 128, 16, 4, 128, 1), (1, 128, 8, 4, 128, 1), (200, 384, 264, 3, 128, 1),
    (256, 512, 512, 4, 128, 1), (2125, 1024, 768, 4, 128, 1), (300, 256, 72, 4, 32, 1),
    (500, 640, 136, 4, 128, 0)])
def test_search_scale_cached_output_form(T, inn, out, w_bit, group, zp):
    X, W = random_layer(T, inn, out, seed=T * 3 + inn + out)
    cfg = awq.AwqConfig.make(w_bit=w_bit, group_size=group, zero_point=zp, search_form=CACHED_Y)
    g = gpu_search(X, W, cfg)
    Xn, Wn = X.numpy(), W.numpy()
    mse, _, _, S = O.search_scale(Xn, Wn, O.act_stats(Xn), w_bit, group, 20, form="fp16_output",
                                  zero_point=bool(zp))
    check_mse(g["mse"], mse)
    check_selection(g["best"], mse, "alpha (cached output)")
    assert np.array_equal(g["s_best"], S[g["best"]])


def test_cached_output_form_matches_direct_form_full_q_proj():
    """Full q_proj workload (T = 65536, in = out = 4096): the cached-output
    form agrees with the error form within the MSE bar and picks the same
    alpha unless tied within 1e-4."""
    d = workload_inputs(1)
    _, X, W = d["groups"][0]
    a = gpu_search(X, W, awq.AwqConfig.make())
    b = gpu_search(X, W, awq.AwqConfig.make(search_form=CACHED_Y))
    rel = np.abs(a["mse"] - b["mse"]) / a["mse"]
    assert rel.max() <= MSE_RTOL, rel.max()
    check_selection(b["best"], a["mse"], "alpha (cached output vs direct)")
