"""GPU parity of the full-size workloads, every output row, against the
oracle: the Llama-7B-shaped MLP (gate|up jointly scaled, and down_proj on its
SwiGLU input, T = 65536) and the Llama-13B-shaped INT3 attention block (q|k|v
jointly scaled and o_proj on its own input, T = 65536, 20 alphas + 20 clip
ratios).  The whole path runs as quantize_layer runs it: abar and s bit-exact,
per-alpha MSE within 1e-3, the same alpha and clip choices unless tied within
1e-4, qweight / qzeros / scales bit-exact.  (The q_proj workload is in
test_gpu_parity.py, the 32-layer decoder in test_gpu_decoder.py.)"""

import pytest

from synthetic import workload_inputs

from gpu_helpers import layer_parity, need_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()


@pytest.fixture(scope="module")
def mlp():
    need_cuda()  # module fixtures run before the per-test skip
    return workload_inputs(2, device="cuda")["groups"]


@pytest.fixture(scope="module")
def attention():
    need_cuda()
    return workload_inputs(3)["groups"]


def test_mlp_gate_up_full(mlp):
    """gate|up [22016 x 4096] on X [65536 x 4096], INT4, 20 alphas."""
    _, X, W = mlp[0]
    layer_parity(X, W, 4, 20, 0)


def test_mlp_down_proj_full(mlp):
    """down_proj [4096 x 11008] on the SwiGLU input [65536 x 11008]."""
    _, X, W = mlp[1]
    layer_parity(X.cpu(), W, 4, 20, 0)


def test_attention_qkv_int3_full(attention):
    """q|k|v [15360 x 5120] on X [65536 x 5120], INT3, 20 alphas + 20 clip
    ratios, packed."""
    _, X, W = attention[0]
    layer_parity(X, W, 3, 20, 20)


def test_attention_o_proj_int3_full(attention):
    """o_proj [5120 x 5120] on its own input X_o [65536 x 5120], INT3, 20
    alphas + 20 clip ratios, packed."""
    _, X, W = attention[1]
    layer_parity(X, W, 3, 20, 20)
