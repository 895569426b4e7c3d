"""The debug library (libawq_debug.so: the same kernels compiled with index
checks on the global accesses whose indices they derive from their grids)
runs every C-ABI call on ragged shapes (tests/debug_bounds_battery.py):
no check fails, and every result is bit-identical to the release library's.
Each library runs in its own child process (the binding loads one library
per process)."""

import os
import subprocess
import sys

import pytest
import torch

from gpu_helpers import need_cuda

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG_LIB = os.path.join(os.path.dirname(HERE), "post_weight_quantization_awq_b200", "libawq_debug.so")


def _run(tmp_path, debug):
    out = str(tmp_path / ("debug.pt" if debug else "release.pt"))
    env = dict(os.environ)
    if debug:
        env["AWQ_LIB"] = "debug"
    else:
        env.pop("AWQ_LIB", None)
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_battery.py"), out], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    return torch.load(out, weights_only=False)


def _equal(a, b, path="res"):
    if isinstance(a, dict):
        assert a.keys() == b.keys(), path
        for k in a:
            _equal(a[k], b[k], f"{path}.{k}")
    elif isinstance(a, torch.Tensor):
        assert a.dtype == b.dtype and a.shape == b.shape, path
        assert torch.equal(a.view(torch.uint8) if a.dtype.is_floating_point else a,
                           b.view(torch.uint8) if b.dtype.is_floating_point else b), path
    else:
        assert a == b, path


def test_debug_library_checks_pass_and_match_release(tmp_path):
    need_cuda()
    if not os.path.exists(DEBUG_LIB):
        pytest.skip("libawq_debug.so not built")
    dbg = _run(tmp_path, debug=True)
    rel = _run(tmp_path, debug=False)
    assert dbg["bounds"]["enabled"] and not rel["bounds"]["enabled"]
    assert dbg["bounds"]["ok"], dbg["bounds"]["message"]
    for k in rel:
        if k != "bounds":
            _equal(dbg[k], rel[k], k)
