"""The allocation-free clip search (awq_search_clip_noalloc).

It exists for callers that cannot allocate device memory while the search
runs (a host framework that owns every device byte through its own arena, or
code that must not let a cudaMalloc synchronise the device mid-stream).  Its
scratch is a static device array inside the library.  This file is collected
last on purpose: if it fails, a run that stops at the first failure has
already run every other test.  It passes both alone and after the others."""

import ctypes

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from post_weight_quantization_awq_b200 import abi
from oracle import awq_oracle as O
from synthetic import random_layer

from gpu_helpers import MSE_RTOL, TIE_RTOL, need_cuda

pytestmark = pytest.mark.gpu


def _with_workspace(Xd, Wd, s, cfg):
    ws = awq.alloc_workspace(Xd.shape[0], Xd.shape[1], Wd.shape[0], cfg)
    idx = torch.empty((Wd.shape[0], Xd.shape[1] // 128), dtype=torch.uint8, device="cuda")
    err = torch.empty((Wd.shape[0], Xd.shape[1] // 128, cfg.n_clip), dtype=torch.float32, device="cuda")
    awq.awq_search_clip(Xd, Wd, s, cfg, ws, idx, err)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), err.cpu().numpy()


def test_noalloc_matches_workspace_entry_twice():
    need_cuda()
    T, inn, out = 3000, 1024, 256  # three token chunks with a workspace, two without
    X, W = random_layer(T, inn, out, seed=77)
    Xn = X.numpy()
    s_np = O.scale_grid(O.act_stats(Xn), O.alpha_grid(20))[9]
    Xd, Wd, s = X.cuda(), W.cuda(), torch.from_numpy(s_np).cuda()
    cfg = awq.AwqConfig.make(w_bit=4, n_clip=20)
    ref_idx, ref_err = _with_workspace(Xd, Wd, s, cfg)

    idx = torch.empty((out, inn // 128), dtype=torch.uint8, device="cuda")
    err = torch.empty((out, inn // 128, 20), dtype=torch.float32, device="cuda")
    free_before = None
    for call in range(2):
        idx.fill_(255)
        err.fill_(float("nan"))
        torch.cuda.synchronize()
        if call == 1:
            free_before = torch.cuda.mem_get_info()[0]
        # straight through the C ABI
        st = abi.LIB.awq_search_clip_noalloc(
            Xd.data_ptr(), T, inn, Xd.stride(0), Wd.data_ptr(), out, s.data_ptr(),
            ctypes.byref(cfg), idx.data_ptr(), err.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        assert st == 0, abi.last_error()
        torch.cuda.synchronize()
        got_idx, got_err = idx.cpu().numpy(), err.cpu().numpy()
        rel = np.abs(got_err - ref_err) / np.maximum(np.abs(ref_err), 1e-30)
        assert rel.max() <= MSE_RTOL, (call, rel.max())
        for o, k in zip(*np.nonzero(got_idx != ref_idx)):
            a, b = ref_err[o, k, got_idx[o, k]], ref_err[o, k, ref_idx[o, k]]
            assert abs(a - b) <= TIE_RTOL * abs(b), (call, o, k, a, b)
    # the second call took no device memory (the static scratch was set up by the first)
    assert torch.cuda.mem_get_info()[0] >= free_before


def test_noalloc_rejects_layers_beyond_its_static_scratch():
    cfg = awq.AwqConfig.make(n_clip=20)
    st = abi.LIB.awq_search_clip_noalloc(16, 256, 16384 + 128, 16384 + 128, 16, 64, None,
                                         ctypes.byref(cfg), 16, None, None)
    assert abi.STATUS[st] == "AWQ_ERR_INVALID_ARG"
    assert "16384" in abi.last_error()
