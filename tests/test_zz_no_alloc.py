"""The allocation-free clip search (awq_search_clip_noalloc).

It exists for callers that cannot allocate device memory while the search
runs (a host framework that owns every device byte through its own arena, or
code that must not let a cudaMalloc synchronise the device mid-stream).  Its
scratch is a static device array inside the library.  This file is collected
last on purpose: if it fails, a run that stops at the first failure has
already run every other test.  It passes both alone and after the others."""

import ctypes
import gc

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


def _noalloc(Xd, Wd, s, cfg, idx, err):
    """One call straight through the C ABI."""
    st = abi.LIB.awq_search_clip_noalloc(
        Xd.data_ptr(), Xd.shape[0], Xd.shape[1], Xd.stride(0), Wd.data_ptr(), Wd.shape[0],
        s.data_ptr(), ctypes.byref(cfg), idx.data_ptr(), err.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == 0, abi.last_error()


def _clear_library_status():
    try:
        awq.awq_device_status(None)
    except awq.AwqError:
        pass


@pytest.mark.parametrize("T,inn,out,exact", [
    (3000, 1024, 256, True),    # three token chunks either way: identical results
    (8000, 8192, 64, False),    # five chunks in the static array, eight with a workspace
])
def test_noalloc_matches_workspace_entry_twice(T, inn, out, exact):
    need_cuda()
    _clear_library_status()
    X, W = random_layer(T, inn, out, seed=77 + inn)
    Xn = X.numpy()
    s_np = O.scale_grid(O.act_stats(Xn), O.alpha_grid(20))[9]
    Xd, Wd, s = X.cuda(), W.cuda(), torch.from_numpy(s_np).cuda()
    cfg = awq.AwqConfig.make(w_bit=4, n_clip=20)
    ref_idx, ref_err = _with_workspace(Xd, Wd, s, cfg)

    idx = torch.empty((out, inn // 128), dtype=torch.uint8, device="cuda")
    err = torch.empty((out, inn // 128, 20), dtype=torch.float32, device="cuda")
    for call in range(2):
        idx.fill_(255)
        err.fill_(float("nan"))
        gc.collect()
        torch.cuda.synchronize()
        before = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(),
                  torch.cuda.memory_reserved())
        _noalloc(Xd, Wd, s, cfg, idx, err)
        awq.awq_device_status(None)  # no device-side failure recorded
        after = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(),
                 torch.cuda.memory_reserved())
        # torch's allocator did not grow (the call allocates nothing through it;
        # unrelated tensors may be freed meanwhile); after the first call's
        # set-up, the device's free memory did not shrink either
        assert after[1] <= before[1] and after[2] <= before[2], (call, before, after)
        if call == 1:
            assert after[0] >= before[0], (before, after)
        got_idx, got_err = idx.cpu().numpy(), err.cpu().numpy()
        if exact:
            assert np.array_equal(got_idx, ref_idx)
            assert np.array_equal(got_err.view(np.uint32), ref_err.view(np.uint32))
            continue
        rel = np.abs(got_err - ref_err) / np.maximum(np.abs(ref_err), 1e-30)
        assert rel.max() <= MSE_RTOL, (call, rel.max())
        for o, k in zip(*np.nonzero(got_idx != ref_idx)):
            a, b = ref_err[o, k, got_idx[o, k]], ref_err[o, k, ref_idx[o, k]]
            assert abs(a - b) <= TIE_RTOL * abs(b), (call, o, k, a, b)


def test_noalloc_reports_a_timeout_and_recovers(monkeypatch):
    """With every bounded wait giving up at once (AWQ_FAULT=timeout), the call
    records AWQ_ERR_TIMEOUT in the library status word instead of returning
    stale Grams silently; the next call is correct."""
    need_cuda()
    _clear_library_status()
    T, inn, out = 2000, 512, 136
    X, W = random_layer(T, inn, out, seed=78)
    s_np = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[12]
    Xd, Wd, s = X.cuda(), W.cuda(), torch.from_numpy(s_np).cuda()
    cfg = awq.AwqConfig.make(n_clip=20)
    ref_idx, ref_err = _with_workspace(Xd, Wd, s, cfg)
    idx = torch.empty((out, inn // 128), dtype=torch.uint8, device="cuda")
    err = torch.empty((out, inn // 128, 20), dtype=torch.float32, device="cuda")
    monkeypatch.setenv("AWQ_FAULT", "timeout")
    _noalloc(Xd, Wd, s, cfg, idx, err)
    with pytest.raises(awq.AwqError) as ei:
        awq.awq_device_status(None)
    assert ei.value.status_name == "AWQ_ERR_TIMEOUT"
    monkeypatch.delenv("AWQ_FAULT")
    awq.awq_device_status(None)  # the read cleared it
    _noalloc(Xd, Wd, s, cfg, idx, err)
    awq.awq_device_status(None)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.array_equal(err.cpu().numpy().view(np.uint32), ref_err.view(np.uint32))
    # AWQ_SYNC_CHECK: the call itself reports the status
    monkeypatch.setenv("AWQ_FAULT", "timeout")
    monkeypatch.setenv("AWQ_SYNC_CHECK", "1")
    with pytest.raises(awq.AwqError) as ei:
        awq.awq_search_clip_noalloc(Xd, Wd, s, cfg, idx, err)
    assert ei.value.status_name == "AWQ_ERR_TIMEOUT"
    monkeypatch.delenv("AWQ_FAULT")
    awq.awq_search_clip_noalloc(Xd, Wd, s, cfg, idx, err)


def test_noalloc_rejects_layers_beyond_its_static_scratch():
    cfg = awq.AwqConfig.make(n_clip=20)
    st = abi.LIB.awq_search_clip_noalloc(16, 256, 16384 + 128, 16384 + 128, 16, 64, None,
                                         ctypes.byref(cfg), 16, None, None)
    assert abi.STATUS[st] == "AWQ_ERR_INVALID_ARG"
    assert "16384" in abi.last_error()
