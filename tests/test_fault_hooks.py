"""CPU checks of the host-side fault injection (environment variable
AWQ_FAULT): "alloc" makes every workspace unobtainable and "launch" fails every
call after its argument checks and before any CUDA call, so both error paths
run here without a GPU.  ("timeout" and "nonfinite" act on the device and are
checked by the GPU tests.)"""

import ctypes

import pytest

import post_weight_quantization_awq_b200 as awq
from post_weight_quantization_awq_b200 import abi

L = abi.LIB
A = 256          # a 256-byte-aligned stand-in for a device pointer (never dereferenced)
BIG = 1 << 40    # workspace bytes: large enough for any layout


def _cfg(**kw):
    return ctypes.byref(awq.AwqConfig.make(**kw))


def _launching_calls():
    """Every C-ABI call that launches work, with valid arguments."""
    T, inn, out = 256, 512, 512
    return {
        "awq_act_stats": lambda: L.awq_act_stats(A, T, inn, inn, A, None),
        "awq_scale_grid": lambda: L.awq_scale_grid(A, inn, 20, A, None),
        "awq_search_scale": lambda: L.awq_search_scale(A, T, inn, inn, A, out, A, _cfg(), A, BIG,
                                                       A, A, A, None),
        "awq_search_scale_sse": lambda: L.awq_search_scale_sse(A, T, inn, inn, A, out, A, _cfg(), A,
                                                               BIG, A, None),
        "awq_select_scale": lambda: L.awq_select_scale(A, T, inn, out, A, _cfg(), A, BIG, A, A, A,
                                                       None),
        "awq_act_sums": lambda: L.awq_act_sums(A, T, inn, inn, A, None),
        "awq_act_stats_finish": lambda: L.awq_act_stats_finish(A, T, inn, A, None),
        "awq_search_clip": lambda: L.awq_search_clip(A, T, inn, inn, A, out, A, _cfg(n_clip=20), A,
                                                     BIG, A, None, None),
        "awq_search_clip_noalloc": lambda: L.awq_search_clip_noalloc(A, T, inn, inn, A, out, A,
                                                                     _cfg(n_clip=20), A, None, None),
        "awq_block_grams": lambda: L.awq_block_grams(A, T, inn, inn, _cfg(n_clip=20), A, BIG, A,
                                                     None),
        "awq_search_clip_grams": lambda: L.awq_search_clip_grams(A, out, inn, A, A, _cfg(n_clip=20),
                                                                 A, BIG, A, None, None),
        "awq_candidate_codes": lambda: L.awq_candidate_codes(A, out, inn, A, _cfg(), A, BIG, A, A, A,
                                                             None),
        "awq_clip_candidate_codes": lambda: L.awq_clip_candidate_codes(A, out, inn, A, A,
                                                                       _cfg(n_clip=20), A, BIG, A,
                                                                       None, A, A, None),
        "awq_quant_pack": lambda: L.awq_quant_pack(A, out, inn, A, A, _cfg(n_clip=20), A, A, A, None),
        "awq_fold_inv_scale": lambda: L.awq_fold_inv_scale(A, inn, 1, A, None),
        "awq_w4a16_gemm": lambda: L.awq_w4a16_gemm(A, T, inn, inn, A, A, A, out, _cfg(), A, out, A,
                                                   BIG, None),
    }


@pytest.mark.parametrize("name", sorted(_launching_calls()))
def test_injected_launch_failure(monkeypatch, name):
    monkeypatch.setenv("AWQ_FAULT", "launch")
    st = _launching_calls()[name]()
    assert abi.STATUS[st] == "AWQ_ERR_CUDA", (name, abi.last_error())
    assert "injected launch failure" in abi.last_error()


def test_launch_gate_comes_after_the_argument_checks(monkeypatch):
    monkeypatch.setenv("AWQ_FAULT", "launch")
    # a bad argument is still reported as such, not as the injected failure
    st = L.awq_act_stats(A, 16, 512, 500, A, None)
    assert abi.STATUS[st] == "AWQ_ERR_INVALID_ARG" and "ldx" in abi.last_error()


def test_every_launching_call_is_gated():
    """The gated calls are every call the header declares except the
    host-only ones."""
    host_only = {"awq_version", "awq_last_error", "awq_workspace_size", "awq_workspace_size_min",
                 "awq_w4a16_workspace_size",
                 "awq_device_status", "awq_bounds_checks_enabled", "awq_bounds_status",
                 "awq_profile_enable", "awq_profile_read", "awq_profile_reset"}
    assert set(abi.header_functions()) - host_only == set(_launching_calls())


def test_injected_allocation_failure(monkeypatch):
    monkeypatch.setenv("AWQ_FAULT", "alloc")
    cfg = awq.AwqConfig.make(n_alpha=20)
    with pytest.raises(awq.AwqError) as ei:
        awq.awq_workspace_size(256, 512, 512, cfg)
    # awq_workspace_size reports failure by returning 0, with the message
    assert "injected allocation failure" in str(ei.value)
    with pytest.raises(awq.AwqError):
        awq.alloc_workspace(256, 512, 512, cfg, device="cpu")
    # a call given a workspace refuses it
    for st in (L.awq_search_scale(A, 256, 512, 512, A, 512, A, _cfg(), A, BIG, A, A, A, None),
               L.awq_search_clip(A, 256, 512, 512, A, 512, A, _cfg(n_clip=20), A, BIG, A, None, None),
               L.awq_w4a16_gemm(A, 256, 512, 512, A, A, A, 512, _cfg(), A, 512, A, BIG, None)):
        assert abi.STATUS[st] == "AWQ_ERR_WORKSPACE"
        assert "injected allocation failure" in abi.last_error()


def test_unknown_fault_name_injects_nothing(monkeypatch):
    monkeypatch.setenv("AWQ_FAULT", "nothing-of-that-name")
    cfg = awq.AwqConfig.make(n_alpha=20)
    assert awq.awq_workspace_size(256, 512, 512, cfg) > 0
    monkeypatch.delenv("AWQ_FAULT")
    assert awq.awq_workspace_size(256, 512, 512, cfg) > 0
