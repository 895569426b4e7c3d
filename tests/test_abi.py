"""CPU-only checks of the C-ABI library: it loads, exports every function the
header declares, and rejects bad arguments on the host before touching CUDA."""

import ctypes

import pytest

import post_weight_quantization_awq_b200 as awq
from post_weight_quantization_awq_b200 import abi


def test_library_exports_every_header_function():
    names = abi.header_functions()
    assert {"awq_act_stats", "awq_search_scale", "awq_search_clip", "awq_quant_pack"} <= set(names)
    for n in names:
        assert hasattr(abi.LIB, n), n
        assert abi.LIB[n] is not None


def test_release_library_has_no_index_checks():
    assert not awq.awq_bounds_checks_enabled()
    awq.awq_bounds_status()  # always AWQ_OK in the release library


def test_debug_library_exports_every_header_function():
    """libawq_debug.so (the same kernels with index checks), when built: the
    same exports, and it reports its checks as enabled."""
    import os
    path = os.path.join(abi.PKG_DIR, "libawq_debug.so")
    if not os.path.exists(path):
        pytest.skip("libawq_debug.so not built")
    lib = ctypes.CDLL(path)
    for n in abi.header_functions():
        assert hasattr(lib, n), n
    lib.awq_bounds_checks_enabled.restype = ctypes.c_int32
    assert lib.awq_bounds_checks_enabled() == 1


def test_python_binding_has_the_abi_names():
    for n in ("awq_act_stats", "awq_scale_grid", "awq_search_scale", "awq_search_clip",
              "awq_quant_pack", "awq_fold_inv_scale", "awq_device_status", "awq_workspace_size"):
        assert callable(getattr(awq, n)), n


def test_version_string():
    assert "sm_100a" in awq.version()


def test_smaller_workspace_runs_the_candidates_in_chunks():
    """The minimum workspace holds one candidate's operand at a time; the
    full one all twenty; a call with a workspace in between is accepted on
    the host, one below the minimum is refused before any CUDA work."""
    cfg = awq.AwqConfig.make(n_alpha=20)
    full = awq.awq_workspace_size(65536, 4096, 4096, cfg)
    low = awq.awq_workspace_size_min(65536, 4096, 4096, cfg)
    assert full - low == 19 * 4096 * 4096 * 2
    st = abi.LIB.awq_search_scale(16, 65536, 4096, 4096, 16, 4096, 16, ctypes.byref(cfg), 256, low - 256,
                                  16, 16, 16, None)
    assert abi.STATUS[st] == "AWQ_ERR_WORKSPACE" and str(low) in abi.last_error()


def test_workspace_size_grows_with_the_problem():
    cfg = awq.AwqConfig.make(n_alpha=20, n_clip=20)
    a = awq.awq_workspace_size(65536, 4096, 4096, cfg)
    b = awq.awq_workspace_size(65536, 4096, 8192, cfg)
    # candidate operand alone: n_alpha * out * in fp16
    assert a >= 20 * 4096 * 4096 * 2 and b > a
    small = awq.awq_workspace_size(256, 512, 512, awq.AwqConfig.make(n_alpha=20))
    assert 20 * 512 * 512 * 2 <= small < 40 * 2 ** 20


@pytest.mark.parametrize("kw,shape,status", [
    (dict(w_bit=5), (256, 512, 512), "AWQ_ERR_UNSUPPORTED"),
    (dict(w_bit=0), (256, 512, 512), "AWQ_ERR_INVALID_ARG"),
    (dict(group_size=96), (256, 576, 512), "AWQ_ERR_UNSUPPORTED"),
    (dict(zero_point=2), (256, 512, 512), "AWQ_ERR_INVALID_ARG"),
    (dict(n_alpha=0), (256, 512, 512), "AWQ_ERR_INVALID_ARG"),
    (dict(n_clip=65), (256, 512, 512), "AWQ_ERR_INVALID_ARG"),
    (dict(clip_min=0.0), (256, 512, 512), "AWQ_ERR_INVALID_ARG"),
    (dict(), (256, 500, 512), "AWQ_ERR_INVALID_ARG"),
    (dict(), (256, 512, 12), "AWQ_ERR_INVALID_ARG"),
    (dict(), (0, 512, 512), "AWQ_ERR_INVALID_ARG"),
    (dict(), ((1 << 22) + 1, 512, 512), "AWQ_ERR_INVALID_ARG"),  # past the exact-sum bound
])
def test_host_validation(kw, shape, status):
    cfg = awq.AwqConfig.make(**kw)
    with pytest.raises(awq.AwqError) as ei:
        awq.awq_workspace_size(*shape, cfg)
    assert "AWQ_ERR_INVALID_ARG" == ei.value.status_name or ei.value.status_name == status
    # the calls report the precise status before any CUDA work
    st = abi.LIB.awq_search_scale(16, shape[0], shape[1], shape[1], 16, shape[2], 16,
                                  ctypes.byref(cfg), 256, 1 << 30, 16, 16, 16, None)
    assert abi.STATUS[st] == status, abi.last_error()


def test_null_and_misaligned_pointers_are_rejected():
    cfg = awq.AwqConfig.make(n_clip=20)
    L = abi.LIB
    assert abi.STATUS[L.awq_act_stats(None, 16, 512, 512, 256, None)] == "AWQ_ERR_INVALID_ARG"
    assert abi.STATUS[L.awq_act_stats(18, 16, 512, 512, 256, None)] == "AWQ_ERR_INVALID_ARG"  # misaligned X
    assert abi.STATUS[L.awq_act_stats(16, 16, 512, 500, 256, None)] == "AWQ_ERR_INVALID_ARG"  # ldx < in
    assert abi.STATUS[L.awq_act_stats(16, 16, 512, 516, 256, None)] == "AWQ_ERR_INVALID_ARG"  # ldx % 8
    assert "ldx" in abi.last_error()
    # workspace missing / misaligned / too small
    for ws, nbytes in ((None, 1 << 30), (128, 1 << 30), (256, 1024)):
        st = L.awq_search_scale(16, 256, 512, 512, 16, 512, 16, ctypes.byref(cfg), ws, nbytes,
                                16, 16, 16, None)
        assert abi.STATUS[st] == "AWQ_ERR_WORKSPACE"
    st = L.awq_search_clip(16, 256, 512, 512, 16, 512, 16, ctypes.byref(awq.AwqConfig.make(n_clip=0)),
                           256, 1 << 30, 16, None, None)
    assert abi.STATUS[st] == "AWQ_ERR_INVALID_ARG" and "n_clip" in abi.last_error()
    st = L.awq_quant_pack(16, 512, 512, None, 16, ctypes.byref(awq.AwqConfig.make(n_clip=0)),
                          16, 16, 16, None)
    assert abi.STATUS[st] == "AWQ_ERR_INVALID_ARG"
    st = L.awq_quant_pack(16, 512, 512, None, None, ctypes.byref(cfg), None, 16, 16, None)
    assert abi.STATUS[st] == "AWQ_ERR_INVALID_ARG"


def test_errors_are_per_thread():
    import threading
    cfg = awq.AwqConfig.make(w_bit=7)
    abi.LIB.awq_workspace_size(256, 512, 512, ctypes.byref(cfg))
    mine = abi.last_error()
    seen = []
    t = threading.Thread(target=lambda: seen.append(abi.last_error()))
    t.start()
    t.join()
    assert "w_bit" in mine and seen == [""]


def test_group_sizes_and_clip_limits():
    """Groups of 32/64/128 for the search, the clip search and packing; the
    clip search works on 128-channel blocks and says so before touching CUDA
    when in is not a multiple of 128."""
    for g in (32, 64, 128):
        assert awq.awq_workspace_size(256, 512, 512, awq.AwqConfig.make(group_size=g)) > 0
        # the clip search's block Grams are counted for every group size
        assert (awq.awq_workspace_size(256, 512, 512, awq.AwqConfig.make(group_size=g, n_clip=20))
                >= 256 + 4 * 128 * 128 * 4)
    cfg = awq.AwqConfig.make(group_size=64, n_clip=20)
    st = abi.LIB.awq_search_clip(16, 256, 576, 576, 16, 512, None, ctypes.byref(cfg), 256, 1 << 30,
                                 16, None, None)
    assert abi.STATUS[st] == "AWQ_ERR_UNSUPPORTED" and "128" in abi.last_error()
    # Gram form needs in % 128 == 0
    cfg = awq.AwqConfig.make(group_size=64, search_form=abi.SEARCH_GRAM)
    st = abi.LIB.awq_search_scale(16, 256, 192, 192, 16, 64, 16, ctypes.byref(cfg), 256, 1 << 30,
                                  16, 16, 16, None)
    assert abi.STATUS[st] == "AWQ_ERR_UNSUPPORTED" and "Gram" in abi.last_error()


def test_w4a16_shape_limits():
    """The W4A16 GEMM states its limits before touching CUDA."""
    cfg = awq.AwqConfig.make()
    st = abi.LIB.awq_w4a16_gemm(16, 256, 512, 512, 16, 16, 16, 264, ctypes.byref(cfg), 16, 264, 256, 1024, None)
    assert abi.STATUS[st] == "AWQ_ERR_UNSUPPORTED" and "out % 32" in abi.last_error()
    st = abi.LIB.awq_w4a16_gemm(16, 256, 512, 512, 16, 16, 16, 256, ctypes.byref(cfg), 16, 200, 256, 1024, None)
    assert abi.STATUS[st] == "AWQ_ERR_INVALID_ARG" and "ldy" in abi.last_error()


def test_sharding_calls_check_their_arguments():
    """The token-sharding calls reject bad arguments on the host, before any
    CUDA work, with the status the header states."""
    L = abi.LIB
    cfg = awq.AwqConfig.make(n_clip=20)
    S = abi.STATUS
    assert S[L.awq_act_sums(16, 256, 512, 512, None, None)] == "AWQ_ERR_INVALID_ARG"
    assert S[L.awq_act_sums(16, 256, 512, 512, 12, None)] == "AWQ_ERR_INVALID_ARG"  # sums misaligned
    assert S[L.awq_act_sums(16, 0, 512, 512, 16, None)] == "AWQ_ERR_INVALID_ARG"   # no tokens
    assert S[L.awq_act_stats_finish(16, 0, 512, 16, None)] == "AWQ_ERR_INVALID_ARG"
    assert S[L.awq_act_stats_finish(None, 10, 512, 16, None)] == "AWQ_ERR_INVALID_ARG"
    st = L.awq_search_scale_sse(16, 256, 512, 512, 16, 512, 16, ctypes.byref(cfg), 256, 1 << 30, None, None)
    assert S[st] == "AWQ_ERR_INVALID_ARG" and "sse" in abi.last_error()
    st = L.awq_select_scale(16, 256, 512, 512, 16, ctypes.byref(cfg), 256, 128, 16, 16, 16, None)
    assert S[st] == "AWQ_ERR_WORKSPACE"
    st = L.awq_block_grams(16, 256, 320, 320, ctypes.byref(cfg), 256, 1 << 30, 16, None)
    assert S[st] == "AWQ_ERR_INVALID_ARG"
    st = L.awq_search_clip_grams(16, 512, 512, 16, 16, ctypes.byref(awq.AwqConfig.make(n_clip=0)),
                                 256, 1024, 16, None, None)
    assert S[st] == "AWQ_ERR_INVALID_ARG" and "n_clip" in abi.last_error()
    st = L.awq_search_clip_grams(16, 512, 512, 16, None, ctypes.byref(cfg), 256, 1024, 16, None, None)
    assert S[st] == "AWQ_ERR_INVALID_ARG" and "G" in abi.last_error()


def test_search_forms_and_zero_point_are_validated():
    for kw, status in ((dict(search_form=4), "AWQ_ERR_INVALID_ARG"), (dict(zero_point=-1), "AWQ_ERR_INVALID_ARG")):
        with pytest.raises(awq.AwqError) as ei:
            awq.awq_workspace_size(256, 512, 512, awq.AwqConfig.make(**kw))
        assert ei.value.status_name == status
    # the cached-output form needs room for the cached output: more workspace than the error form
    a = awq.awq_workspace_size(1000, 512, 512, awq.AwqConfig.make())
    b = awq.awq_workspace_size(1000, 512, 512, awq.AwqConfig.make(search_form=abi.SEARCH_CACHED_Y))
    assert b - a >= 1024 * 512 * 2
    # the fused form keeps 8 bytes per (alpha, row, group) instead of the
    # n_alpha x out_pad x in fp16 operand, whatever the workspace
    c = awq.awq_workspace_size(1000, 512, 512, awq.AwqConfig.make(search_form=abi.SEARCH_FUSED))
    assert a - c == 20 * 512 * 512 * 2 - 20 * 512 * 4 * 8
    assert awq.awq_workspace_size_min(1000, 512, 512, awq.AwqConfig.make(search_form=abi.SEARCH_FUSED)) <= c


def test_binding_constants_match_the_header():
    """Status codes and scoring forms in the binding are the header's."""
    import re
    text = open(abi.HEADER_PATH).read()
    for name, val in re.findall(r"\b(AWQ_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", text):
        assert abi.STATUS[int(val)] == name, name
    forms = dict(re.findall(r"\b(AWQ_SEARCH_[A-Z_]+)\s*=\s*(\d+)", text))
    assert int(forms["AWQ_SEARCH_DIRECT"]) == abi.SEARCH_DIRECT
    assert int(forms["AWQ_SEARCH_GRAM"]) == abi.SEARCH_GRAM
    assert int(forms["AWQ_SEARCH_CACHED_Y"]) == abi.SEARCH_CACHED_Y
    assert int(forms["AWQ_SEARCH_FUSED"]) == abi.SEARCH_FUSED
