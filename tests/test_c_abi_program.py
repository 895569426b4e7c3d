"""The C ABI from plain C (tests/c_abi/quantize_layer.c): the header compiles
as C11 with gcc and the program links against libawq.so (CPU); on the GPU the
program quantises a seeded layer through the four calls, and the same calls
made through the Python binding on the same inputs give the same bits."""

import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import post_weight_quantization_awq_b200 as awq
from post_weight_quantization_awq_b200 import abi

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "c_abi", "quantize_layer.c")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path) -> str:
    if shutil.which("gcc") is None or not os.path.exists(os.path.join(CUDA_HOME, "include", "cuda_runtime.h")):
        pytest.skip("gcc or the CUDA headers are missing")
    exe = str(tmp_path / "quantize_layer")
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA_HOME, "include"), SRC, "-o", exe,
           "-L", os.path.join(CUDA_HOME, "lib64"), "-lcudart", "-L", abi.PKG_DIR, "-lawq",
           f"-Wl,-rpath,{abi.PKG_DIR}", f"-Wl,-rpath,{os.path.join(CUDA_HOME, 'lib64')}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_header_compiles_as_c_and_the_program_links(tmp_path):
    assert os.path.exists(_compile(tmp_path))


def _inputs(T, inn, out):
    """The program's generator: a 64-bit LCG, u in [0, 1), x = (u - 0.5) c_j
    (c_j = 20 on every 50th channel from 7), w = (u - 0.5) / 16, each value
    rounded double -> float -> half."""
    mask = (1 << 64) - 1
    state = 12345
    n = T * inn + out * inn
    u = np.empty(n, dtype=np.float64)
    for i in range(n):
        state = (state * 6364136223846793005 + 1442695040888963407) & mask
        u[i] = (state >> 11) * (1.0 / 9007199254740992.0)
    c = np.where(np.arange(inn) % 50 == 7, 20.0, 1.0)
    X = ((u[:T * inn].reshape(T, inn) - 0.5) * c).astype(np.float32).astype(np.float16)
    W = ((u[T * inn:].reshape(out, inn) - 0.5) / 16.0).astype(np.float32).astype(np.float16)
    return X, W


def test_c_program_inputs_match_numpy(tmp_path):
    """The program's generator and its round-to-nearest-even fp16 conversion
    (written out in C) give numpy's float16 bits for every value, subnormal
    halves included (w values below 2^-14)."""
    exe = _compile(tmp_path)
    T, inn, out = 200, 256, 136
    path = str(tmp_path / "in.bin")
    r = subprocess.run([exe, "--inputs", path, str(T), str(inn), str(out)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    raw = np.fromfile(path, dtype=np.uint16)
    X, W = _inputs(T, inn, out)
    assert np.array_equal(raw[:T * inn], X.view(np.uint16).ravel())
    assert np.array_equal(raw[T * inn:], W.view(np.uint16).ravel())
    assert np.any(np.abs(W.astype(np.float32)) < 2.0 ** -14)  # subnormal halves were exercised


@pytest.mark.gpu
def test_c_program_matches_the_python_binding(tmp_path):
    from gpu_helpers import need_cuda
    need_cuda()
    exe = _compile(tmp_path)
    T, inn, out = 1000, 512, 264
    res_path = str(tmp_path / "out.bin")
    r = subprocess.run([exe, res_path, str(T), str(inn), str(out)], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    g, n_alpha = inn // 128, 20
    raw = open(res_path, "rb").read()
    off = 0

    def take(dtype, count):
        nonlocal off
        a = np.frombuffer(raw, dtype=dtype, count=count, offset=off)
        off += a.nbytes
        return a

    best = int(take(np.int32, 1)[0])
    mse = take(np.float64, n_alpha)
    clip = take(np.uint8, out * g).reshape(out, g)
    qw = take(np.int32, inn * out // 8).reshape(inn, out // 8)
    qz = take(np.int32, g * out // 8).reshape(g, out // 8)
    sc = take(np.uint16, g * out).reshape(g, out)
    Xc = take(np.uint16, T * inn).reshape(T, inn)
    Wc = take(np.uint16, out * inn).reshape(out, inn)
    assert off == len(raw)
    X, W = _inputs(T, inn, out)
    assert np.array_equal(Xc, X.view(np.uint16)) and np.array_equal(Wc, W.view(np.uint16))
    cfg = awq.AwqConfig.make(w_bit=4, group_size=128, n_alpha=n_alpha, n_clip=20, clip_min=0.5)
    res = awq.quantize_layer(torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda(), cfg)
    torch.cuda.synchronize()
    assert best == int(res.best_idx.item())
    assert np.array_equal(mse, res.mse.cpu().numpy())
    assert np.array_equal(clip, res.clip_idx.cpu().numpy())
    assert np.array_equal(qw, res.qweight.cpu().numpy())
    assert np.array_equal(qz, res.qzeros.cpu().numpy())
    assert np.array_equal(sc, res.scales.cpu().numpy().view(np.uint16))
