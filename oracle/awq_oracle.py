"""CPU oracle for AWQ's per-layer activation-aware scale search.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product (the
CUDA library and its Python binding) never calls it, and it shares no code
with the product: it is a plain, slow, fp64 restatement of what the method
computes, written so that a reader can check each step against the pages.

Sources (web pages about AWQ, Lin et al.):
  [P1] "AWQ and Activation-Aware Scaling" — "Scaling instead of protecting":
       s = abar^alpha, abar the per-channel mean activation magnitude, alpha in
       [0, 1] found by a small per-layer grid search minimising reconstruction
       error; alpha = 0 is plain quantisation.
  [P4] "05 — AWQ: Activation-Aware Weight Scaling"
       §3 (the scaling trick): X W = (X diag(s)^-1)(diag(s) W) for positive s;
       §4 (how to find s): ~20 values of alpha in [0, 1], apply the scaling,
       quantize, measure MSE against the fp16 output, keep the best; optional
       clipping-ratio search over 0.5 – 1.0 of the max;
       §5 (bit-level output format): qweight [in, out/8] int32, qzeros
       [in/g, out/8] int32, scales fp16 [in/g, out], g = 128, 4.156 bits/weight;
       §9 (quant_config): zero_point = True, q_group_size = 128, w_bit = 4.

Readings where the pages are silent:
  * group-wise asymmetric min/max quantisation of g consecutive INPUT channels
    of one output row; zero point rounded and clamped to [0, 2^b - 1];
  * without a zero point ([P4] §9 zero_point = False; [P4] §3 describes the
    symmetric scheme only by its half-step error): step = max |wt| /
    (2^(b-1) - 1), codes centred on z = 2^(b-1) in the same unsigned nibble;
  * every float step of the quantiser in fp32, correctly rounded, with
    round-half-to-even; guards d >= 1e-5 and abar >= 1e-4;
  * alpha_i = i / (n_alpha - 1); clip ratio r_c = 1 - c (1 - r_min)/(n_clip - 1)
    applied to both ends of the group range, one ratio per (row, group), scored
    by that group's own output error over all tokens;
  * MSE reference = the exact product X W^T (fp64), not an fp16-rounded copy;
  * ties resolve to the lowest index (smaller alpha, less clipping);
  * nibble order: output o sits in nibble (o mod 8) of word o // 8, low nibble
    first; INT3 codes use the same 4-bit container.

Every array argument is a numpy array; fp16 inputs are ``np.float16``.
"""

from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

__all__ = [
    "act_stats",
    "alpha_grid",
    "scale_grid",
    "quantize_groups",
    "effective_error",
    "gram",
    "mse_direct",
    "mse_fp16_output",
    "mse_gram",
    "search_scale",
    "clip_ratios",
    "block_grams",
    "search_clip",
    "quant_pack",
    "unpack_nibbles",
    "dequant_packed",
    "w4a16_matmul",
    "fold_inv_scale",
]

ABAR_FLOOR = 1e-4          # dead-channel guard on abar (fp64)
RANGE_FLOOR = np.float32(1e-5)  # constant-group guard on max - min (fp32)


# --------------------------------------------------------------------------
# D1  activation statistic  abar_j = mean_t |X_tj|        ([P1], [P4] §4)
# --------------------------------------------------------------------------
def act_stats(X: np.ndarray) -> np.ndarray:
    """Per-input-channel mean |x| over the calibration tokens, fp64 [in].

    The sum is exact: every fp16 value is an integer multiple of 2^-24, so
    sum_t |X_tj| is an integer count of 2^-24 units (< 2^57 for T <= 2^16 ...
    2^17), held in int64.  abar = RN64(RN64(S) * 2^-24 / T)."""
    X = np.asarray(X)
    assert X.dtype == np.float16 and X.ndim == 2
    T, d = X.shape
    S = np.zeros(d, dtype=np.int64)
    # Integer addition is exact and associative, so summing token blocks in
    # turn gives the same S as one sum; blocks only bound the memory used.
    for t0 in range(0, T, 4096):
        units = np.abs(X[t0:t0 + 4096].astype(np.float64)) * 2.0 ** 24
        S += units.astype(np.int64).sum(axis=0, dtype=np.int64)
    return (S.astype(np.float64) * 2.0 ** -24) / float(T)


# --------------------------------------------------------------------------
# D2, D3  the alpha grid and s = abar^alpha                ([P1], [P4] §4)
# --------------------------------------------------------------------------
def alpha_grid(n_alpha: int) -> np.ndarray:
    """alpha_i = i / (n_alpha - 1), i = 0..n_alpha-1, fp64 (both ends kept)."""
    if n_alpha == 1:
        return np.zeros(1, dtype=np.float64)
    return np.array([i / float(n_alpha - 1) for i in range(n_alpha)], dtype=np.float64)


def scale_grid(abar: np.ndarray, alphas: np.ndarray) -> np.ndarray:
    """s_ij = RN32(pow(max(abar_j, 1e-4), alpha_i)), fp32 [n_alpha, in].

    pow is the C library's double pow (math.pow); no normalising constant."""
    a = np.maximum(np.asarray(abar, dtype=np.float64), ABAR_FLOOR)
    s = np.empty((len(alphas), a.shape[0]), dtype=np.float32)
    for i, al in enumerate(alphas):
        s[i] = np.array([math.pow(float(x), float(al)) for x in a], dtype=np.float64).astype(np.float32)
    return s


# --------------------------------------------------------------------------
# D4  group-wise asymmetric INT-b fake quantisation of diag(s) W
#     ([P4] §5 layout, §9 zero_point / q_group_size / w_bit)
# --------------------------------------------------------------------------
def quantize_groups(W: np.ndarray, s: Optional[np.ndarray], group: int, w_bit: int,
                    ratio: Optional[np.ndarray] = None, zero_point: bool = True) -> dict:
    """Quantise every (row o, group k) of diag(s) W, all in fp32.

    W [out, in] fp16; s [in] fp32 (None = 1); ratio [out, in/g] fp32 (None = 1).
    Per group: wt = RN32(s w); mx, mn = max, min of wt (each scaled by the
    ratio when one is given); then
      zero_point (asymmetric, [P4] §9 zero_point = True):
        d = max(mx - mn, 1e-5); delta = d / (2^b - 1);
        z = clamp(rne(-mn / delta), 0, 2^b - 1);
      no zero point (the symmetric scheme of [P4] §3, codes centred on 0):
        d = max(|mx|, |mn|, 1e-5); delta = d / (2^(b-1) - 1); z = 2^(b-1);
    q = clamp(rne(wt / delta) + z, 0, 2^b - 1); deq = (q - z) delta.

    Returns dict with q uint8 [out, in], z uint8 [out, in/g], delta fp32
    [out, in/g], deq fp32 [out, in], wt fp32 [out, in]."""
    W = np.asarray(W)
    assert W.dtype == np.float16 and W.ndim == 2
    out, inn = W.shape
    assert inn % group == 0
    G = inn // group
    qmax = np.float32(2 ** w_bit - 1)
    w32 = W.astype(np.float32)
    wt = w32 if s is None else np.asarray(s, dtype=np.float32)[None, :] * w32
    wt3 = wt.reshape(out, G, group)
    mx = wt3.max(axis=2)
    mn = wt3.min(axis=2)
    if ratio is not None:
        r = np.asarray(ratio, dtype=np.float32)
        mx = r * mx
        mn = r * mn
    if zero_point:
        d = np.maximum(mx - mn, RANGE_FLOOR)
        delta = d / qmax
        z = np.clip(np.rint(-mn / delta), np.float32(0), qmax)
    else:
        d = np.maximum(np.maximum(np.abs(mx), np.abs(mn)), RANGE_FLOOR)
        delta = d / np.float32(2 ** (w_bit - 1) - 1)
        z = np.full(delta.shape, np.float32(2 ** (w_bit - 1)), dtype=np.float32)
    q = np.clip(np.rint(wt3 / delta[:, :, None]) + z[:, :, None], np.float32(0), qmax)
    deq = (q - z[:, :, None]) * delta[:, :, None]
    assert wt.dtype == np.float32 and delta.dtype == np.float32 and deq.dtype == np.float32
    return {
        "q": q.reshape(out, inn).astype(np.uint8),
        "z": z.astype(np.uint8),
        "delta": delta,
        "deq": deq.reshape(out, inn),
        "wt": wt,
    }


def effective_error(W: np.ndarray, s: Optional[np.ndarray], deq: np.ndarray) -> np.ndarray:
    """Effective weight error of a candidate, fp64 [out, in]:
    delta_oj = deq_oj / s_j - W_oj.  By the scaling invariance ([P4] §3),
    (X diag(s)^-1) Qdeq^T - X W^T = X delta^T."""
    d = np.asarray(deq, dtype=np.float64)
    if s is not None:
        d = d / np.asarray(s, dtype=np.float64)[None, :]
    return d - np.asarray(W, dtype=np.float64)


# --------------------------------------------------------------------------
# D5  candidate score: MSE of the candidate output against X W^T  ([P4] §4)
# --------------------------------------------------------------------------
def gram(X: np.ndarray) -> np.ndarray:
    """G = X^T X in fp64 [in, in]."""
    X64 = np.asarray(X, dtype=np.float64)
    return X64.T @ X64


def mse_direct(X: np.ndarray, delta: np.ndarray) -> float:
    """(1 / (T out)) sum_t sum_o (sum_j X_tj delta_oj)^2, fp64 (direct form)."""
    X64 = np.asarray(X, dtype=np.float64)
    T = X64.shape[0]
    total = 0.0
    # Squared errors are summed one token block at a time to bound memory.
    for t0 in range(0, T, 4096):
        E = X64[t0:t0 + 4096] @ delta.T
        total += float(np.sum(E * E))
    return total / (T * delta.shape[0])


def mse_fp16_output(X: np.ndarray, W: np.ndarray, s: Optional[np.ndarray],
                    deq: np.ndarray) -> float:
    """The literal reading of [P4] §4, "measure MSE against the fp16 output":
    the candidate's weights deq/s (fp32 quotient) and the reference output
    X W^T (exact) are each rounded to fp16, and the mean squared difference of
    X (deq/s)^T and that fp16 output is taken in fp64.  It differs from the
    exact score (mse_direct of effective_error) only through the two fp16
    roundings."""
    X64 = np.asarray(X, dtype=np.float64)
    W64 = np.asarray(W, dtype=np.float64)
    d32 = np.asarray(deq, dtype=np.float32)
    B = d32 if s is None else d32 / np.asarray(s, dtype=np.float32)[None, :]
    B64 = B.astype(np.float16).astype(np.float64)
    T = X64.shape[0]
    total = 0.0
    for t0 in range(0, T, 4096):
        Xb = X64[t0:t0 + 4096]
        Y16 = (Xb @ W64.T).astype(np.float16).astype(np.float64)
        E = Xb @ B64.T - Y16
        total += float(np.sum(E * E))
    return total / (T * W64.shape[0])


def mse_gram(G: np.ndarray, delta: np.ndarray, T: int) -> float:
    """(1 / (T out)) sum_o delta_o^T G delta_o, fp64 (Gram form; equal to the
    direct form in exact arithmetic since sum_t (x_t . d)^2 = d^T X^T X d)."""
    return float(np.sum((delta @ G) * delta)) / (T * delta.shape[0])


def search_scale(X: np.ndarray, W: np.ndarray, abar: np.ndarray, w_bit: int, group: int,
                 n_alpha: int, form: str = "gram", G: Optional[np.ndarray] = None,
                 zero_point: bool = True) -> Tuple[np.ndarray, int, np.ndarray, np.ndarray]:
    """alpha-grid search ([P1], [P4] §4).

    For every alpha_i: s_i = abar^alpha_i, fake-quantise diag(s_i) W, score
    MSE_i of (X diag(s_i)^-1) Qdeq^T against X W^T; keep the first argmin.
    form "gram" / "direct" score against the exact X W^T; "fp16_output"
    against its fp16 rounding (mse_fp16_output).
    Returns (mse fp64 [n_alpha], best index, s_best fp32 [in], s grid)."""
    alphas = alpha_grid(n_alpha)
    S = scale_grid(abar, alphas)
    T = X.shape[0]
    if form == "gram" and G is None:
        G = gram(X)
    mse = np.empty(n_alpha, dtype=np.float64)
    for i in range(n_alpha):
        qd = quantize_groups(W, S[i], group, w_bit, zero_point=zero_point)
        if form == "fp16_output":
            mse[i] = mse_fp16_output(X, W, S[i], qd["deq"])
            continue
        delta = effective_error(W, S[i], qd["deq"])
        mse[i] = mse_gram(G, delta, T) if form == "gram" else mse_direct(X, delta)
    best = int(np.argmin(mse))  # first index attaining the minimum
    return mse, best, S[best].copy(), S


# --------------------------------------------------------------------------
# D7  per-(row, group) clip-ratio search                     ([P4] §4)
# --------------------------------------------------------------------------
def clip_ratios(n_clip: int, clip_min: float) -> np.ndarray:
    """r_c = 1 - c (1 - clip_min) / (n_clip - 1), c = 0..n_clip-1, fp64."""
    if n_clip == 1:
        return np.ones(1, dtype=np.float64)
    cm = float(np.float32(clip_min))
    return np.array([1.0 - c * (1.0 - cm) / (n_clip - 1) for c in range(n_clip)], dtype=np.float64)


def block_grams(X: np.ndarray, group: int) -> list:
    """G_k = X_k^T X_k (fp64) for every group k of g input channels."""
    X64 = np.asarray(X, dtype=np.float64)
    Gn = X64.shape[1] // group
    return [X64[:, k * group:(k + 1) * group].T @ X64[:, k * group:(k + 1) * group] for k in range(Gn)]


def search_clip(X: np.ndarray, W: np.ndarray, s: np.ndarray, w_bit: int, group: int,
                n_clip: int, clip_min: float, Gk: Optional[list] = None,
                zero_point: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """For every (row o, group k) pick the clip ratio whose fake-quantised
    group gives the smallest output error over all tokens,
    E_okc = sum_t (sum_{j in k} X_tj delta^(c)_oj)^2 = d^T (X_k^T X_k) d.
    ``Gk`` may pass the block Grams of X already computed.

    Returns (clip_idx uint8 [out, in/g], E fp64 [out, in/g, n_clip])."""
    out, inn = W.shape
    Gn = inn // group
    r = clip_ratios(n_clip, clip_min).astype(np.float32)
    if Gk is None:
        Gk = block_grams(X, group)
    E = np.empty((out, Gn, n_clip), dtype=np.float64)
    for c in range(n_clip):
        ratio = np.full((out, Gn), r[c], dtype=np.float32)
        qd = quantize_groups(W, s, group, w_bit, ratio, zero_point)
        delta = effective_error(W, s, qd["deq"]).reshape(out, Gn, group)
        for k in range(Gn):
            dk = delta[:, k, :]
            E[:, k, c] = np.sum((dk @ Gk[k]) * dk, axis=1)
    clip_idx = np.argmin(E, axis=2).astype(np.uint8)  # first index on ties
    return clip_idx, E


# --------------------------------------------------------------------------
# D8  final codes and packing                                ([P4] §5)
# --------------------------------------------------------------------------
def quant_pack(W: np.ndarray, s: Optional[np.ndarray], clip_idx: Optional[np.ndarray],
               w_bit: int, group: int, n_clip: int = 1, clip_min: float = 0.5,
               zero_point: bool = True) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Final codes with (s, r_clip) and the pages' storage layout:
    qweight [in, out/8] int32 with q[o, j] in nibble (o mod 8) of word
    [j, o // 8]; qzeros [in/g, out/8] int32 likewise for z[o, k] (without a
    zero point every z is 2^(b-1), so (q - z) scale dequantises either kind);
    scales [in/g, out] fp16 = RN16(delta[o, k])."""
    out, inn = W.shape
    assert out % 8 == 0
    ratio = None
    if clip_idx is not None:
        r = clip_ratios(n_clip, clip_min).astype(np.float32)
        ratio = r[np.asarray(clip_idx, dtype=np.int64)]
    qd = quantize_groups(W, s, group, w_bit, ratio, zero_point)
    q = qd["q"].astype(np.uint32)
    z = qd["z"].astype(np.uint32)
    qweight = np.zeros((inn, out // 8), dtype=np.uint32)
    qzeros = np.zeros((inn // group, out // 8), dtype=np.uint32)
    for e in range(8):
        qweight |= q[e::8, :].T << np.uint32(4 * e)
        qzeros |= z[e::8, :].T << np.uint32(4 * e)
    scales = np.ascontiguousarray(qd["delta"].T.astype(np.float16))
    return qweight.view(np.int32), qzeros.view(np.int32), scales


def unpack_nibbles(words: np.ndarray) -> np.ndarray:
    """Inverse of the packing: int32 [R, C] -> codes uint8 [8 C, R], with code
    [o, r] taken from nibble (o mod 8) of word [r, o // 8]."""
    u = np.asarray(words).view(np.uint32)
    R, C = u.shape
    q = np.zeros((8 * C, R), dtype=np.uint8)
    for e in range(8):
        q[e::8, :] = ((u >> np.uint32(4 * e)) & np.uint32(0xF)).T.astype(np.uint8)
    return q


# --------------------------------------------------------------------------
# The step after the path: a W4A16 product on the packed output  ([P4] §5
# layout; the pages' inference kernels dequantise the weights on the fly)
# --------------------------------------------------------------------------
def dequant_packed(qweight: np.ndarray, qzeros: np.ndarray, scales: np.ndarray,
                   group: int) -> np.ndarray:
    """fp16 weights [out, in] of a packed layer: RN16((q - z) * scale), with q
    from qweight [in, out/8], z from qzeros [in/g, out/8] and scale from
    scales [in/g, out].  (q - z) * scale is exact in fp32 (a small integer times
    an fp16), so the one rounding is the final RN16."""
    q = unpack_nibbles(qweight).astype(np.float32)                        # [out, in]
    z = np.repeat(unpack_nibbles(qzeros).astype(np.float32), group, axis=1)
    sc = np.repeat(np.asarray(scales).astype(np.float32).T, group, axis=1)
    return ((q - z) * sc).astype(np.float16)


def w4a16_matmul(X: np.ndarray, qweight: np.ndarray, qzeros: np.ndarray, scales: np.ndarray,
                 group: int) -> np.ndarray:
    """Y = X Wd^T in fp64 with Wd = dequant_packed(...) (the GPU accumulates in
    fp32 and rounds Y to fp16)."""
    Wd = dequant_packed(qweight, qzeros, scales, group).astype(np.float64)
    return np.asarray(X, dtype=np.float64) @ Wd.T


# --------------------------------------------------------------------------
# Fold of 1/s into the preceding operation   ([P1] "Scaling instead of
# protecting": the activation-side division is absorbed by the previous
# normalisation's scale or the previous linear layer)
# --------------------------------------------------------------------------
def fold_inv_scale(v: np.ndarray, s: np.ndarray) -> np.ndarray:
    """RN16(RN32(v) / s) along the last axis: a norm's gamma [d] or the rows
    of a preceding linear stored [d, in] (row j divided by s_j)."""
    v32 = np.asarray(v).astype(np.float32)
    s32 = np.asarray(s, dtype=np.float32)
    if v32.ndim == 1:
        return (v32 / s32).astype(np.float16)
    return (v32 / s32[:, None]).astype(np.float16)
