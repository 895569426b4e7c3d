"""Pins for the CPU oracle: each test checks the oracle against something
other than itself — hand-worked examples, exact rational arithmetic, brute
force, closed forms and the special cases the AWQ pages state.  CPU only."""

import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import awq_oracle as O
from synthetic import OutlierSpec, heavy_tailed_activations, gaussian_weight, random_layer


def _group_row(entries, group, fill=0.0):
    w = np.full((1, group), fill, dtype=np.float16)
    for j, v in entries.items():
        w[0, j] = np.float16(v)
    return w


# --------------------------------------------------------------------------
# D1  activation statistic
# --------------------------------------------------------------------------
def test_act_stats_matches_exact_rational_mean():
    rng = np.random.default_rng(1)
    T, d = 37, 24
    mags = 2.0 ** rng.integers(-24, 15, size=(T, d))
    X = (np.clip(rng.standard_normal((T, d)), -1.9, 1.9) * mags).astype(np.float16)
    X[0, 0] = np.float16(65504.0)
    X[1:, 0] = np.float16(2.0 ** -24)          # subnormal tail next to the max
    X[:, 1] = np.float16(-1.0)
    abar = O.act_stats(X)
    for j in range(d):
        S = sum(Fraction(float(abs(x))) for x in X[:, j].astype(np.float64))
        want = float(S) / T                      # RN64(S), then RN64(. / T)
        assert abar[j] == want, (j, abar[j], want)
    assert abar[1] == 1.0


def test_act_stats_single_nonzero_and_fp32_loss():
    T = 4096
    X = np.zeros((T, 8), dtype=np.float16)
    X[5, 3] = np.float16(-3.0)
    X[:, 4] = np.float16(2.0 ** -24)
    X[0, 4] = np.float16(2048.0)
    abar = O.act_stats(X)
    assert abar[3] == 3.0 / T
    assert np.all(abar[[0, 1, 2, 5, 6, 7]] == 0.0)
    exact = (2048.0 + (T - 1) * 2.0 ** -24) / T
    assert abar[4] == exact
    # a naive fp32 running sum loses the small terms entirely
    acc = np.float32(0)
    for x in X[:, 4].astype(np.float32):
        acc = np.float32(acc + abs(x))
    assert float(acc) / T != exact


# --------------------------------------------------------------------------
# D2, D3  alpha grid and s = abar^alpha
# --------------------------------------------------------------------------
def test_alpha_grid_endpoints_and_spacing():
    a = O.alpha_grid(20)
    assert a[0] == 0.0 and a[-1] == 1.0 and len(a) == 20
    assert np.allclose(np.diff(a), 1.0 / 19, rtol=0, atol=1e-15)
    assert list(O.alpha_grid(1)) == [0.0]


def test_alpha_grid_is_the_correctly_rounded_quotient():
    """alpha_i is the double nearest the rational i / (n - 1) (the even grid
    on [0, 1] of "05 — AWQ" §4): checked in exact arithmetic against both
    neighbouring doubles.  A grid built as i * (1 / (n - 1)) misses this at
    i = 13 and 17 for n = 20 (and at i = 7 for n = 10)."""
    for n in (2, 3, 7, 10, 20, 64):
        a = O.alpha_grid(n)
        for i in range(n):
            exact = Fraction(i, n - 1)
            err = abs(Fraction(float(a[i])) - exact)
            for nb in (math.nextafter(float(a[i]), -math.inf), math.nextafter(float(a[i]), math.inf)):
                assert err <= abs(Fraction(nb) - exact), (n, i)
    recip = [i * (1.0 / 19) for i in range(20)]
    assert [i for i in range(20) if recip[i] != O.alpha_grid(20)[i]] == [13, 17]


def test_scale_grid_closed_forms():
    rng = np.random.default_rng(2)
    abar = np.exp(rng.normal(0, 2, size=2000))
    abar[:5] = [0.0, 1e-9, 1e-4, 1.0, 300.0]
    S = O.scale_grid(abar, O.alpha_grid(3))   # alpha = 0, 0.5, 1
    floor = np.maximum(abar, 1e-4)
    assert np.all(S[0] == np.float32(1.0))                       # alpha = 0: plain RTN scale
    assert np.array_equal(S[2], floor.astype(np.float32))       # alpha = 1: s = abar
    assert np.array_equal(S[1], np.sqrt(floor).astype(np.float32))  # alpha = 1/2: sqrt
    assert S[0, 0] == 1.0 and S[2, 0] == np.float32(1e-4)


# --------------------------------------------------------------------------
# D4  quantiser
# --------------------------------------------------------------------------
HAND_WORKED = ["quant_group_int4.txt", "quant_group_int3.txt", "quant_group_clip.txt",
               "quant_group_clip_interior.txt",
               "quant_group_sym_int4.txt", "quant_group_sym_int3.txt", "quant_group_sym_clip.txt"]


@pytest.mark.parametrize("name", HAND_WORKED)
def test_quantiser_hand_worked(golden, name):
    hdr, rows = golden(name)
    g, b = int(hdr["group"]), int(hdr["w_bit"])
    zp = bool(int(hdr.get("zero_point", 1)))
    W = _group_row({int(r[0]): float(r[1]) for r in rows}, g)
    ratio = None
    if "clip_index" in hdr:
        r = O.clip_ratios(int(hdr["n_clip"]), 0.5)[int(hdr["clip_index"])]
        ratio = np.full((1, 1), np.float32(r), dtype=np.float32)
    qd = O.quantize_groups(W, None, g, b, ratio, zero_point=zp)
    assert qd["delta"][0, 0] == np.float32(float(hdr["delta"]))
    assert int(qd["z"][0, 0]) == int(hdr["zero"])
    for r in rows:
        j = int(r[0])
        assert int(qd["q"][0, j]) == int(r[2]), (name, j)
        assert float(qd["deq"][0, j]) == float(r[3]), (name, j)
    zero_code = int(hdr["zero"])
    listed = {int(r[0]) for r in rows}
    for j in range(g):
        if j not in listed:
            assert int(qd["q"][0, j]) == zero_code and qd["deq"][0, j] == 0.0


def _nearest_code_bruteforce(wt, delta, z, qmax):
    """Exact nearest point of the grid {(q - z) delta : 0 <= q <= qmax};
    a tie goes to even (q - z).  Returns (code, margin), margin being the
    exact distance of wt/delta from the nearest half-integer."""
    wt, delta = Fraction(float(wt)), Fraction(float(delta))
    best, bestd = None, None
    for q in range(qmax + 1):
        dist = abs((q - z) * delta - wt)
        if bestd is None or dist < bestd or (dist == bestd and (q - z) % 2 == 0):
            best, bestd = q, dist
    u = wt / delta
    margin = abs(u - (math.floor(u) + Fraction(1, 2)))
    return best, margin


@pytest.mark.parametrize("w_bit,group,zp", [(3, 128, True), (4, 128, True), (4, 32, True),
                                             (3, 64, True), (4, 128, False), (3, 32, False)])
def test_alpha0_is_plain_rtn_nearest_grid_point(w_bit, group, zp):
    """alpha = 0 reduces to plain round-to-nearest ("AWQ and Activation-Aware
    Scaling", Scaling instead of protecting): codes are the nearest in-range
    grid point, checked by exhaustive search in exact arithmetic."""
    X, W = random_layer(16, 256, 12, seed=11)
    abar = O.act_stats(X.numpy())
    S = O.scale_grid(abar, O.alpha_grid(20))
    Wn = W.numpy()
    q0 = O.quantize_groups(Wn, S[0], group, w_bit, zero_point=zp)
    qr = O.quantize_groups(Wn, None, group, w_bit, zero_point=zp)
    assert np.array_equal(q0["q"], qr["q"]) and np.array_equal(q0["delta"], qr["delta"])
    qmax = 2 ** w_bit - 1
    checked = 0
    for o in range(Wn.shape[0]):
        for j in range(Wn.shape[1]):
            k = j // group
            code, margin = _nearest_code_bruteforce(qr["wt"][o, j], qr["delta"][o, k], int(qr["z"][o, k]), qmax)
            if margin < Fraction(1, 2 ** 18):
                continue  # the fp32 quotient may round across a half-integer
            assert int(qr["q"][o, j]) == code, (o, j)
            checked += 1
    assert checked > 0.99 * Wn.size


@pytest.mark.parametrize("w_bit", [3, 4])
def test_half_step_bound(w_bit):
    """|deq - s w| <= delta / 2 (+ fp32 rounding) for groups whose range spans 0
    ("05 — AWQ" §3: rounding error at most half a step)."""
    X, W = random_layer(64, 512, 64, seed=3)
    abar = O.act_stats(X.numpy())
    S = O.scale_grid(abar, O.alpha_grid(20))
    for i in (0, 7, 19):
        qd = O.quantize_groups(W.numpy(), S[i], 128, w_bit)
        wt3 = qd["wt"].reshape(64, 4, 128)
        spans0 = (wt3.min(2) <= 0) & (wt3.max(2) >= 0)
        assert spans0.all()
        err = np.abs(qd["deq"].astype(np.float64) - qd["wt"]).reshape(64, 4, 128)
        bound = qd["delta"].astype(np.float64)[:, :, None] * (0.5 + 2.0 ** -18)
        assert np.all(err <= bound)


@pytest.mark.parametrize("w_bit", [3, 4])
def test_half_step_bound_without_zero_point(w_bit):
    """The symmetric scheme of "05 — AWQ" §3: every weight's rounding error
    is at most half a step, with no clamping at ratio 1 and no condition on the
    group's range (one-signed groups included); the codes stay in
    [1, 2^b - 1], symmetric about z = 2^(b-1)."""
    X, W = random_layer(64, 512, 64, seed=3)
    Wn = W.numpy().copy()
    Wn[:8] = np.abs(Wn[:8])  # one-signed rows
    abar = O.act_stats(X.numpy())
    S = O.scale_grid(abar, O.alpha_grid(20))
    for i in (0, 7, 19):
        qd = O.quantize_groups(Wn, S[i], 128, w_bit, zero_point=False)
        err = np.abs(qd["deq"].astype(np.float64) - qd["wt"]).reshape(64, 4, 128)
        bound = qd["delta"].astype(np.float64)[:, :, None] * (0.5 + 2.0 ** -18)
        assert np.all(err <= bound)
        assert np.all(qd["z"] == 2 ** (w_bit - 1))
        assert qd["q"].min() >= 1 and qd["q"].max() <= 2 ** w_bit - 1
        m = np.abs(qd["wt"]).reshape(64, 4, 128).max(2)
        assert np.array_equal(qd["delta"], (m / np.float32(2 ** (w_bit - 1) - 1)).astype(np.float32))


def test_constant_group_guard_without_zero_point():
    W = _group_row({}, 128, fill=0.25)
    qd = O.quantize_groups(W, None, 128, 4, zero_point=False)
    assert qd["delta"][0, 0] == np.float32(np.float32(0.25) / np.float32(7))
    assert np.all(qd["q"] == 15) and int(qd["z"][0, 0]) == 8
    W0 = _group_row({}, 128, fill=0.0)
    qd0 = O.quantize_groups(W0, None, 128, 4, zero_point=False)
    assert qd0["delta"][0, 0] == np.float32(np.float32(1e-5) / np.float32(7))
    assert np.all(qd0["q"] == 8) and np.all(qd0["deq"] == 0.0)


def test_one_signed_group_clamps():
    """A group with min > 0: the zero point clamps to 0 and codes clamp to
    2^b - 1 (the range is not widened to include 0)."""
    W = _group_row({j: 1.0 + j / 128.0 for j in range(128)}, 128)
    qd = O.quantize_groups(W, None, 128, 4)
    assert int(qd["z"][0, 0]) == 0
    delta = float(qd["delta"][0, 0])
    assert delta == float(np.float32(np.float32(1.0 + 127 / 128 - 1.0) / np.float32(15)))
    want = np.clip(np.rint(qd["wt"][0] / np.float32(delta)), 0, 15)
    assert np.array_equal(qd["q"][0], want.astype(np.uint8))
    assert qd["q"][0].max() == 15


def test_constant_group_guard():
    W = _group_row({}, 128, fill=0.25)
    qd = O.quantize_groups(W, None, 128, 4)
    assert qd["delta"][0, 0] == np.float32(np.float32(1e-5) / np.float32(15))
    assert int(qd["z"][0, 0]) == 0 and np.all(qd["q"] == 15)


@pytest.mark.parametrize("k,zp", [(-3, True), (4, True), (-5, False), (3, False)])
def test_power_of_two_scale_invariance(k, zp):
    """s -> 2^k s leaves codes and zeros unchanged and scales delta by 2^k
    exactly (every fp32 step commutes with an exact power-of-two scaling)."""
    X, W = random_layer(32, 256, 16, seed=5)
    abar = O.act_stats(X.numpy())
    s = O.scale_grid(abar, O.alpha_grid(20))[12]
    a = O.quantize_groups(W.numpy(), s, 128, 4, zero_point=zp)
    b = O.quantize_groups(W.numpy(), (s * np.float32(2.0 ** k)).astype(np.float32), 128, 4,
                          zero_point=zp)
    assert np.array_equal(a["q"], b["q"]) and np.array_equal(a["z"], b["z"])
    assert np.array_equal(a["delta"] * np.float32(2.0 ** k), b["delta"])


# --------------------------------------------------------------------------
# D5, D6  scoring and the alpha search
# --------------------------------------------------------------------------
def _literal_mse(X, W, s, deq):
    """The pages' score written literally: ((X diag(s)^-1) Qdeq^T - X W^T)^2
    averaged over tokens and outputs, fp64."""
    X64 = X.astype(np.float64)
    Yhat = (X64 / s.astype(np.float64)[None, :]) @ deq.astype(np.float64).T
    Y = X64 @ W.astype(np.float64).T
    return float(np.mean((Yhat - Y) ** 2))


def _pure_python_mse(X, W, s, deq):
    T, inn = X.shape
    out = W.shape[0]
    tot = 0.0
    for t in range(T):
        for o in range(out):
            yh = sum(float(X[t, j]) / float(s[j]) * float(deq[o, j]) for j in range(inn))
            y = sum(float(X[t, j]) * float(W[o, j]) for j in range(inn))
            tot += (yh - y) ** 2
    return tot / (T * out)


def test_scaling_invariance_identity():
    """X W^T = (X diag(s)^-1)(diag(s) W)^T in fp64 ("05 — AWQ" §3)."""
    X, W = random_layer(64, 256, 16, seed=6)
    abar = O.act_stats(X.numpy())
    s = O.scale_grid(abar, O.alpha_grid(20))[19].astype(np.float64)
    X64, W64 = X.numpy().astype(np.float64), W.numpy().astype(np.float64)
    a = X64 @ W64.T
    b = (X64 / s[None, :]) @ (W64 * s[None, :]).T
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(a))


def test_mse_forms_match_pure_python_definition():
    X, W = random_layer(6, 128, 8, seed=7)
    Xn, Wn = X.numpy(), W.numpy()
    abar = O.act_stats(Xn)
    S = O.scale_grid(abar, O.alpha_grid(20))
    for i in (0, 10, 19):
        qd = O.quantize_groups(Wn, S[i], 128, 4)
        want = _pure_python_mse(Xn, Wn, S[i], qd["deq"])
        delta = O.effective_error(Wn, S[i], qd["deq"])
        assert O.mse_direct(Xn, delta) == pytest.approx(want, rel=1e-10)
        assert O.mse_gram(O.gram(Xn), delta, Xn.shape[0]) == pytest.approx(want, rel=1e-10)


def test_fp16_output_score_is_exact_when_nothing_rounds():
    """The fp16-output reading of "05 — AWQ" §4 equals the exact score when the
    candidate weights and X W^T are fp16-representable: X in {-2..2}, W on a
    1/8 grid spanning [-1, 0.875] (so delta = 1.875 / 15 = 1/8 and deq = W),
    outputs multiples of 1/8 below 2^8."""
    rng = np.random.default_rng(21)
    T, inn, out = 24, 128, 16
    X = rng.integers(-2, 3, size=(T, inn)).astype(np.float16)
    W = (rng.integers(-8, 8, size=(out, inn)) / 8.0).astype(np.float16)
    W[:, 0], W[:, 1] = -1.0, 0.875
    qd = O.quantize_groups(W, None, 128, 4)
    assert np.all(qd["delta"] == np.float32(0.125)) and np.array_equal(qd["deq"], W.astype(np.float32))
    # perturb a few weights off the grid so the exact score is not zero
    W2 = W.copy()
    W2[:, 5] += np.float16(1.0 / 64)
    qd2 = O.quantize_groups(W2, None, 128, 4)
    exact = O.mse_direct(X, O.effective_error(W2, None, qd2["deq"]))
    assert exact > 0
    assert O.mse_fp16_output(X, W2, None, qd2["deq"]) == exact


def _ulp16(v):
    """Spacing of fp16 numbers around |v| (subnormal spacing 2^-24 below 2^-14)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return np.exp2(e - 10)


def test_fp16_output_score_within_half_ulp_bound():
    """|sqrt(N MSE16) - sqrt(N MSE)| <= || X u_B^T + u_Y ||_F, u being half an
    fp16 ulp of each rounded candidate weight and reference output: the only
    difference from the exact score is the two roundings (triangle
    inequality), whatever the scale s."""
    X, W = random_layer(40, 256, 24, seed=23)
    Xn, Wn = X.numpy(), W.numpy()
    abar = O.act_stats(Xn)
    S = O.scale_grid(abar, O.alpha_grid(20))
    X64, W64 = Xn.astype(np.float64), Wn.astype(np.float64)
    N = Xn.shape[0] * Wn.shape[0]
    for i in (0, 9, 19):
        qd = O.quantize_groups(Wn, S[i], 128, 4)
        exact = O.mse_direct(Xn, O.effective_error(Wn, S[i], qd["deq"]))
        m16 = O.mse_fp16_output(Xn, Wn, S[i], qd["deq"])
        B = qd["deq"] / S[i][None, :]
        uB = _ulp16(B) / 2 * (1 + 2.0 ** -20)
        uY = _ulp16(X64 @ W64.T) / 2
        bound = np.sqrt(np.sum((np.abs(X64) @ uB.T + uY) ** 2))
        assert abs(np.sqrt(N * m16) - np.sqrt(N * exact)) <= bound
        assert m16 != exact  # the roundings are there


@pytest.mark.parametrize("T,inn,out,w_bit,zp", [(64, 128, 16, 4, True), (48, 256, 8, 3, True),
                                                (33, 256, 16, 4, True), (40, 256, 8, 4, False),
                                                (24, 128, 16, 3, False)])
def test_search_bruteforce_tiny(T, inn, out, w_bit, zp):
    X, W = random_layer(T, inn, out, seed=T + inn + out + w_bit)
    Xn, Wn = X.numpy(), W.numpy()
    abar = O.act_stats(Xn)
    mse, best, s_best, S = O.search_scale(Xn, Wn, abar, w_bit, 128, 20, form="direct", zero_point=zp)
    mse_g, best_g, _, _ = O.search_scale(Xn, Wn, abar, w_bit, 128, 20, form="gram", zero_point=zp)
    lit = np.array([_literal_mse(Xn, Wn, S[i], O.quantize_groups(Wn, S[i], 128, w_bit, zero_point=zp)["deq"])
                    for i in range(20)])
    assert np.allclose(mse, lit, rtol=1e-10, atol=0)
    assert np.allclose(mse_g, lit, rtol=1e-10, atol=0)
    assert best == int(np.argmin(lit)) == best_g
    assert np.array_equal(s_best, S[best])


def test_ties_resolve_to_lowest_alpha():
    """abar = 1 everywhere makes s = 1 for every alpha: all scores are equal
    bit for bit and the search keeps alpha = 0."""
    T, inn = 32, 256
    X = np.where(np.arange(T * inn).reshape(T, inn) % 2 == 0, 1.0, -1.0).astype(np.float16)
    _, W = random_layer(4, inn, 8, seed=9)
    abar = O.act_stats(X)
    assert np.all(abar == 1.0)
    mse, best, s_best, _ = O.search_scale(X, W.numpy(), abar, 4, 128, 20)
    assert np.all(mse == mse[0]) and best == 0 and np.all(s_best == 1.0)


def test_search_beats_rtn_on_heavy_tailed_tiny_workload():
    """Qualitative expectations on heavy-tailed activations ("AWQ and
    Activation-Aware Scaling"): scaling improves on plain RTN (alpha = 0) and
    alpha = 1 over-corrects relative to the optimum."""
    X = heavy_tailed_activations(256, 512, OutlierSpec(0.01, 20.0), 0)
    W = gaussian_weight(512, 512, 0)
    Xn, Wn = X.numpy(), W.numpy()
    mse, best, _, _ = O.search_scale(Xn, Wn, O.act_stats(Xn), 4, 128, 20)
    assert mse[best] < mse[0] and mse[best] < mse[-1] and 0 < best < 19


# --------------------------------------------------------------------------
# D7  clip search
# --------------------------------------------------------------------------
def test_clip_ratio_grid():
    r = O.clip_ratios(20, 0.5)
    assert r[0] == 1.0 and r[-1] == 0.5 and np.all(np.diff(r) < 0)
    assert list(O.clip_ratios(1, 0.5)) == [1.0]


def _rn32_exact(x: Fraction) -> Fraction:
    """Round-half-to-even of a positive rational to the fp32 grid (normal
    range), in exact arithmetic."""
    e = math.floor(math.log2(x))
    while Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    m = x / Fraction(2) ** (e - 23)
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl * Fraction(2) ** (e - 23)


@pytest.mark.parametrize("n_clip,clip_min", [(20, 0.5), (7, 0.5), (2, 0.5)])
def test_clip_ratio_grid_closed_form(n_clip, clip_min):
    """Every ratio of the grid, interior ones included, is the fp32 rounding
    of the exact 1 - c (1 - clip_min)/(n_clip - 1) ("05 — AWQ" §4: ratios of
    0.5 - 1.0).  At 20 ratios an fp32 evaluation of the formula, or an fp32
    linspace, misses it at c = 8, 11, 15, 17 (one ulp)."""
    r = O.clip_ratios(n_clip, clip_min).astype(np.float32)
    cm = Fraction(float(np.float32(clip_min)))
    for c in range(n_clip):
        want = _rn32_exact(1 - c * (1 - cm) / (n_clip - 1))
        assert Fraction(float(r[c])) == want, (c, float(r[c]), float(want))
    if n_clip == 20:
        lin = np.linspace(np.float32(1), np.float32(0.5), 20, dtype=np.float32)
        f32 = np.float32(1) - np.arange(20, dtype=np.float32) * np.float32(0.5) / np.float32(19)
        assert sorted(set(np.flatnonzero(lin != r)) | set(np.flatnonzero(f32 != r))) == [8, 11, 15, 17]


def test_fold_rounding_chain_hand_worked(golden):
    """The fold rounds the quotient to fp32, then to fp16; the fixture's value
    sits where one rounding, or the product with a rounded reciprocal, gives
    the other fp16 neighbour."""
    hdr, _ = golden("fold_rounding.txt")
    v = np.array([int(hdr["v_hex"], 16)], dtype=np.uint16).view(np.float16)
    s = np.array([int(hdr["s_hex"], 16)], dtype=np.uint32).view(np.float32)
    got = O.fold_inv_scale(v, s).view(np.uint16)[0]
    assert got == int(hdr["folded_hex"], 16)
    one = np.float16(Fraction(float(v[0])) / Fraction(float(s[0])))  # RN16 of the exact quotient
    assert abs(Fraction(float(v[0])) / Fraction(float(s[0])) - Fraction(float(one))) < Fraction(1, 2 ** 14)
    assert one.view(np.uint16) == int(hdr["one_rounding_hex"], 16)
    rec = np.float16(np.float32(v[0]) * (np.float32(1) / s[0]))
    assert rec.view(np.uint16) == int(hdr["reciprocal_hex"], 16)


def test_clip_ratio_one_is_unclipped():
    X, W = random_layer(16, 256, 8, seed=12)
    abar = O.act_stats(X.numpy())
    s = O.scale_grid(abar, O.alpha_grid(20))[9]
    a = O.quantize_groups(W.numpy(), s, 128, 4)
    b = O.quantize_groups(W.numpy(), s, 128, 4, np.ones((8, 2), np.float32))
    for key in ("q", "z", "delta", "deq"):
        assert np.array_equal(a[key], b[key])


@pytest.mark.parametrize("zp,group", [(True, 128), (False, 128), (True, 32), (False, 64)])
def test_clip_search_bruteforce_tokens(zp, group):
    T, inn, out, nc = 40, 256, 8, 6
    X, W = random_layer(T, inn, out, seed=13)
    Xn, Wn = X.numpy(), W.numpy()
    s = O.scale_grid(O.act_stats(Xn), O.alpha_grid(20))[8]
    idx, E = O.search_clip(Xn, Wn, s, 4, group, nc, 0.5, zero_point=zp)
    r = O.clip_ratios(nc, 0.5).astype(np.float32)
    X64 = Xn.astype(np.float64)
    ng = inn // group
    for c in range(nc):
        qd = O.quantize_groups(Wn, s, group, 4, np.full((out, ng), r[c], np.float32), zero_point=zp)
        for o in range(out):
            for k in range(ng):
                sl = slice(group * k, group * (k + 1))
                d = qd["deq"][o, sl].astype(np.float64) / s[sl].astype(np.float64) - Wn[o, sl].astype(np.float64)
                e = float(np.sum((X64[:, sl] @ d) ** 2))
                assert E[o, k, c] == pytest.approx(e, rel=1e-10)
    assert np.array_equal(idx, np.argmin(E, axis=2))


# --------------------------------------------------------------------------
# D8  packing
# --------------------------------------------------------------------------
def test_pack_hand_worked(golden):
    hdr, rows = golden("pack_int4.txt")
    out, inn = int(hdr["out"]), int(hdr["in"])
    W = np.zeros((out, inn), dtype=np.float16)
    for o in range(out):
        for j in range(8):
            W[o, j] = ((o + j) % 16) - 8
        W[o, 126], W[o, 127] = -8.0, 7.0
    qweight, qzeros, scales = O.quant_pack(W, None, None, 4, 128)
    assert qweight.shape == (inn, out // 8) and qzeros.shape == (1, 1) and scales.shape == (1, out)
    for r in rows:
        assert int(qweight.view(np.uint32)[int(r[0]), 0]) == int(r[1], 16), r
    assert int(qzeros.view(np.uint32)[0, 0]) == int(hdr["qzeros_hex"], 16)
    assert np.all(scales == np.float16(float(hdr["scale"])))


def test_pack_roundtrip_and_storage_bits(golden):
    hdr, _ = golden("storage_bits.txt")
    X, W = random_layer(16, 512, 64, seed=15)
    Wn = W.numpy()
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[11]
    idx = np.random.default_rng(0).integers(0, 20, size=(64, 4)).astype(np.uint8)
    qweight, qzeros, scales = O.quant_pack(Wn, s, idx, 3, 128, 20, 0.5)
    r = O.clip_ratios(20, 0.5).astype(np.float32)[idx.astype(np.int64)]
    qd = O.quantize_groups(Wn, s, 128, 3, r)
    assert np.array_equal(O.unpack_nibbles(qweight), qd["q"])
    assert np.array_equal(O.unpack_nibbles(qzeros), qd["z"])
    assert np.array_equal(scales, qd["delta"].T.astype(np.float16))
    assert O.unpack_nibbles(qweight).max() <= 7
    g = int(hdr["group"])
    Xg, Wg = random_layer(4, 1024, 256, seed=16)
    qw, qz, sc = O.quant_pack(Wg.numpy(), None, None, 4, g)
    bits = 8.0 * (qw.nbytes + qz.nbytes + sc.nbytes) / Wg.numel()
    assert bits == float(hdr["bits_per_weight"])
    assert round(bits, 3) == float(hdr["printed"])
    # the same closed form, 4 + 16/g + 4/g, at the other group sizes
    for gs in (32, 64):
        qw, qz, sc = O.quant_pack(Wg.numpy(), None, None, 4, gs)
        assert 8.0 * (qw.nbytes + qz.nbytes + sc.nbytes) / Wg.numel() == 4 + 16 / gs + 4 / gs


def test_fold_keeps_the_product():
    """Folding 1/s into the preceding op keeps the layer's function
    ("AWQ and Activation-Aware Scaling"): (gamma / s) * (s w) = gamma * w up to
    the fp16 rounding of the folded vector."""
    rng = np.random.default_rng(3)
    gamma = rng.uniform(0.5, 1.5, 256).astype(np.float16)
    s = np.exp(rng.normal(0, 1, 256)).astype(np.float32)
    g2 = O.fold_inv_scale(gamma, s)
    assert np.allclose(g2.astype(np.float64) * s, gamma.astype(np.float64), rtol=2 ** -10)
    rows = rng.normal(0, 0.02, (256, 64)).astype(np.float16)
    r2 = O.fold_inv_scale(rows, s)
    # half an fp16 ulp of the folded value (relative 2^-11, or 2^-25 absolute in
    # the subnormal range), carried back through the multiplication by s
    err = np.abs(r2.astype(np.float64) * s[:, None] - rows.astype(np.float64))
    assert np.all(err <= 2.0 ** -11 * np.abs(rows.astype(np.float64)) * 1.001 + 2.0 ** -25 * s[:, None])


@pytest.mark.parametrize("w_bit", [3, 4])
def test_pack_without_zero_point(w_bit):
    """Without a zero point every qzeros nibble holds 2^(b-1) (0x88888888 per
    word at INT4), the codes round-trip, and (q - z) scale gives back the
    fp32 dequantised weights up to the fp16 rounding of the scale."""
    X, W = random_layer(16, 256, 32, seed=17)
    Wn = W.numpy()
    s = O.scale_grid(O.act_stats(X.numpy()), O.alpha_grid(20))[6]
    qw, qz, sc = O.quant_pack(Wn, s, None, w_bit, 128, zero_point=False)
    nib = 2 ** (w_bit - 1)
    assert np.all(O.unpack_nibbles(qz) == nib)
    assert np.all(qz.view(np.uint32) == np.uint32(int(("%x" % nib) * 8, 16)))
    q = O.unpack_nibbles(qw).astype(np.int64)  # [out, in]
    qd = O.quantize_groups(Wn, s, 128, w_bit, zero_point=False)
    assert np.array_equal(q, qd["q"])
    deq16 = (q - nib) * np.repeat(sc.T.astype(np.float64), 128, axis=1)
    assert np.allclose(deq16, qd["deq"], rtol=2.0 ** -10, atol=0)


# --------------------------------------------------------------------------
# The W4A16 product on the packed output
# --------------------------------------------------------------------------
def test_w4a16_exact_on_the_hand_worked_packing(golden):
    """The hand-worked packing example has step 1 and zero 8, so the packed
    weights dequantise to W itself; with integer X the product is exact."""
    W = np.zeros((16, 128), dtype=np.float16)
    for o in range(16):
        for j in range(8):
            W[o, j] = ((o + j) % 16) - 8
        W[o, 126], W[o, 127] = -8.0, 7.0
    qw, qz, sc = O.quant_pack(W, None, None, 4, 128)
    assert np.all(sc == np.float16(1.0))
    assert np.array_equal(O.dequant_packed(qw, qz, sc, 128), W)
    X = np.random.default_rng(3).integers(-3, 4, size=(9, 128)).astype(np.float16)
    want = X.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(O.w4a16_matmul(X, qw, qz, sc, 128), want.astype(np.float64))


@pytest.mark.parametrize("w_bit,group,zp", [(4, 128, True), (3, 64, True), (4, 32, False)])
def test_w4a16_weights_within_half_a_step(w_bit, group, zp):
    """Dequantised packed weights sit within half a step of the weights they
    came from (s = 1, no clip, groups spanning 0), up to the fp16 rounding of
    the stored step and of the product."""
    _, W = random_layer(4, 256, 32, seed=19)
    Wn = W.numpy()
    qw, qz, sc = O.quant_pack(Wn, None, None, w_bit, group, zero_point=zp)
    Wd = O.dequant_packed(qw, qz, sc, group).astype(np.float64)
    step = np.repeat(sc.astype(np.float64).T, group, axis=1)
    qmax = 2 ** w_bit - 1
    bound = step * (0.5 + qmax * 2.0 ** -11) + np.abs(Wd) * 2.0 ** -11
    assert np.all(np.abs(Wd - Wn.astype(np.float64)) <= bound)
