"""Seeded synthetic calibration inputs for the AWQ per-layer scale search.

This module draws random numbers and shapes them like the workloads the AWQ
pages describe; it performs none of the method's arithmetic (no statistic, no
scale, no quantisation).  Both the CPU oracle and the CUDA path consume what it
returns, so it is the only code the two sides share.

Recipe (the pages calibrate on ~128 samples of an unnamed text set, "05 — AWQ"
study notes §4; no dataset or trained weight is available, so these stand in):

* heavy-tailed activations  X[t, j] = RN16(z[t, j] * c[j]) with z ~ N(0, 1) and
  c[j] = exp(0.5 * n[j]), n ~ N(0, 1) (log-normal(0, 0.5) channel scales); a set
  of round(p * d) outlier channels, drawn without replacement, has c[j]
  multiplied by m[j] (a constant or U[lo, hi]);  salient channels are the ~0.1–1 %
  with large activations ("AWQ and Activation-Aware Scaling", The observation).
* weights  W = RN16(0.02 * N(0, 1)), laid out [out, in] like nn.Linear.

All draws are fp32 from ``torch.Generator('cpu')`` and are rounded once to fp16.
Each tensor gets its own generator, derived from the config seed, so that a
tensor does not change when another one's shape does.
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import torch

__all__ = [
    "OutlierSpec",
    "EDGE_PATTERNS",
    "edge_layer",
    "heavy_tailed_activations",
    "gaussian_weight",
    "swiglu_activations",
    "Workload",
    "WORKLOADS",
    "workload_inputs",
    "DecoderSpec",
    "decoder_layer_weights",
    "decoder_embeddings",
    "decoder_layer_forward",
]


@dataclasses.dataclass(frozen=True)
class OutlierSpec:
    """Outlier channels: ``round(frac * d)`` channels multiplied by ``lo`` (if
    ``hi`` is None) or by U[lo, hi]."""

    frac: float
    lo: float
    hi: Optional[float] = None


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def channel_profile(d: int, outliers: OutlierSpec, seed: int) -> torch.Tensor:
    """Per-channel magnitudes c[j] (fp32 [d]) of the heavy-tailed recipe."""
    g = _gen(seed)
    c = torch.exp(0.5 * torch.randn(d, generator=g, dtype=torch.float32))
    n_out = int(round(outliers.frac * d))
    if n_out > 0:
        idx = torch.randperm(d, generator=g)[:n_out]
        if outliers.hi is None:
            m = torch.full((n_out,), float(outliers.lo), dtype=torch.float32)
        else:
            m = outliers.lo + (outliers.hi - outliers.lo) * torch.rand(
                n_out, generator=g, dtype=torch.float32)
        c[idx] = c[idx] * m
    return c


def heavy_tailed_activations(T: int, d: int, outliers: OutlierSpec, seed: int,
                             chunk: int = 8192) -> torch.Tensor:
    """Calibration activations X [T, d] fp16 (CPU), token-major.

    Rows are drawn in chunks of ``chunk`` tokens, each chunk from its own
    generator, so the first T' rows do not depend on T."""
    c = channel_profile(d, outliers, seed)
    X = torch.empty((T, d), dtype=torch.float16)
    for i, t0 in enumerate(range(0, T, chunk)):
        t1 = min(T, t0 + chunk)
        g = _gen(seed * 1_000_003 + 17 + i)
        z = torch.randn((t1 - t0, d), generator=g, dtype=torch.float32)
        X[t0:t1] = (z * c).to(torch.float16)
    return X


def gaussian_weight(out: int, inn: int, seed: int, std: float = 0.02) -> torch.Tensor:
    """Weight W [out, in] fp16 (CPU), entries RN16(std * N(0, 1))."""
    g = _gen(seed * 1_000_003 + 5)
    return (std * torch.randn((out, inn), generator=g, dtype=torch.float32)).to(torch.float16)


def swiglu_activations(X: torch.Tensor, W_gate: torch.Tensor, W_up: torch.Tensor,
                       outliers: OutlierSpec, seed: int, device: str = "cpu",
                       chunk: int = 4096) -> torch.Tensor:
    """Input of a down projection: SiLU(X W_gate^T) * (X W_up^T) in fp32,
    divided by its global RMS (keeps the product inside fp16's range once the
    outlier profile is applied), multiplied by its own heavy-tailed channel
    profile, rounded once to fp16.  Returns a CPU tensor [T, d_ff].

    This is the model's forward pass (synthetic input), not part of AWQ."""
    T = X.shape[0]
    d_ff = W_gate.shape[0]
    c = channel_profile(d_ff, outliers, seed).to(device)
    wg = W_gate.to(device=device, dtype=torch.float32)
    wu = W_up.to(device=device, dtype=torch.float32)
    sq = torch.zeros((), dtype=torch.float64, device=device)
    parts = []
    for t0 in range(0, T, chunk):
        x = X[t0:t0 + chunk].to(device=device, dtype=torch.float32)
        h = torch.nn.functional.silu(x @ wg.T) * (x @ wu.T)
        sq += (h.double() ** 2).sum()
        parts.append(h)
    rms = float(torch.sqrt(sq / (T * d_ff)))
    out = torch.empty((T, d_ff), dtype=torch.float16)
    t0 = 0
    for h in parts:
        out[t0:t0 + h.shape[0]] = ((h / rms) * c).to(torch.float16).cpu()
        t0 += h.shape[0]
    return out


@dataclasses.dataclass(frozen=True)
class Workload:
    """One of the five benchmark workloads (shapes and value recipes)."""

    name: str
    T: int
    w_bit: int
    group_size: int
    n_alpha: int
    n_clip: int
    seed: int
    description: str


WORKLOADS: Tuple[Workload, ...] = (
    Workload("tiny_linear_512", 256, 4, 128, 20, 0, 0,
             "X [256 x 512], W [512 x 512], 5 outlier channels x20, INT4 g128, 20 alphas, no clip"),
    Workload("llama7b_q_proj_4096", 65536, 4, 128, 20, 20, 1,
             "X [65536 x 4096], W [4096 x 4096], 41 outlier channels x U[20,50], INT4 g128, "
             "20 alphas + 20 clip ratios, packed"),
    Workload("llama7b_mlp_4096_11008", 65536, 4, 128, 20, 0, 2,
             "X [65536 x 4096]; gate|up [22016 x 4096] jointly; down [4096 x 11008] on the "
             "SwiGLU output; INT4 g128, 20 alphas"),
    Workload("llama13b_attn_5120_int3", 65536, 3, 128, 20, 20, 3,
             "X [65536 x 5120] (5 outlier channels x50); qkv [15360 x 5120]; o_proj [5120 x 5120] "
             "on its own X; INT3 g128, 20 alphas + 20 clip ratios"),
)


def workload_inputs(index: int, T: Optional[int] = None, device: str = "cpu") -> dict:
    """Inputs of workload ``index`` (0-based into WORKLOADS) as CPU fp16 tensors.

    Returns {"groups": [(name, X, W), ...], "workload": Workload}.  Joint
    scaling groups are returned with their weights already concatenated along
    ``out`` (they share one scale vector).  ``T`` overrides the token count
    (smaller parity cases of the same structure); ``device`` is only used for
    the SwiGLU forward of workload 2."""
    wl = WORKLOADS[index]
    T = wl.T if T is None else int(T)
    s = wl.seed
    if index == 0:
        X = heavy_tailed_activations(T, 512, OutlierSpec(0.01, 20.0), s)
        W = gaussian_weight(512, 512, s)
        return {"groups": [("linear", X, W)], "workload": wl}
    if index == 1:
        X = heavy_tailed_activations(T, 4096, OutlierSpec(0.01, 20.0, 50.0), s)
        W = gaussian_weight(4096, 4096, s)
        return {"groups": [("q_proj", X, W)], "workload": wl}
    if index == 2:
        X = heavy_tailed_activations(T, 4096, OutlierSpec(0.01, 20.0, 50.0), s)
        Wg = gaussian_weight(11008, 4096, s * 10 + 1)
        Wu = gaussian_weight(11008, 4096, s * 10 + 2)
        Wd = gaussian_weight(4096, 11008, s * 10 + 3)
        Xd = swiglu_activations(X, Wg, Wu, OutlierSpec(0.01, 20.0, 50.0), s * 10 + 4, device=device)
        return {"groups": [("gate_up", X, torch.cat([Wg, Wu], 0)), ("down_proj", Xd, Wd)],
                "workload": wl}
    if index == 3:
        X = heavy_tailed_activations(T, 5120, OutlierSpec(0.001, 50.0), s)
        Wqkv = gaussian_weight(15360, 5120, s * 10 + 1)
        Xo = heavy_tailed_activations(T, 5120, OutlierSpec(0.001, 50.0), s + 100)
        Wo = gaussian_weight(5120, 5120, s * 10 + 2)
        return {"groups": [("qkv", X, Wqkv), ("o_proj", Xo, Wo)], "workload": wl}
    raise ValueError(f"no workload {index}")


def random_layer(T: int, d_in: int, d_out: int, seed: int,
                 outliers: OutlierSpec = OutlierSpec(0.01, 20.0, 50.0),
                 w_std: float = 0.02) -> Tuple[torch.Tensor, torch.Tensor]:
    """A small (X, W) pair of arbitrary shape with the same recipe, for
    parity and edge-case tests."""
    X = heavy_tailed_activations(T, d_in, outliers, seed)
    W = gaussian_weight(d_out, d_in, seed, std=w_std)
    return X, W


# Weight-group patterns of edge_layer (name, description):
EDGE_PATTERNS = (
    ("normal", "N(0, 0.02)"),
    ("pos_narrow", "0.5 + 0.001 U: one-signed, range far below the values"),
    ("neg_narrow", "-0.25 - 0.0005 U: one-signed negative, narrow"),
    ("pos_wide", "0.01 + 0.02 U: one-signed, range wider than the offset"),
    ("const", "the constant 0.03"),
    ("zero", "all zeros"),
    ("const_pow2", "the constant -0.0625"),
    ("tiny", "1e-4 N(0, 1): partly fp16 subnormals"),
    ("spike", "N(0, 0.02) with one weight set to 0.3"),
)


def edge_layer(T: int, d_in: int, d_out: int, seed: int, group: int = 128
               ) -> Tuple[torch.Tensor, torch.Tensor]:
    """An (X, W) pair that reaches the quantiser's and the search's special
    cases, for edge-case tests.

    X is heavy_tailed_activations with dead channels: columns 0..2 are zero
    (mean |x| = 0), columns group+1..group+3 (if present) are ~1e-5 (mean |x|
    below 1e-4), and, when d_in >= 3 group, the whole group 2 is zero.
    W has one pattern of EDGE_PATTERNS per (row o, group k), pattern number
    (5 o + 3 k) mod 9, so every group column and every row meets several."""
    X = heavy_tailed_activations(T, d_in, OutlierSpec(0.01, 20.0, 50.0), seed)
    X[:, 0:3] = 0
    if d_in >= 2 * group:
        tiny = torch.randn((T, 3), generator=_gen(seed + 11)) * 1e-5
        X[:, group + 1:group + 4] = tiny.to(torch.float16)
    if d_in >= 3 * group:
        X[:, 2 * group:3 * group] = 0
    n_groups = d_in // group
    W = torch.randn((d_out, d_in), generator=_gen(seed + 12)) * 0.02
    u = torch.rand((d_out, d_in), generator=_gen(seed + 13))
    z = torch.randn((d_out, d_in), generator=_gen(seed + 14))
    pos = torch.randint(0, group, (d_out, n_groups), generator=_gen(seed + 15))
    for o in range(d_out):
        for k in range(n_groups):
            sl = slice(k * group, (k + 1) * group)
            p = EDGE_PATTERNS[(5 * o + 3 * k) % len(EDGE_PATTERNS)][0]
            if p == "pos_narrow":
                W[o, sl] = 0.5 + 0.001 * u[o, sl]
            elif p == "neg_narrow":
                W[o, sl] = -0.25 - 0.0005 * u[o, sl]
            elif p == "pos_wide":
                W[o, sl] = 0.01 + 0.02 * u[o, sl]
            elif p == "const":
                W[o, sl] = 0.03
            elif p == "zero":
                W[o, sl] = 0.0
            elif p == "const_pow2":
                W[o, sl] = -0.0625
            elif p == "tiny":
                W[o, sl] = 1e-4 * z[o, sl]
            elif p == "spike":
                W[o, k * group + int(pos[o, k])] = 0.3
    return X, W.to(torch.float16)


# ---------------------------------------------------------------------------
# Synthetic Llama-2-7B-architecture decoder (random init) for layer-by-layer
# calibration captures.  This is the model's fp16 forward pass (input
# synthesis), not AWQ: hidden states propagate through the unmodified layer.
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class DecoderSpec:
    hidden: int = 4096
    heads: int = 32
    ffn: int = 11008
    layers: int = 32
    vocab: int = 32000
    seq: int = 512
    n_seq: int = 128
    rope_theta: float = 10000.0
    eps: float = 1e-5
    w_std: float = 0.02
    outliers: OutlierSpec = OutlierSpec(0.01, 20.0, 50.0)
    seed: int = 4


def decoder_layer_weights(spec: DecoderSpec, layer: int, device: str = "cpu") -> dict:
    """fp16 weights of one decoder layer, N(0, w_std), nn.Linear layout
    [out, in]; RMSNorm gammas are 1.  Drawn on `device` with a generator of
    that device seeded from (spec.seed, layer), so a CUDA device gives the
    same weights on every run of the same build."""
    h, f = spec.hidden, spec.ffn
    shapes = {"q": (h, h), "k": (h, h), "v": (h, h), "o": (h, h), "gate": (f, h), "up": (f, h),
              "down": (h, f)}
    g = torch.Generator(device=device)
    g.manual_seed(spec.seed * 100_000 + layer)
    w = {name: (spec.w_std * torch.randn(shp, generator=g, dtype=torch.float32, device=device)
                ).to(torch.float16) for name, shp in shapes.items()}
    w["gamma1"] = torch.ones(h, dtype=torch.float16, device=device)
    w["gamma2"] = torch.ones(h, dtype=torch.float16, device=device)
    return w


def decoder_embeddings(spec: DecoderSpec, n_seq: Optional[int] = None, device: str = "cpu") -> torch.Tensor:
    """Calibration input of layer 0: n_seq random token sequences of spec.seq
    tokens looked up in a random N(0, w_std) embedding table whose outlier
    channels are multiplied by U[lo, hi]; fp16 [n_seq * seq, hidden]."""
    n_seq = spec.n_seq if n_seq is None else n_seq
    g = _gen(spec.seed * 1_000_003 + 11)
    ids = torch.randint(0, spec.vocab, (n_seq * spec.seq,), generator=g)
    table = spec.w_std * torch.randn((spec.vocab, spec.hidden), generator=g, dtype=torch.float32)
    n_out = int(round(spec.outliers.frac * spec.hidden))
    idx = torch.randperm(spec.hidden, generator=g)[:n_out]
    mult = spec.outliers.lo + (spec.outliers.hi - spec.outliers.lo) * torch.rand(n_out, generator=g)
    table[:, idx] *= mult
    return table.to(torch.float16)[ids].to(device)


def _rms_norm(x: torch.Tensor, gamma: torch.Tensor, eps: float) -> torch.Tensor:
    xf = x.float()
    return (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + eps) * gamma.float()).to(torch.float16)


def _rope(x: torch.Tensor, theta: float) -> torch.Tensor:
    # x: [B, heads, S, d]
    d = x.shape[-1]
    pos = torch.arange(x.shape[-2], device=x.device, dtype=torch.float32)
    inv = theta ** (-torch.arange(0, d, 2, device=x.device, dtype=torch.float32) / d)
    ang = pos[:, None] * inv[None, :]
    cos, sin = ang.cos(), ang.sin()
    xf = x.float()
    x1, x2 = xf[..., ::2], xf[..., 1::2]
    out = torch.empty_like(xf)
    out[..., ::2] = x1 * cos - x2 * sin
    out[..., 1::2] = x1 * sin + x2 * cos
    return out.to(torch.float16)


@torch.no_grad()
def decoder_layer_forward(x: torch.Tensor, w: dict, spec: DecoderSpec):
    """One fp16 decoder layer (RMSNorm, RoPE causal attention, SwiGLU MLP).
    Returns (captures, x_next) where captures holds the inputs of the four
    linear groups: 'qkv' (RMSNorm1 output), 'o' (attention output), 'gate_up'
    (RMSNorm2 output), 'down' (SiLU(gate) * up)."""
    T, h = x.shape
    B, S, H = T // spec.seq, spec.seq, spec.heads
    d = h // H
    a_in = _rms_norm(x, w["gamma1"], spec.eps)
    q = (a_in @ w["q"].T).view(B, S, H, d).transpose(1, 2)
    k = (a_in @ w["k"].T).view(B, S, H, d).transpose(1, 2)
    v = (a_in @ w["v"].T).view(B, S, H, d).transpose(1, 2)
    q, k = _rope(q, spec.rope_theta), _rope(k, spec.rope_theta)
    att = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    o_in = att.transpose(1, 2).reshape(T, h).contiguous()
    x = x + o_in @ w["o"].T
    m_in = _rms_norm(x, w["gamma2"], spec.eps)
    d_in = (torch.nn.functional.silu((m_in @ w["gate"].T).float()) * (m_in @ w["up"].T).float()).to(torch.float16)
    x = x + d_in @ w["down"].T
    return {"qkv": a_in, "o": o_in, "gate_up": m_in, "down": d_in.contiguous()}, x
