"""Seeded synthetic inputs for the TTT layer, shared by the tests, the smoke check and the
benchmark.  This module only draws random numbers: it holds none of the layer's arithmetic.

Recipe (one torch CPU generator per call, seeded): draw Q, K, V, then the inner weights, in
that order, each as standard-normal float32, scale it to the stated spread, then round to
the stated storage dtype (round-to-nearest-even).  The oracle and the GPU receive the
identical stored values.

Shapes and spreads follow the layer's workloads: a 224x224 image at patch 16 gives a 14x14
token grid (N = 196); the high-resolution stage-1 grid is 56x56 (N = 3136) with C = 64; a
1280x1280 image at patch 16 gives 80x80 (N = 6400).
"""
from __future__ import annotations

import math

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(shape, g, scale, dtype):
    return (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(dtype).contiguous()


def linear_inputs(B, H, N, d, dtype="bf16", seed=0, qkv_scale=None, w_scale=None):
    """Q, K, V [B,H,N,d] ~ N(0,1)/sqrt(d) in `dtype`; W0 [H,d,d] fp32 ~ N(0, 1/d)."""
    g = _gen(seed)
    dt = DTYPES[dtype]
    s = 1.0 / math.sqrt(d) if qkv_scale is None else qkv_scale
    ws = 1.0 / math.sqrt(d) if w_scale is None else w_scale
    q = _randn((B, H, N, d), g, s, dt)
    k = _randn((B, H, N, d), g, s, dt)
    v = _randn((B, H, N, d), g, s, dt)
    w0 = _randn((H, d, d), g, ws, torch.float32)
    return {"q": q, "k": k, "v": v, "w0": w0}


def dwconv_inputs(B, Hg, Wg, C, dtype="bf16", seed=0, qkv_scale=1.0, w_scale=1.0 / 3.0):
    """Q, K, V [B,Hg,Wg,C] (channels-last) ~ N(0,1) in `dtype`; taps [C,3,3] fp32 ~ N(0,1/9)."""
    g = _gen(seed)
    dt = DTYPES[dtype]
    q = _randn((B, Hg, Wg, C), g, qkv_scale, dt)
    k = _randn((B, Hg, Wg, C), g, qkv_scale, dt)
    v = _randn((B, Hg, Wg, C), g, qkv_scale, dt)
    w0 = _randn((C, 3, 3), g, w_scale, torch.float32)
    return {"q": q, "k": k, "v": v, "w0": w0}


def mlp_inputs(B, H, N, d, hidden=None, dtype="bf16", seed=0):
    """Q, K, V ~ N(0,1)/sqrt(d); W1 [H,d,h] ~ N(0,1/d); W2 [H,h,d] ~ N(0,1/h); h = 4d."""
    h = 4 * d if hidden is None else hidden
    g = _gen(seed)
    dt = DTYPES[dtype]
    s = 1.0 / math.sqrt(d)
    q = _randn((B, H, N, d), g, s, dt)
    k = _randn((B, H, N, d), g, s, dt)
    v = _randn((B, H, N, d), g, s, dt)
    w1 = _randn((H, d, h), g, 1.0 / math.sqrt(d), torch.float32)
    w2 = _randn((H, h, d), g, 1.0 / math.sqrt(h), torch.float32)
    return {"q": q, "k": k, "v": v, "w1": w1, "w2": w2}


def chunked_inputs(B, H, N, d, dtype="bf16", seed=0):
    """Same recipe as :func:`linear_inputs` (the chunked scan is a TTT-Linear variant)."""
    return linear_inputs(B, H, N, d, dtype=dtype, seed=seed)


def linear_bwd_inputs(B, H, N, d, dtype="bf16", seed=0):
    """The TTT-Linear inputs plus an upstream gradient dO [B,H,N,d] ~ N(0,1)/sqrt(d) in `dtype`
    (drawn from its own stream after the layer's inputs)."""
    inp = linear_inputs(B, H, N, d, dtype=dtype, seed=seed)
    g = _gen(seed + 104729)
    inp["dout"] = _randn((B, H, N, d), g, 1.0 / math.sqrt(d), DTYPES[dtype])
    return inp


def chunked_conv_inputs(B, H, Hg, Wg, d, dtype="bf16", seed=0):
    """Chunked-scan inputs on an Hg x Wg grid plus the two 3x3 depthwise filters of the Conv2d
    preprocessing: wk, wv [H,d,3,3] fp32 ~ N(0, 1/9) (drawn after W0, K's filter first)."""
    inp = linear_inputs(B, H, Hg * Wg, d, dtype=dtype, seed=seed)
    g = _gen(seed + 7919)
    inp["wk"] = _randn((H, d, 3, 3), g, 1.0 / 3.0, torch.float32)
    inp["wv"] = _randn((H, d, 3, 3), g, 1.0 / 3.0, torch.float32)
    return inp


def block_inputs(B, Hg, Wg, C, H, dtype="bf16", seed=0):
    """Inputs of the ViT^3 TTT block: x [B, Hg*Wg, C] ~ N(0,1) and the weights, drawn in the
    order x, Wqkvg, W0, wc, Wo: Wqkvg [C, 4C] (Q, K, V columns ~ N(0, 1/(C d)) so that Q, K, V
    have the spread N(0,1)/sqrt(d) of the layer's other workloads, gate columns ~ N(0, 1/C)),
    W0 [H, d, d] fp32 ~ N(0, 1/d), wc [C, 3, 3] fp32 ~ N(0, 1/9), Wo [2C, C] ~ N(0, 1/(2C));
    x and the two projection matrices are stored in `dtype`."""
    d = C // H
    g = _gen(seed)
    dt = DTYPES[dtype]
    x = _randn((B, Hg * Wg, C), g, 1.0, dt)
    w = torch.randn((C, 4 * C), generator=g, dtype=torch.float32)
    w[:, :3 * C] *= 1.0 / math.sqrt(C * d)
    w[:, 3 * C:] *= 1.0 / math.sqrt(C)
    wqkvg = w.to(dt).contiguous()
    w0 = _randn((H, d, d), g, 1.0 / math.sqrt(d), torch.float32)
    wc = _randn((C, 3, 3), g, 1.0 / 3.0, torch.float32)
    wo = _randn((2 * C, C), g, 1.0 / math.sqrt(2 * C), dt)
    return {"x": x, "wqkvg": wqkvg, "w0": w0, "wc": wc, "wo": wo}


# The workloads of the layer, by name.  Each entry: (kind, kwargs for the generator, eta, extra)
CONFIGS = {
    # TTT-Linear, fp32, one 14x14 grid, one head of d = 64
    "linear_f32_14x14": ("linear", dict(B=1, H=1, N=196, d=64, dtype="f32"), 1.0, {}),
    # TTT-Linear, ViT-S-like layer: 224^2 image, patch 16, C = 384 as 6 heads of 64
    "linear_vits_bf16": ("linear", dict(B=64, H=6, N=196, d=64, dtype="bf16"), 1.0, {}),
    # TTT-Linear at the high-resolution stage-1 grid 56x56, one head of 64 (the throughput shape)
    "linear_56x56_bf16": ("linear", dict(B=32, H=1, N=3136, d=64, dtype="bf16"), 1.0, {}),
    # 3x3 depthwise-conv inner module, stage-1 shape 56x56, C = 64
    "dwconv_56x56_bf16": ("dwconv", dict(B=32, Hg=56, Wg=56, C=64, dtype="bf16"), 1.0, {}),
    # TTT-MLP, d = 64, hidden 256, 64x64 grid, 12 heads
    "mlp_64x64_bf16": ("mlp", dict(B=16, H=12, N=4096, d=64, dtype="bf16"), 1.0, {}),
    # chunked bidirectional TTT-Linear, 1280^2 at patch 16 (80x80), C = 192 as 3 heads of 64
    "chunked_80x80_bf16": ("chunked", dict(B=8, H=3, N=6400, d=64, dtype="bf16"), 1.0,
                           {"chunk": 64}),
}


def make(kind, seed=0, **kw):
    if kind == "linear":
        return linear_inputs(seed=seed, **kw)
    if kind == "dwconv":
        return dwconv_inputs(seed=seed, **kw)
    if kind == "mlp":
        return mlp_inputs(seed=seed, **kw)
    if kind == "chunked":
        return chunked_inputs(seed=seed, **kw)
    raise ValueError(kind)
