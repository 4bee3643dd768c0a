"""GPU parity of the depthwise-conv, TTT-MLP and chunked bidirectional paths (C ABI vs oracle)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_split_b200 import inputs, ttt
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def cuda(inp):
    return {k: v.to(DEV) for k, v in inp.items()}


# ============================================================== depthwise conv ========
def check_dwconv(B, Hg, Wg, C, dtype, eta=1.0, seed=0):
    inp = inputs.dwconv_inputs(B, Hg, Wg, C, dtype=dtype, seed=seed)
    g = cuda(inp)
    out, ws = ttt.dwconv_fullbatch(g["q"], g["k"], g["v"], g["w0"], eta=eta, with_w_star=True)
    assert ttt.device_error() == 0
    ro, rw = oracle.dwconv_fullbatch(inp["q"], inp["k"], inp["v"], inp["w0"], eta=eta)
    dt = inp["q"].dtype
    # heavy-tailed conv output: the bar is taken beyond the output's own bf16 rounding
    assert_close(out, ro, dt, f"dwconv O {B}x{Hg}x{Wg}x{C} {dtype}", rounding_floor=True)
    assert_close(ws, rw, torch.float32 if dt == torch.float32 else dt, "dwconv w*")


def test_dwconv_56x56_bf16_full():
    """Stage-1 shape: B=32, 56x56 grid, C=64, bf16, every output."""
    check_dwconv(32, 56, 56, 64, "bf16")


@pytest.mark.parametrize("Hg,Wg", [(1, 1), (1, 7), (7, 1), (3, 5), (14, 14), (17, 9)])
def test_dwconv_grids(Hg, Wg):
    check_dwconv(2, Hg, Wg, 64, "bf16", seed=Hg * 100 + Wg)


@pytest.mark.parametrize("B,Hg,Wg", [(3, 56, 56), (2, 64, 64), (2, 20, 84), (1, 150, 12), (40, 8, 8), (2, 9, 90)])
def test_dwconv_c64_shapes(B, Hg, Wg):
    """C = 64 bf16 shapes around the fused kernel's limits: an odd batch, the widest fused grid
    (eight strips, one band), more clusters than fit at once (two waves), and grids past the
    fused kernel (wider than 64 tokens, more than 16 rows per CTA: general kernel)."""
    check_dwconv(B, Hg, Wg, 64, "bf16", seed=B * 1000 + Hg + Wg)


@pytest.mark.parametrize("C", [8, 24, 3])
def test_dwconv_channels(C):
    check_dwconv(3, 10, 12, C, "bf16")


@pytest.mark.parametrize("eta", [0.0, 0.37, -0.5])
def test_dwconv_eta(eta):
    check_dwconv(2, 8, 8, 64, "bf16", eta=eta)


def test_dwconv_f32():
    check_dwconv(2, 14, 14, 16, "f32")


# ============================================================== TTT-MLP ===============
def check_mlp(B, H, N, d, hidden, dtype, eta=1.0, seed=0):
    inp = inputs.mlp_inputs(B, H, N, d, hidden=hidden, dtype=dtype, seed=seed)
    g = cuda(inp)
    out, w1s, w2s = ttt.mlp_fullbatch(g["q"], g["k"], g["v"], g["w1"], g["w2"], eta=eta, with_w_star=True)
    assert ttt.device_error() == 0
    dt = inp["q"].dtype
    wdt = torch.float32 if dt == torch.float32 else dt
    # every unit at once (the oracle threads over units); each unit is also checked on its
    # own so that a slip confined to one (b, h) cannot hide under the whole-tensor RMS
    ro, r1, r2 = oracle.mlp_fullbatch(inp["q"], inp["k"], inp["v"], inp["w1"], inp["w2"], eta=eta)
    assert_close(out, ro, dt, f"mlp O B={B} H={H} N={N}")
    assert_close(w1s, r1, wdt, "mlp W1*")
    assert_close(w2s, r2, wdt, "mlp W2*")
    for b in range(B):
        for h in range(H):
            assert_close(out[b:b + 1, h:h + 1], ro[b:b + 1, h:h + 1], dt, f"mlp O unit ({b},{h})")
    return out, w1s, w2s


def test_mlp_64x64_bf16_full():
    """Full shape B=16, 12 heads, N=4096, d=64, hidden 256: all 192 units against the oracle."""
    check_mlp(16, 12, 4096, 64, 256, "bf16")


@pytest.mark.parametrize("N", [1, 100, 300, 1000])
def test_mlp_small_full(N):
    check_mlp(2, 2, N, 64, 256, "bf16", seed=N)


@pytest.mark.parametrize("eta", [0.0, 0.37, -0.5])
def test_mlp_eta(eta):
    check_mlp(1, 2, 256, 64, 256, "bf16", eta=eta)


def test_mlp_f32_and_other_widths():
    check_mlp(2, 2, 64, 16, 64, "f32")
    check_mlp(1, 2, 70, 32, 128, "bf16")


# ============================================================== chunked bidirectional ==
def check_chunked(B, H, N, d, chunk, dtype, eta=1.0, seed=0):
    inp = inputs.chunked_inputs(B, H, N, d, dtype=dtype, seed=seed)
    g = cuda(inp)
    out = ttt.linear_chunked_bidir(g["q"], g["k"], g["v"], g["w0"], chunk, eta=eta)
    assert ttt.device_error() == 0
    ro = oracle.linear_chunked(inp["q"], inp["k"], inp["v"], inp["w0"], chunk, eta=eta, direction=0)
    assert_close(out, ro, inp["q"].dtype, f"chunked B={B} H={H} N={N} b={chunk} {dtype}")
    return out


def test_chunked_80x80_bf16_full():
    """1280^2 at patch 16: B=8, 3 heads of 64, N=6400, chunk 64, every output."""
    check_chunked(8, 3, 6400, 64, 64, "bf16")


@pytest.mark.parametrize("N,chunk", [(64, 64), (128, 64), (192, 64), (640, 64), (256, 16), (128, 32), (48, 1), (320, 320)])
def test_chunked_shapes(N, chunk):
    check_chunked(2, 2, N, 64, chunk, "bf16", seed=N + chunk)


@pytest.mark.parametrize("eta", [0.0, 0.37, -0.5])
def test_chunked_eta(eta):
    check_chunked(1, 2, 512, 64, 64, "bf16", eta=eta)


def test_chunked_f32():
    check_chunked(2, 1, 96, 32, 16, "f32")


def test_chunked_full_chunk_is_twice_fullbatch():
    """chunk = N: each scan is the full-batch step, so the sum is twice the full-batch output."""
    inp = inputs.linear_inputs(2, 2, 512, 64, dtype="bf16", seed=5)
    g = cuda(inp)
    out = ttt.linear_chunked_bidir(g["q"], g["k"], g["v"], g["w0"], 512)
    ref, _ = oracle.linear_fullbatch(inp["q"], inp["k"], inp["v"], inp["w0"])
    assert_close(out, 2 * ref, torch.bfloat16, "chunk = N")


# ============================================================== determinism ===========
def test_dwconv_deterministic_full_shape():
    """Fixed-order reductions: two calls give bit-identical O and w* (B=32, 56x56, C=64)."""
    g = cuda(inputs.dwconv_inputs(32, 56, 56, 64, dtype="bf16", seed=4))
    o1, w1 = ttt.dwconv_fullbatch(g["q"], g["k"], g["v"], g["w0"], with_w_star=True)
    o2, w2 = ttt.dwconv_fullbatch(g["q"], g["k"], g["v"], g["w0"], with_w_star=True)
    assert torch.equal(o1, o2) and torch.equal(w1, w2)


def test_mlp_deterministic_full_shape():
    """Split-order partial sums: two calls give bit-identical O, W1*, W2* (B=16, H=12, N=4096)."""
    g = cuda(inputs.mlp_inputs(16, 12, 4096, 64, dtype="bf16", seed=4))
    r1 = ttt.mlp_fullbatch(g["q"], g["k"], g["v"], g["w1"], g["w2"], with_w_star=True)
    r2 = ttt.mlp_fullbatch(g["q"], g["k"], g["v"], g["w1"], g["w2"], with_w_star=True)
    assert all(torch.equal(a, b) for a, b in zip(r1, r2))


def test_chunked_deterministic_full_shape():
    """Parked partials combined in a fixed order: two calls give bit-identical O (80x80)."""
    g = cuda(inputs.chunked_inputs(8, 3, 6400, 64, dtype="bf16", seed=4))
    o1 = ttt.linear_chunked_bidir(g["q"], g["k"], g["v"], g["w0"], 64)
    o2 = ttt.linear_chunked_bidir(g["q"], g["k"], g["v"], g["w0"], 64)
    assert torch.equal(o1, o2)
