"""GPU parity of the inner-training variants against the oracle: one-way chunked scans, the
mini-batch / multi-epoch step, and the chunked scan on a Conv2d-preprocessed dataset."""
import pytest
import torch

import oracle
from linear_attention_split_b200 import inputs, ttt
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def cuda(inp):
    return {k: v.to(DEV) for k, v in inp.items()}


# ============================================================== one-way scans ==========
@pytest.mark.parametrize("direction", [1, -1])
def test_chunked_one_way_80x80(direction):
    """1280^2 at patch 16: B=8, 3 heads of 64, N=6400, chunk 64, one direction, every output."""
    inp = inputs.chunked_inputs(8, 3, 6400, 64, dtype="bf16", seed=3)
    g = cuda(inp)
    out = ttt.linear_chunked(g["q"], g["k"], g["v"], g["w0"], 64, direction=direction)
    assert ttt.device_error() == 0
    ro = oracle.linear_chunked(inp["q"], inp["k"], inp["v"], inp["w0"], 64, direction=direction)
    # heavy-tailed one-way output: the bar is taken beyond its own bf16 rounding when that
    # rounding alone exceeds it (checked on the exact result)
    assert_close(out, ro, torch.bfloat16, f"one-way scan direction {direction}", rounding_floor="auto")


@pytest.mark.parametrize("N,chunk,dtype", [(64, 64, "bf16"), (128, 64, "bf16"), (192, 64, "bf16"),
                                           (256, 16, "bf16"), (96, 16, "f32"), (48, 1, "f32")])
@pytest.mark.parametrize("direction", [1, -1, 0])
def test_chunked_one_way_shapes(N, chunk, dtype, direction):
    d = 32 if dtype == "f32" else 64
    inp = inputs.chunked_inputs(2, 2, N, d, dtype=dtype, seed=N + chunk)
    g = cuda(inp)
    out = ttt.linear_chunked(g["q"], g["k"], g["v"], g["w0"], chunk, eta=0.8, direction=direction)
    assert ttt.device_error() == 0
    ro = oracle.linear_chunked(inp["q"], inp["k"], inp["v"], inp["w0"], chunk, eta=0.8, direction=direction)
    assert_close(out, ro, inp["q"].dtype, f"scan N={N} b={chunk} dir={direction} {dtype}", rounding_floor="auto")


def test_one_way_scans_sum_to_bidirectional_on_gpu():
    inp = inputs.chunked_inputs(2, 3, 640, 64, dtype="bf16", seed=9)
    g = cuda(inp)
    f = ttt.linear_chunked(g["q"], g["k"], g["v"], g["w0"], 64, direction=1).double()
    r = ttt.linear_chunked(g["q"], g["k"], g["v"], g["w0"], 64, direction=-1).double()
    both = oracle.linear_chunked(inp["q"], inp["k"], inp["v"], inp["w0"], 64, direction=0)
    assert_close((f + r).cpu().numpy(), both, torch.bfloat16, "forward + reverse")


# ============================================================== mini-batch / epochs =====
@pytest.mark.parametrize("B,H,N,d,chunk,epochs,dtype", [
    (4, 2, 3136, 64, 3136, 1, "bf16"),   # one epoch, full batch: the full-batch kernel
    (2, 2, 3136, 64, 64, 1, "bf16"),     # mini-batches of 64, one epoch
    (2, 2, 1024, 64, 64, 2, "bf16"),     # two epochs
    (8, 1, 3136, 64, 64, 2, "bf16"),     # the benchmarked 56x56 shape: 49 chunks x 2 epochs
    (2, 3, 1000, 64, 40, 2, "bf16"),     # chunks of 40 (CUDA-core training), tensor-core output pass, ragged tile
    (2, 1, 196, 64, 196, 3, "f32"),      # full batch, three epochs
    (1, 2, 96, 32, 16, 2, "f32"),
])
def test_minibatch(B, H, N, d, chunk, epochs, dtype):
    inp = inputs.linear_inputs(B, H, N, d, dtype=dtype, seed=chunk + epochs)
    g = cuda(inp)
    out, wf = ttt.linear_minibatch(g["q"], g["k"], g["v"], g["w0"], chunk, epochs, with_w_final=True)
    assert ttt.device_error() == 0
    ro, rw = oracle.linear_minibatch(inp["q"], inp["k"], inp["v"], inp["w0"], chunk, epochs)
    dt = inp["q"].dtype
    assert_close(out, ro, dt, f"mini-batch O N={N} b={chunk} E={epochs} {dtype}")
    assert_close(wf, rw, torch.float32 if dt == torch.float32 else dt, "W_final")


# ============================================================== Conv2d preprocessing ====
@pytest.mark.parametrize("direction", [0, 1])
def test_chunked_conv_80x80(direction):
    """Conv2d-preprocessed scan at 80x80 (B=2 images, 3 heads of 64, chunk 64)."""
    inp = inputs.chunked_conv_inputs(2, 3, 80, 80, 64, dtype="bf16", seed=5)
    g = cuda(inp)
    out = ttt.linear_chunked_conv(g["q"], g["k"], g["v"], g["w0"], g["wk"], g["wv"], 80, 80, 64,
                                  direction=direction)
    assert ttt.device_error() == 0
    ro = oracle.linear_chunked_prep(inp["q"], inp["k"], inp["v"], inp["w0"], inp["wk"], inp["wv"], 80, 80, 64,
                                    direction=direction)
    assert_close(out, ro, torch.bfloat16, f"conv-preprocessed scan dir={direction}", rounding_floor="auto")


@pytest.mark.parametrize("Hg,Wg,d,chunk,dtype", [(8, 16, 64, 64, "bf16"), (7, 9, 32, 9, "f32"), (1, 64, 64, 64, "bf16")])
def test_chunked_conv_shapes(Hg, Wg, d, chunk, dtype):
    inp = inputs.chunked_conv_inputs(2, 2, Hg, Wg, d, dtype=dtype, seed=Hg * Wg)
    g = cuda(inp)
    out = ttt.linear_chunked_conv(g["q"], g["k"], g["v"], g["w0"], g["wk"], g["wv"], Hg, Wg, chunk, eta=0.7)
    assert ttt.device_error() == 0
    ro = oracle.linear_chunked_prep(inp["q"], inp["k"], inp["v"], inp["w0"], inp["wk"], inp["wv"], Hg, Wg, chunk,
                                    eta=0.7)
    assert_close(out, ro, inp["q"].dtype, f"conv scan {Hg}x{Wg} d={d} b={chunk} {dtype}", rounding_floor="auto")


# ============================================================== determinism ===========
def test_minibatch_deterministic_full_shape():
    """Training-mode scan and the output pass: two calls give bit-identical O and W_final at
    the benchmarked shape (B=32 images of 56x56, b = 64, two epochs)."""
    g = cuda(inputs.linear_inputs(32, 1, 3136, 64, dtype="bf16", seed=6))
    o1, w1 = ttt.linear_minibatch(g["q"], g["k"], g["v"], g["w0"], 64, 2, with_w_final=True)
    o2, w2 = ttt.linear_minibatch(g["q"], g["k"], g["v"], g["w0"], 64, 2, with_w_final=True)
    assert ttt.device_error() == 0
    assert torch.equal(o1, o2) and torch.equal(w1, w2)


@pytest.mark.parametrize("direction", [1, -1])
def test_one_way_deterministic_full_shape(direction):
    g = cuda(inputs.chunked_inputs(8, 3, 6400, 64, dtype="bf16", seed=6))
    o1 = ttt.linear_chunked(g["q"], g["k"], g["v"], g["w0"], 64, direction=direction)
    o2 = ttt.linear_chunked(g["q"], g["k"], g["v"], g["w0"], 64, direction=direction)
    assert ttt.device_error() == 0
    assert torch.equal(o1, o2)


def test_chunked_conv_deterministic_full_shape():
    """Preprocessing pass + bidirectional scan at the benchmarked shape (B=8, 3 heads, 80x80)."""
    g = cuda(inputs.chunked_conv_inputs(8, 3, 80, 80, 64, dtype="bf16", seed=6))
    args = (g["q"], g["k"], g["v"], g["w0"], g["wk"], g["wv"], 80, 80, 64)
    o1 = ttt.linear_chunked_conv(*args)
    o2 = ttt.linear_chunked_conv(*args)
    assert ttt.device_error() == 0
    assert torch.equal(o1, o2)
