"""GPU parity of TTT-Linear full batch (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_split_b200 import inputs, ttt
from tolerance import assert_close

pytestmark = pytest.mark.gpu


def run(inp, eta):
    dev = torch.device("cuda:0")
    q, k, v, w0 = (inp[x].to(dev) for x in ("q", "k", "v", "w0"))
    out, ws = ttt.linear_fullbatch(q, k, v, w0, eta=eta, with_w_star=True)
    torch.cuda.synchronize()
    assert ttt.device_error() == 0
    return out, ws


def check(B, H, N, d, dtype, eta=1.0, seed=0, **kw):
    inp = inputs.linear_inputs(B, H, N, d, dtype=dtype, seed=seed, **kw)
    out, ws = run(inp, eta)
    ro, rw = oracle.linear_fullbatch(inp["q"], inp["k"], inp["v"], inp["w0"], eta=eta)
    dt = inp["q"].dtype
    eo = assert_close(out, ro, dt, f"O B={B} H={H} N={N} d={d} {dtype} eta={eta}")
    ew = assert_close(ws, rw, torch.float32 if dt == torch.float32 else dt, "W*")
    return eo, ew


def test_linear_f32_14x14():
    """TTT-Linear, fp32, B=1, one head, 14x14 grid (N=196), d=64."""
    check(1, 1, 196, 64, "f32")


def test_linear_vits_bf16():
    """ViT-S-like layer: B=64, 6 heads of d=64, N=196, bf16."""
    check(64, 6, 196, 64, "bf16")


def test_linear_56x56_bf16_full():
    """The throughput shape: B=32, one head of 64, 56x56 grid (N=3136), bf16, every output."""
    check(32, 1, 3136, 64, "bf16")


def test_linear_56x56_two_heads_d32():
    """Stage-1 head split: B=32, 2 heads of d=32, N=3136."""
    check(32, 2, 3136, 32, "bf16")


@pytest.mark.parametrize("N", [1, 17, 195, 197, 257, 1000])
@pytest.mark.parametrize("d", [32, 64])
def test_linear_ragged_tails(N, d):
    check(2, 3, N, d, "bf16", seed=N)


@pytest.mark.parametrize("eta", [0.0, 0.37, -0.5])
def test_linear_eta(eta):
    check(3, 2, 300, 64, "bf16", eta=eta)


def test_linear_single_unit_low_occupancy():
    check(1, 1, 3136, 64, "bf16")


@pytest.mark.parametrize("N", [5000, 16384])
def test_linear_long_sequence_streams_q(N):
    """N large enough that Q no longer fits the resident region and streams through the ring."""
    check(2, 1, N, 64, "bf16")


@pytest.mark.parametrize("N,d", [(17, 48), (196, 64), (50, 16)])
def test_linear_f32_shapes(N, d):
    check(2, 2, N, d, "f32")


def test_linear_bf16_generic_width():
    """bf16 with a width the tensor-core kernel does not take (d=48) runs the CUDA-core path."""
    check(2, 2, 200, 48, "bf16")


def test_linear_l2_proof_batch_sampled():
    """B=256 (inputs > L2), compared on a sample of units the oracle computes one by one."""
    B, H, N, d = 256, 1, 3136, 64
    inp = inputs.linear_inputs(B, H, N, d, dtype="bf16", seed=7)
    out, ws = run(inp, 1.0)
    for b in (0, 1, 127, 255):
        ro, rw = oracle.linear_fullbatch(inp["q"][b:b + 1], inp["k"][b:b + 1], inp["v"][b:b + 1],
                                         inp["w0"])
        assert_close(out[b:b + 1], ro, torch.bfloat16, f"unit {b}")
        assert_close(ws[b:b + 1], rw, torch.bfloat16, f"W* unit {b}")


def test_linear_deterministic():
    inp = inputs.linear_inputs(32, 1, 3136, 64, dtype="bf16", seed=3)
    o1, w1 = run(inp, 1.0)
    o2, w2 = run(inp, 1.0)
    assert torch.equal(o1, o2) and torch.equal(w1, w2)


def test_linear_zero_init_is_linear_attention():
    """W0 = 0 reduces the layer to (eta/N) Q (K^T V) -- a property at any size."""
    inp = inputs.linear_inputs(4, 2, 3136, 64, dtype="bf16", seed=11)
    inp["w0"] = torch.zeros_like(inp["w0"])
    out, _ = run(inp, 1.0)
    q, k, v = (inp[x].double() for x in ("q", "k", "v"))
    ref = (q @ (k.transpose(-1, -2) @ v)) / 3136
    assert_close(out, ref.numpy(), torch.bfloat16, "linear attention")


# ---- few long units (the tensor-core kernel's cluster split at other token counts) -------
@pytest.mark.parametrize("N", [3000, 1000, 6272, 3137])
def test_linear_long_units_ragged(N):
    """B=32 units of one head at ragged token counts: other tile heights and a partial last tile."""
    check(32, 1, N, 64, "bf16", seed=N)


@pytest.mark.parametrize("B,H", [(16, 2), (20, 2), (36, 1)])
def test_linear_long_units_heads(B, H):
    """Several heads per image (W0 differs between neighbouring units) and unit counts that
    change the cluster size."""
    check(B, H, 3136, 64, "bf16", seed=B * H)


@pytest.mark.parametrize("eta", [0.0, -0.5])
def test_linear_long_units_eta(eta):
    check(32, 1, 3136, 64, "bf16", eta=eta, seed=3)
