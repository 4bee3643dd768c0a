"""GPU parity of the TTT-Linear backward (gradients through the inner step) against the
oracle's hand-derived chain rule, itself pinned by finite differences and autograd."""
import pytest
import torch

import oracle
from linear_attention_split_b200 import inputs, ttt
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def check_bwd(B, H, N, d, dtype, eta=1.0, seed=0):
    inp = inputs.linear_bwd_inputs(B, H, N, d, dtype=dtype, seed=seed)
    g = {k: v.to(DEV) for k, v in inp.items()}
    dq, dk, dv, dw0 = ttt.linear_fullbatch_bwd(g["q"], g["k"], g["v"], g["w0"], g["dout"], eta=eta)
    assert ttt.device_error() == 0
    rq, rk, rv, rw = oracle.linear_fullbatch_bwd(inp["q"], inp["k"], inp["v"], inp["w0"], inp["dout"], eta=eta)
    dt = inp["q"].dtype
    what = f"B={B} H={H} N={N} d={d} {dtype} eta={eta}"
    assert_close(dq, rq, dt, "dQ " + what, rounding_floor="auto")
    assert_close(dv, rv, dt, "dV " + what, rounding_floor="auto")
    assert_close(dk, rk, dt, "dK " + what, rounding_floor="auto")
    assert_close(dw0, rw, torch.float32 if dt == torch.float32 else dt, "dW0 " + what)
    return dq, dk, dv, dw0


def test_bwd_56x56_bf16_full():
    """The forward's throughput shape: B=32, one head of 64, 56x56 grid (N=3136), every output."""
    check_bwd(32, 1, 3136, 64, "bf16")


def test_bwd_vits_bf16():
    """ViT-S-like layer: B=64, 6 heads of 64, N=196."""
    check_bwd(64, 6, 196, 64, "bf16")


@pytest.mark.parametrize("N", [1, 17, 197, 1000, 5000])
def test_bwd_ragged(N):
    check_bwd(3, 2, N, 64, "bf16", seed=N)


@pytest.mark.parametrize("eta", [0.0, 0.37, -0.5])
def test_bwd_eta(eta):
    check_bwd(2, 2, 300, 64, "bf16", eta=eta)


@pytest.mark.parametrize("N,d,dtype", [(196, 64, "f32"), (50, 48, "f32"), (257, 32, "bf16")])
def test_bwd_cuda_core_paths(N, d, dtype):
    check_bwd(2, 2, N, d, dtype)


def test_bwd_deterministic():
    inp = inputs.linear_bwd_inputs(32, 1, 3136, 64, dtype="bf16", seed=8)
    g = {k: v.to(DEV) for k, v in inp.items()}
    r1 = ttt.linear_fullbatch_bwd(g["q"], g["k"], g["v"], g["w0"], g["dout"])
    r2 = ttt.linear_fullbatch_bwd(g["q"], g["k"], g["v"], g["w0"], g["dout"])
    assert all(torch.equal(a, b) for a, b in zip(r1, r2))
