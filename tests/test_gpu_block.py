"""GPU parity of the ViT^3 TTT block around the core (projections, TTT-Linear per head, GLU
gate, 3x3 depthwise-conv branch, concat, output projection) against the oracle."""
import pytest
import torch

import oracle
from linear_attention_split_b200 import inputs, ttt
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def check_block(B, Hg, Wg, C, H, dtype, eta=1.0, seed=0):
    inp = inputs.block_inputs(B, Hg, Wg, C, H, dtype=dtype, seed=seed)
    g = {k: v.to(DEV) for k, v in inp.items()}
    y = ttt.vit3_block(g["x"], g["wqkvg"], g["w0"], g["wc"], g["wo"], Hg, Wg, H, eta=eta)
    assert ttt.device_error() == 0
    ref = oracle.vit3_block(inp["x"], inp["wqkvg"], inp["w0"], inp["wc"], inp["wo"], Hg, Wg, H, eta=eta)
    assert_close(y, ref, inp["x"].dtype, f"block B={B} {Hg}x{Wg} C={C} H={H} {dtype} eta={eta}",
                 rounding_floor="auto")
    return y


def test_block_stage1_56x56():
    """High-resolution stage-1 block: B=32, 56x56 grid, C=64 as 2 heads of 32, every output."""
    check_block(32, 56, 56, 64, 2, "bf16")


def test_block_one_head_of_64():
    check_block(4, 14, 14, 64, 1, "bf16", seed=1)


@pytest.mark.parametrize("Hg,Wg", [(7, 9), (1, 1), (3, 50), (17, 17)])
def test_block_ragged_grids(Hg, Wg):
    check_block(3, Hg, Wg, 64, 2, "bf16", seed=Hg * Wg)


@pytest.mark.parametrize("eta", [0.0, 0.37, -0.5])
def test_block_eta(eta):
    check_block(2, 8, 8, 64, 2, "bf16", eta=eta)


@pytest.mark.parametrize("C,H,dtype", [(16, 2, "f32"), (48, 3, "bf16"), (64, 4, "bf16")])
def test_block_cuda_core_paths(C, H, dtype):
    check_block(2, 6, 5, C, H, dtype)


def test_block_deterministic():
    inp = inputs.block_inputs(8, 56, 56, 64, 2, dtype="bf16", seed=6)
    g = {k: v.to(DEV) for k, v in inp.items()}
    y1 = ttt.vit3_block(g["x"], g["wqkvg"], g["w0"], g["wc"], g["wo"], 56, 56, 2)
    y2 = ttt.vit3_block(g["x"], g["wqkvg"], g["w0"], g["wc"], g["wo"], 56, 56, 2)
    assert torch.equal(y1, y2)
