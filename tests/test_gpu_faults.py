"""Failure detection without a GPU fault (GPU).

A simulated lost transfer -- the TTT-Linear tensor-core kernel leaves out its last K/V tile
load when a host-armed test hook is set -- makes a bounded wait run out.  The kernel gives up
that wait, ends normally, and the host reads TTT_ERR_TIMEOUT from the device error word; the
CUDA context stays usable and the next call, with the hook cleared, is bit-identical to a call
made before.  The shape is a single CTA per unit (N <= 112 tokens: one tile, no cluster peers),
and the wait limit is lowered to about a millisecond for the test.
"""
import pytest
import torch

import oracle
from linear_attention_split_b200 import inputs, ttt
from tolerance import assert_close

pytestmark = pytest.mark.gpu


def test_lost_tile_load_reports_timeout_and_recovers():
    dev = torch.device("cuda:0")
    inp = inputs.linear_inputs(2, 1, 100, 64, dtype="bf16", seed=31)
    q, k, v, w0 = (inp[x].to(dev) for x in ("q", "k", "v", "w0"))
    good = ttt.linear_fullbatch(q, k, v, w0)
    torch.cuda.synchronize()
    assert ttt.device_error() == 0
    ro, _ = oracle.linear_fullbatch(inp["q"], inp["k"], inp["v"], inp["w0"])
    assert_close(good, ro, torch.bfloat16, "before the simulated fault")

    ttt.debug_set_wait_limit(2_000_000)  # about a millisecond
    ttt.debug_arm_fault(ttt.TTT_FAULT_SKIP_LOAD)
    try:
        ttt.linear_fullbatch(q, k, v, w0)
        torch.cuda.synchronize()
        with pytest.raises(ttt.TTTError) as exc:
            ttt.device_error()
        assert exc.value.status == 5  # TTT_ERR_TIMEOUT
    finally:
        ttt.debug_arm_fault(0)
        ttt.debug_set_wait_limit(0)
    # the error word was read and cleared: the context is usable and results are exact again
    assert ttt.device_error() == 0
    again = ttt.linear_fullbatch(q, k, v, w0)
    torch.cuda.synchronize()
    assert ttt.device_error() == 0
    assert torch.equal(again, good)


def test_wait_limit_hook_restores_default():
    ttt.debug_set_wait_limit(123456)
    ttt.debug_set_wait_limit(0)
    dev = torch.device("cuda:0")
    inp = inputs.linear_inputs(1, 1, 3136, 64, dtype="bf16", seed=2)
    out = ttt.linear_fullbatch(*(inp[x].to(dev) for x in ("q", "k", "v", "w0")))
    torch.cuda.synchronize()
    assert ttt.device_error() == 0
    ro, _ = oracle.linear_fullbatch(inp["q"], inp["k"], inp["v"], inp["w0"])
    assert_close(out, ro, torch.bfloat16, "default wait limit")
