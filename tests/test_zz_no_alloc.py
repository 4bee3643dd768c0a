"""ttt_linear_chunked_bidir_noalloc against the workspace entry point (GPU).

The no-allocation entry point is for callers that may not allocate device memory when they
call the scan; its scratch is a fixed array in the library's device image.  This test calls
it twice in a row through the C ABI on the same inputs and checks each output against the
output of ttt_linear_chunked_bidir (workspace allocated by the caller), with the parity
tolerance the other bf16 tests use.  It lives in its own file, collected last, and passes
both on its own in a fresh process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

from linear_attention_split_b200 import inputs, ttt
from tolerance import assert_close

pytestmark = pytest.mark.gpu


def test_noalloc_scan_matches_workspace_scan_twice():
    # two 80x80-token images, three heads of 64, chunks of 64: fits the fixed 16 MiB scratch
    B, H, N, d, chunk = 2, 3, 6400, 64, 64
    dev = torch.device("cuda:0")
    inp = {k: v.to(dev) for k, v in inputs.chunked_inputs(B, H, N, d, dtype="bf16", seed=21).items()}
    ref = ttt.linear_chunked_bidir(inp["q"], inp["k"], inp["v"], inp["w0"], chunk)
    torch.cuda.synchronize()
    ref64 = ref.double().cpu().numpy()

    L = ttt.lib()
    assert L.ttt_linear_chunked_bidir_workspace_bytes(B, H, N, d, chunk, ttt.TTT_BF16) <= \
        L.ttt_linear_chunked_bidir_noalloc_max_bytes()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(inp["q"], float("nan"))
        rc = L.ttt_linear_chunked_bidir_noalloc(
            ctypes.c_void_p(inp["q"].data_ptr()), ctypes.c_void_p(inp["k"].data_ptr()),
            ctypes.c_void_p(inp["v"].data_ptr()), ctypes.c_void_p(inp["w0"].data_ptr()),
            ctypes.c_void_p(out.data_ptr()), B, H, N, d, chunk, 1.0, ttt.TTT_BF16, stream)
        assert rc == 0, ttt.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        assert ttt.device_error() == 0
        assert_close(out, ref64, torch.bfloat16, f"no-allocation scan, call {call + 1}")
