"""Out-of-bounds writes, checked with guard bands (GPU; a stand-in for a memory checker).

Every output, optional W* output and workspace of each path is carved out of a larger buffer
whose margins (64 KB before and after) hold a sentinel byte.  After each call the margins must
be untouched and the output must still match the oracle.  Shapes are ragged (token counts
that are not multiples of the tiles, odd grids) so that the clipped TMA stores, the tail tiles
and the parked partials of the chunked scan all run at their edges.
"""
import math

import pytest
import torch

import oracle
from linear_attention_split_b200 import inputs, ttt
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
SENTINEL = 0xA5
MARGIN = 65536


class Guarded:
    """A tensor of `shape`/`dtype` inside a byte buffer with sentinel-filled margins."""

    def __init__(self, shape, dtype):
        esize = torch.empty((), dtype=dtype).element_size()
        self.nbytes = math.prod(shape) * esize
        self.raw = torch.full((2 * MARGIN + max(self.nbytes, 1),), SENTINEL, dtype=torch.uint8, device=DEV)
        self.t = self.raw[MARGIN:MARGIN + self.nbytes].view(dtype).view(shape) if self.nbytes else None

    def intact(self):
        lo = self.raw[:MARGIN]
        hi = self.raw[MARGIN + self.nbytes:]
        return bool((lo == SENTINEL).all().item()) and bool((hi == SENTINEL).all().item())


def cuda(inp):
    return {k: v.to(DEV) for k, v in inp.items()}


def check_guards(*gs):
    torch.cuda.synchronize()
    assert ttt.device_error() == 0
    for g in gs:
        assert g.intact(), "a write landed outside its buffer"


@pytest.mark.parametrize("B,H,N,d,dtype", [(2, 3, 197, 64, "bf16"), (2, 3, 257, 32, "bf16"),
                                           (3, 1, 5000, 64, "bf16"), (2, 2, 17, 48, "f32")])
def test_linear_guard_bands(B, H, N, d, dtype):
    inp = inputs.linear_inputs(B, H, N, d, dtype=dtype, seed=N)
    g = cuda(inp)
    out = Guarded(g["q"].shape, g["q"].dtype)
    ws = Guarded((B, H, d, d), torch.float32)
    nb = ttt.ttt_linear_fullbatch_workspace_bytes(B, H, N, d, ttt._DT[g["q"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_linear_fullbatch(g["q"], g["k"], g["v"], g["w0"], out.t, ws.t, 1.0, work.t)
    check_guards(out, ws, work)
    ro, rw = oracle.linear_fullbatch(inp["q"], inp["k"], inp["v"], inp["w0"])
    assert_close(out.t, ro, inp["q"].dtype, "guarded linear O")


@pytest.mark.parametrize("Hg,Wg,C,dtype", [(17, 9, 64, "bf16"), (10, 12, 24, "bf16"), (7, 5, 16, "f32")])
def test_dwconv_guard_bands(Hg, Wg, C, dtype):
    B = 2
    inp = inputs.dwconv_inputs(B, Hg, Wg, C, dtype=dtype, seed=Hg * Wg)
    g = cuda(inp)
    out = Guarded(g["q"].shape, g["q"].dtype)
    ws = Guarded((B, C, 3, 3), torch.float32)
    nb = ttt.ttt_dwconv_fullbatch_workspace_bytes(B, Hg, Wg, C, ttt._DT[g["q"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_dwconv_fullbatch(g["q"], g["k"], g["v"], g["w0"], out.t, ws.t, 1.0, work.t)
    check_guards(out, ws, work)
    ro, _ = oracle.dwconv_fullbatch(inp["q"], inp["k"], inp["v"], inp["w0"])
    assert_close(out.t, ro, inp["q"].dtype, "guarded dwconv O", rounding_floor=True)


@pytest.mark.parametrize("B,H,N,d,hid,dtype", [(2, 2, 300, 64, 256, "bf16"), (2, 2, 64, 16, 64, "f32")])
def test_mlp_guard_bands(B, H, N, d, hid, dtype):
    inp = inputs.mlp_inputs(B, H, N, d, hidden=hid, dtype=dtype, seed=N)
    g = cuda(inp)
    out = Guarded(g["q"].shape, g["q"].dtype)
    w1s = Guarded((B, H, d, hid), torch.float32)
    w2s = Guarded((B, H, hid, d), torch.float32)
    nb = ttt.ttt_mlp_fullbatch_workspace_bytes(B, H, N, d, hid, ttt._DT[g["q"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_mlp_fullbatch(g["q"], g["k"], g["v"], g["w1"], g["w2"], out.t, w1s.t, w2s.t, 1.0, work.t)
    check_guards(out, w1s, w2s, work)
    ro, _, _ = oracle.mlp_fullbatch(inp["q"], inp["k"], inp["v"], inp["w1"], inp["w2"])
    assert_close(out.t, ro, inp["q"].dtype, "guarded mlp O")


@pytest.mark.parametrize("B,H,N,d,chunk,dtype", [(2, 2, 192, 64, 64, "bf16"), (1, 3, 640, 64, 64, "bf16"),
                                                 (2, 1, 96, 32, 16, "f32")])
def test_chunked_guard_bands(B, H, N, d, chunk, dtype):
    inp = inputs.chunked_inputs(B, H, N, d, dtype=dtype, seed=N + chunk)
    g = cuda(inp)
    out = Guarded(g["q"].shape, g["q"].dtype)
    nb = ttt.ttt_linear_chunked_bidir_workspace_bytes(B, H, N, d, chunk, ttt._DT[g["q"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_linear_chunked_bidir(g["q"], g["k"], g["v"], g["w0"], out.t, chunk, 1.0, work.t)
    check_guards(out, work)
    ro = oracle.linear_chunked(inp["q"], inp["k"], inp["v"], inp["w0"], chunk)
    assert_close(out.t, ro, inp["q"].dtype, "guarded chunked O")


@pytest.mark.parametrize("B,H,N,d,chunk,dtype,direction", [(2, 2, 192, 64, 64, "bf16", 1),
                                                           (1, 3, 640, 64, 64, "bf16", -1),
                                                           (2, 1, 96, 32, 16, "f32", -1)])
def test_one_way_scan_guard_bands(B, H, N, d, chunk, dtype, direction):
    inp = inputs.chunked_inputs(B, H, N, d, dtype=dtype, seed=N + chunk)
    g = cuda(inp)
    out = Guarded(g["q"].shape, g["q"].dtype)
    nb = ttt.ttt_linear_chunked_workspace_bytes(B, H, N, d, chunk, direction, ttt._DT[g["q"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_linear_chunked(g["q"], g["k"], g["v"], g["w0"], out.t, chunk, 1.0, direction, work.t)
    check_guards(out, work)
    ro = oracle.linear_chunked(inp["q"], inp["k"], inp["v"], inp["w0"], chunk, direction=direction)
    assert_close(out.t, ro, inp["q"].dtype, "guarded one-way O", rounding_floor="auto")


@pytest.mark.parametrize("B,H,N,d,chunk,epochs,dtype", [(2, 1, 3136, 64, 64, 2, "bf16"),
                                                        (2, 3, 1000, 64, 40, 2, "bf16"),
                                                        (1, 2, 96, 32, 16, 2, "f32")])
def test_minibatch_guard_bands(B, H, N, d, chunk, epochs, dtype):
    inp = inputs.linear_inputs(B, H, N, d, dtype=dtype, seed=chunk + epochs)
    g = cuda(inp)
    out = Guarded(g["q"].shape, g["q"].dtype)
    wf = Guarded((B, H, d, d), torch.float32)
    nb = ttt.ttt_linear_minibatch_workspace_bytes(B, H, N, d, chunk, epochs, ttt._DT[g["q"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_linear_minibatch(g["q"], g["k"], g["v"], g["w0"], out.t, chunk, epochs, wf.t, 1.0, work.t)
    check_guards(out, wf, work)
    ro, _ = oracle.linear_minibatch(inp["q"], inp["k"], inp["v"], inp["w0"], chunk, epochs)
    assert_close(out.t, ro, inp["q"].dtype, "guarded mini-batch O")


@pytest.mark.parametrize("Hg,Wg,d,chunk,dtype", [(8, 16, 64, 64, "bf16"), (7, 9, 32, 9, "f32")])
def test_chunked_conv_guard_bands(Hg, Wg, d, chunk, dtype):
    B, H = 2, 2
    inp = inputs.chunked_conv_inputs(B, H, Hg, Wg, d, dtype=dtype, seed=Hg * Wg)
    g = cuda(inp)
    out = Guarded(g["q"].shape, g["q"].dtype)
    nb = ttt.ttt_linear_chunked_conv_workspace_bytes(B, H, Hg, Wg, d, chunk, 0, ttt._DT[g["q"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_linear_chunked_conv(g["q"], g["k"], g["v"], g["w0"], g["wk"], g["wv"], out.t, Hg, Wg, chunk, 0.7, 0,
                                work.t)
    check_guards(out, work)
    ro = oracle.linear_chunked_prep(inp["q"], inp["k"], inp["v"], inp["w0"], inp["wk"], inp["wv"], Hg, Wg, chunk,
                                    eta=0.7)
    assert_close(out.t, ro, inp["q"].dtype, "guarded conv scan O", rounding_floor="auto")


@pytest.mark.parametrize("B,H,N,d,dtype", [(3, 2, 197, 64, "bf16"), (2, 2, 1000, 64, "bf16"), (2, 1, 50, 48, "f32")])
def test_backward_guard_bands(B, H, N, d, dtype):
    inp = inputs.linear_bwd_inputs(B, H, N, d, dtype=dtype, seed=N)
    g = cuda(inp)
    dq, dk, dv = (Guarded(g["q"].shape, g["q"].dtype) for _ in range(3))
    dw0 = Guarded((H, d, d), torch.float32)
    nb = ttt.ttt_linear_fullbatch_bwd_workspace_bytes(B, H, N, d, ttt._DT[g["q"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_linear_fullbatch_bwd(g["q"], g["k"], g["v"], g["w0"], g["dout"], dq.t, dk.t, dv.t, dw0.t, 1.0, work.t)
    check_guards(dq, dk, dv, dw0, work)
    rq, rk, rv, _ = oracle.linear_fullbatch_bwd(inp["q"], inp["k"], inp["v"], inp["w0"], inp["dout"])
    for got, ref, name in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
        assert_close(got.t, ref, inp["q"].dtype, "guarded backward " + name, rounding_floor="auto")


@pytest.mark.parametrize("B,Hg,Wg,C,H,dtype", [(3, 7, 9, 64, 2, "bf16"), (2, 17, 17, 64, 1, "bf16"),
                                               (2, 5, 6, 32, 2, "f32")])
def test_block_guard_bands(B, Hg, Wg, C, H, dtype):
    inp = inputs.block_inputs(B, Hg, Wg, C, H, dtype=dtype, seed=Hg * Wg)
    g = cuda(inp)
    y = Guarded(g["x"].shape, g["x"].dtype)
    nb = ttt.ttt_vit3_block_workspace_bytes(B, Hg, Wg, C, H, ttt._DT[g["x"].dtype])
    work = Guarded((nb,), torch.uint8)
    ttt.ttt_vit3_block(g["x"], g["wqkvg"], g["w0"], g["wc"], g["wo"], y.t, Hg, Wg, H, 1.0, work.t)
    check_guards(y, work)
    ref = oracle.vit3_block(inp["x"], inp["wqkvg"], inp["w0"], inp["wc"], inp["wo"], Hg, Wg, H)
    assert_close(y.t, ref, inp["x"].dtype, "guarded block y", rounding_floor="auto")
