"""C ABI checks that need no GPU: the library loads, exports every function include/ttt.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes

import pytest

from linear_attention_split_b200 import build, ttt

FAKE = ctypes.c_void_p(0x100000)      # 16-byte aligned, never dereferenced: checks fail first
MISALIGNED = ctypes.c_void_p(0x100008)


@pytest.fixture(scope="module")
def L():
    build.build()
    return ttt.lib()


EXPECTED = {
    "ttt_status_string", "ttt_version", "ttt_kernel_launch_count", "ttt_device_error",
    "ttt_debug_set_wait_limit", "ttt_debug_arm_fault",
    "ttt_linear_fullbatch_workspace_bytes", "ttt_linear_fullbatch",
    "ttt_dwconv_fullbatch_workspace_bytes", "ttt_dwconv_fullbatch",
    "ttt_mlp_fullbatch_workspace_bytes", "ttt_mlp_fullbatch",
    "ttt_linear_chunked_bidir_workspace_bytes", "ttt_linear_chunked_bidir",
    "ttt_linear_chunked_bidir_noalloc", "ttt_linear_chunked_bidir_noalloc_max_bytes",
    "ttt_linear_chunked_workspace_bytes", "ttt_linear_chunked",
    "ttt_linear_minibatch_workspace_bytes", "ttt_linear_minibatch",
    "ttt_linear_chunked_conv_workspace_bytes", "ttt_linear_chunked_conv",
    "ttt_linear_fullbatch_bwd_workspace_bytes", "ttt_linear_fullbatch_bwd",
    "ttt_vit3_block_workspace_bytes", "ttt_vit3_block",
}


def test_exports_every_declared_symbol(L):
    names = set(ttt.declared_functions())
    assert EXPECTED <= names, EXPECTED - names
    for n in sorted(names):
        assert hasattr(L, n), n


def test_status_strings(L):
    for s in range(6):
        assert L.ttt_status_string(s)
    assert L.ttt_status_string(99) == b"unknown status"
    assert L.ttt_version() == 100


def test_workspace_queries(L):
    # tensor-core TTT-Linear needs no workspace; the CUDA-core paths do
    assert L.ttt_linear_fullbatch_workspace_bytes(32, 1, 3136, 64, 1) == 0
    assert L.ttt_linear_fullbatch_workspace_bytes(1, 1, 196, 64, 0) >= 3 * 64 * 64 * 4
    assert L.ttt_linear_fullbatch_workspace_bytes(0, 1, 196, 64, 0) == 0
    assert L.ttt_dwconv_fullbatch_workspace_bytes(2, 5, 5, 8, 1) > 0
    assert L.ttt_mlp_fullbatch_workspace_bytes(1, 1, 10, 8, 32, 0) > 0
    assert L.ttt_linear_chunked_bidir_workspace_bytes(1, 1, 64, 64, 16, 1) >= 0


def lin(L, q=FAKE, w0=FAKE, B=1, H=1, N=16, d=64, eta=1.0, dt=1, ws=None, wsb=0):
    return L.ttt_linear_fullbatch(q, FAKE, FAKE, w0, FAKE, None, B, H, N, d, eta, dt, ws, wsb, None)


def test_linear_rejects_bad_arguments(L):
    assert lin(L, q=None) == 1
    assert lin(L, q=MISALIGNED) == 1
    assert lin(L, w0=None) == 1
    assert lin(L, B=0) == 1
    assert lin(L, N=-3) == 1
    assert lin(L, eta=float("nan")) == 1
    assert lin(L, eta=float("inf")) == 1
    assert lin(L, dt=7) == 1
    assert lin(L, d=256) == 2
    # the CUDA-core path needs a workspace
    assert lin(L, dt=0) == 3
    assert lin(L, dt=0, ws=FAKE, wsb=16) == 3


def test_dwconv_rejects_bad_arguments(L):
    f = L.ttt_dwconv_fullbatch
    assert f(None, FAKE, FAKE, FAKE, FAKE, None, 1, 4, 4, 8, 1.0, 1, FAKE, 1 << 20, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 0, 4, 8, 1.0, 1, FAKE, 1 << 20, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, MISALIGNED, 1, 4, 4, 8, 1.0, 1, FAKE, 1 << 20, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 4, 4, 8, float("nan"), 1, FAKE, 1 << 20, None) == 1


def test_mlp_rejects_bad_arguments(L):
    f = L.ttt_mlp_fullbatch
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 1, 64, 64, 256, 1.0, 1, FAKE, 1 << 30, None]
    a = list(args)
    a[3] = None
    assert f(*a) == 1
    a = list(args)
    a[12] = 0
    assert f(*a) == 1
    a = list(args)
    a[11] = 512
    assert f(*a) == 2
    a = list(args)
    a[16] = 8
    assert f(*a) == 3


def test_chunked_rejects_bad_arguments(L):
    f = L.ttt_linear_chunked_bidir
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 100, 64, 64, 1.0, 1, FAKE, 1 << 30, None) == 1  # N % b
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, 1.0, 1, FAKE, 1 << 30, None) == 1
    assert f(FAKE, FAKE, FAKE, None, FAKE, 1, 1, 128, 64, 64, 1.0, 1, FAKE, 1 << 30, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 256, 64, 1.0, 1, FAKE, 1 << 30, None) == 2


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 4, 8)
    with pytest.raises(ValueError):
        ttt.ttt_linear_fullbatch(q, q, q, torch.zeros(1, 8, 8), q)


def test_noalloc_scan_rejects_sizes_beyond_its_scratch(L):
    """8 images x 3 heads x 6400 tokens need 39 MB of scratch, more than the fixed 16 MiB:
    rejected on the host with TTT_ERR_WORKSPACE before anything reaches the device."""
    assert L.ttt_linear_chunked_bidir_noalloc_max_bytes() == 16 << 20
    rc = L.ttt_linear_chunked_bidir_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 3, 6400, 64, 64, 1.0, 1, None)
    assert rc == 3


def test_one_way_scan_rejects_bad_arguments(L):
    f = L.ttt_linear_chunked
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 64, 1.0, 1, 1, FAKE, 1 << 30, None]
    for direction in (2, -2):
        a = list(ok)
        a[11] = direction
        assert f(*a) == 1
    a = list(ok)
    a[7] = 100  # N % chunk != 0
    assert f(*a) == 1
    # a one-way scan on the tensor-core path needs no workspace; both directions do
    assert L.ttt_linear_chunked_workspace_bytes(2, 3, 640, 64, 64, 1, 1) == 0
    assert L.ttt_linear_chunked_workspace_bytes(2, 3, 640, 64, 64, 0, 1) == \
        L.ttt_linear_chunked_bidir_workspace_bytes(2, 3, 640, 64, 64, 1) > 0
    assert L.ttt_linear_chunked_workspace_bytes(2, 3, 640, 32, 16, -1, 0) > 0


def test_minibatch_rejects_bad_arguments(L):
    f = L.ttt_linear_minibatch
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 128, 64, 64, 2, 1.0, 1, FAKE, 1 << 30, None]
    a = list(ok)
    a[11] = 0  # epochs
    assert f(*a) == 1
    a = list(ok)
    a[10] = 48  # 128 % 48
    assert f(*a) == 1
    a = list(ok)
    a[14] = None  # the workspace is always needed
    assert f(*a) == 3
    assert L.ttt_linear_minibatch_workspace_bytes(2, 2, 128, 64, 64, 2, 1) >= 2 * 2 * 64 * 64 * 4


def test_chunked_conv_rejects_bad_arguments(L):
    f = L.ttt_linear_chunked_conv
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 8, 64, 64, 1.0, 0, 1, FAKE, 1 << 30, None]
    a = list(ok)
    a[4] = None  # wk
    assert f(*a) == 1
    a = list(ok)
    a[12] = 48  # 64 tokens % 48
    assert f(*a) == 1
    a = list(ok)
    a[17] = 16
    assert f(*a) == 3
    need = L.ttt_linear_chunked_conv_workspace_bytes(2, 3, 80, 80, 64, 64, 0, 1)
    assert need >= 2 * 2 * 3 * 6400 * 64 * 2


def test_backward_rejects_bad_arguments(L):
    f = L.ttt_linear_fullbatch_bwd
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 1, 128, 64, 1.0, 1, FAKE, 1 << 30, None]
    for idx in (4, 5, 8):  # dout, dq, dw0
        a = list(ok)
        a[idx] = None
        assert f(*a) == 1
    a = list(ok)
    a[6] = MISALIGNED
    assert f(*a) == 1
    a = list(ok)
    a[12] = 256
    assert f(*a) == 2
    a = list(ok)
    a[16] = 64
    assert f(*a) == 3
    assert L.ttt_linear_fullbatch_bwd_workspace_bytes(2, 1, 128, 48, 0) >= 2 * 6 * 48 * 48 * 4


def test_block_rejects_bad_arguments(L):
    f = L.ttt_vit3_block
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 8, 64, 2, 1.0, 1, FAKE, 1 << 30, None]
    a = list(ok)
    a[10] = 3  # 64 % 3
    assert f(*a) == 1
    a = list(ok)
    a[3] = None  # wc
    assert f(*a) == 1
    a = list(ok)
    a[14] = 64
    assert f(*a) == 3
    assert L.ttt_vit3_block_workspace_bytes(2, 8, 8, 64, 2, 1) >= 5 * 2 * 64 * 64 * 2


def test_misaligned_workspace_is_rejected(L):
    """The workspace, like every tensor, must be 16-byte aligned: a misaligned one is refused on
    the host (TTT_ERR_INVALID_ARG) instead of reaching a TMA or bulk copy on the device."""
    big = 1 << 30
    assert lin(L, dt=0, ws=MISALIGNED, wsb=big) == 1
    assert L.ttt_dwconv_fullbatch(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 4, 4, 8, 1.0, 1, MISALIGNED, big,
                                  None) == 1
    assert L.ttt_mlp_fullbatch(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 1, 64, 64, 256, 1.0, 1,
                               MISALIGNED, big, None) == 1
    assert L.ttt_linear_chunked_bidir(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 64, 1.0, 1, MISALIGNED, big,
                                      None) == 1
    assert L.ttt_linear_chunked(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 64, 1.0, -1, 1, MISALIGNED, big,
                                None) == 1
    assert L.ttt_linear_minibatch(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 128, 64, 64, 2, 1.0, 1, MISALIGNED,
                                  big, None) == 1
    assert L.ttt_linear_chunked_conv(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 8, 64, 64, 1.0, 0, 1,
                                     MISALIGNED, big, None) == 1
    assert L.ttt_linear_fullbatch_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 1, 128, 64, 1.0, 1,
                                      MISALIGNED, big, None) == 1
    assert L.ttt_vit3_block(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 8, 64, 2, 1.0, 1, MISALIGNED, big,
                            None) == 1
