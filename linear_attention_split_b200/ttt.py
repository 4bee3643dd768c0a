"""Thin Python binding of libttt_b200.so (the C ABI declared in include/ttt.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch provides device memory and streams.  The functions carry the C names and take
torch CUDA tensors; ``*_workspace_bytes`` mirror the C queries.  If the library has not
been built this module raises on first use -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libttt_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "ttt.h")

TTT_F32, TTT_BF16 = 0, 1
_DT = {torch.float32: TTT_F32, torch.bfloat16: TTT_BF16}

STATUS = {0: "TTT_OK", 1: "TTT_ERR_INVALID_ARG", 2: "TTT_ERR_UNSUPPORTED", 3: "TTT_ERR_WORKSPACE",
          4: "TTT_ERR_CUDA", 5: "TTT_ERR_TIMEOUT"}


class TTTError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} returned {STATUS.get(status, status)}: "
                         f"{lib().ttt_status_string(status).decode()}")


_lib = None


def lib():
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m linear_attention_split_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        p, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.ttt_status_string.restype = ctypes.c_char_p
        L.ttt_status_string.argtypes = [i]
        L.ttt_version.restype = i
        L.ttt_version.argtypes = []
        L.ttt_kernel_launch_count.restype = ctypes.c_ulonglong
        L.ttt_kernel_launch_count.argtypes = []
        L.ttt_device_error.restype = i
        L.ttt_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        L.ttt_debug_set_wait_limit.restype = i
        L.ttt_debug_set_wait_limit.argtypes = [ctypes.c_longlong]
        L.ttt_debug_arm_fault.restype = i
        L.ttt_debug_arm_fault.argtypes = [ctypes.c_uint]
        L.ttt_linear_fullbatch_workspace_bytes.restype = sz
        L.ttt_linear_fullbatch_workspace_bytes.argtypes = [i, i, i, i, i]
        L.ttt_linear_fullbatch.restype = i
        L.ttt_linear_fullbatch.argtypes = [p, p, p, p, p, p, i, i, i, i, f, i, p, sz, p]
        L.ttt_vit3_block_workspace_bytes.restype = sz
        L.ttt_vit3_block_workspace_bytes.argtypes = [i, i, i, i, i, i]
        L.ttt_vit3_block.restype = i
        L.ttt_vit3_block.argtypes = [p, p, p, p, p, p, i, i, i, i, i, f, i, p, sz, p]
        L.ttt_linear_fullbatch_bwd_workspace_bytes.restype = sz
        L.ttt_linear_fullbatch_bwd_workspace_bytes.argtypes = [i, i, i, i, i]
        L.ttt_linear_fullbatch_bwd.restype = i
        L.ttt_linear_fullbatch_bwd.argtypes = [p, p, p, p, p, p, p, p, p, i, i, i, i, f, i, p, sz, p]
        L.ttt_dwconv_fullbatch_workspace_bytes.restype = sz
        L.ttt_dwconv_fullbatch_workspace_bytes.argtypes = [i, i, i, i, i]
        L.ttt_dwconv_fullbatch.restype = i
        L.ttt_dwconv_fullbatch.argtypes = [p, p, p, p, p, p, i, i, i, i, f, i, p, sz, p]
        L.ttt_mlp_fullbatch_workspace_bytes.restype = sz
        L.ttt_mlp_fullbatch_workspace_bytes.argtypes = [i, i, i, i, i, i]
        L.ttt_mlp_fullbatch.restype = i
        L.ttt_mlp_fullbatch.argtypes = [p, p, p, p, p, p, p, p, i, i, i, i, i, f, i, p, sz, p]
        L.ttt_linear_chunked_bidir_workspace_bytes.restype = sz
        L.ttt_linear_chunked_bidir_workspace_bytes.argtypes = [i, i, i, i, i, i]
        L.ttt_linear_chunked_bidir.restype = i
        L.ttt_linear_chunked_bidir.argtypes = [p, p, p, p, p, i, i, i, i, i, f, i, p, sz, p]
        L.ttt_linear_chunked_workspace_bytes.restype = sz
        L.ttt_linear_chunked_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        L.ttt_linear_chunked.restype = i
        L.ttt_linear_chunked.argtypes = [p, p, p, p, p, i, i, i, i, i, f, i, i, p, sz, p]
        L.ttt_linear_minibatch_workspace_bytes.restype = sz
        L.ttt_linear_minibatch_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        L.ttt_linear_minibatch.restype = i
        L.ttt_linear_minibatch.argtypes = [p, p, p, p, p, p, i, i, i, i, i, i, f, i, p, sz, p]
        L.ttt_linear_chunked_conv_workspace_bytes.restype = sz
        L.ttt_linear_chunked_conv_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
        L.ttt_linear_chunked_conv.restype = i
        L.ttt_linear_chunked_conv.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, i, f, i, i, p, sz, p]
        L.ttt_linear_chunked_bidir_noalloc.restype = i
        L.ttt_linear_chunked_bidir_noalloc.argtypes = [p, p, p, p, p, i, i, i, i, i, f, i, p]
        L.ttt_linear_chunked_bidir_noalloc_max_bytes.restype = sz
        L.ttt_linear_chunked_bidir_noalloc_max_bytes.argtypes = []
        _lib = L
    return _lib


def declared_functions() -> list[str]:
    """Names of the functions include/ttt.h declares."""
    with open(HEADER_PATH) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"\b(ttt_[a-z0-9_]+)\s*\(", text)))


# ----------------------------------------------------------------------- helpers -------
def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dtype(*ts):
    dt = ts[0].dtype
    for t in ts:
        if t.dtype != dt:
            raise TypeError("q, k, v and out must share one dtype")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if dt not in _DT:
        raise TypeError(f"unsupported dtype {dt}")
    return _DT[dt]


def _weights(*ws):
    for w in ws:
        if w is None:
            continue
        if w.dtype != torch.float32 or not w.is_cuda or not w.is_contiguous():
            raise ValueError("inner weights must be contiguous fp32 CUDA tensors")


def _workspace(nbytes, workspace, device):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError("workspace too small")
    return workspace, workspace.numel() * workspace.element_size()


def _check(fn, rc):
    if rc != 0:
        raise TTTError(fn, rc)


# ----------------------------------------------------------------------- entry points --
def ttt_linear_fullbatch_workspace_bytes(B, H, N, d, dtype):
    return lib().ttt_linear_fullbatch_workspace_bytes(B, H, N, d, dtype)


def ttt_linear_fullbatch(q, k, v, w0, out, w_star=None, eta=1.0, workspace=None, stream=None):
    """q, k, v, out [B,H,N,d] (fp32 or bf16); w0 [H,d,d] fp32; w_star [B,H,d,d] fp32 or None."""
    dt = _dtype(q, k, v, out)
    _weights(w0, w_star)
    B, H, N, d = q.shape
    ws, nbytes = _workspace(ttt_linear_fullbatch_workspace_bytes(B, H, N, d, dt), workspace, q.device)
    rc = lib().ttt_linear_fullbatch(_ptr(q), _ptr(k), _ptr(v), _ptr(w0), _ptr(out), _ptr(w_star), B, H, N,
                                    d, float(eta), dt, _ptr(ws), nbytes, _stream(stream))
    _check("ttt_linear_fullbatch", rc)
    return out


def ttt_vit3_block_workspace_bytes(B, Hg, Wg, C, H, dtype):
    return lib().ttt_vit3_block_workspace_bytes(B, Hg, Wg, C, H, dtype)


def ttt_vit3_block(x, wqkvg, w0, wc, wo, y, Hg, Wg, H, eta=1.0, workspace=None, stream=None):
    """The ViT^3 TTT block: x, y [B, Hg*Wg, C]; wqkvg [C, 4C] and wo [2C, C] in x's dtype;
    w0 [H, C/H, C/H] and wc [C, 3, 3] fp32."""
    dt = _dtype(x, wqkvg, wo, y)
    _weights(w0, wc)
    B, N, C = x.shape
    if N != Hg * Wg:
        raise ValueError("N must equal Hg * Wg")
    ws, nbytes = _workspace(ttt_vit3_block_workspace_bytes(B, Hg, Wg, C, H, dt), workspace, x.device)
    rc = lib().ttt_vit3_block(_ptr(x), _ptr(wqkvg), _ptr(w0), _ptr(wc), _ptr(wo), _ptr(y), B, Hg, Wg, C, H,
                              float(eta), dt, _ptr(ws), nbytes, _stream(stream))
    _check("ttt_vit3_block", rc)
    return y


def vit3_block(x, wqkvg, w0, wc, wo, Hg, Wg, H, eta=1.0):
    y = torch.empty_like(x)
    return ttt_vit3_block(x, wqkvg, w0, wc, wo, y, Hg, Wg, H, eta)


def ttt_linear_fullbatch_bwd_workspace_bytes(B, H, N, d, dtype):
    return lib().ttt_linear_fullbatch_bwd_workspace_bytes(B, H, N, d, dtype)


def ttt_linear_fullbatch_bwd(q, k, v, w0, dout, dq, dk, dv, dw0, eta=1.0, workspace=None, stream=None):
    """Gradients of the full-batch TTT-Linear layer: dq, dk, dv [B,H,N,d] (dtype of q), dw0 [H,d,d] fp32."""
    dt = _dtype(q, k, v, dout, dq, dk, dv)
    _weights(w0, dw0)
    B, H, N, d = q.shape
    ws, nbytes = _workspace(ttt_linear_fullbatch_bwd_workspace_bytes(B, H, N, d, dt), workspace, q.device)
    rc = lib().ttt_linear_fullbatch_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(w0), _ptr(dout), _ptr(dq), _ptr(dk),
                                        _ptr(dv), _ptr(dw0), B, H, N, d, float(eta), dt, _ptr(ws), nbytes,
                                        _stream(stream))
    _check("ttt_linear_fullbatch_bwd", rc)
    return dq, dk, dv, dw0


def ttt_dwconv_fullbatch_workspace_bytes(B, Hg, Wg, C, dtype):
    return lib().ttt_dwconv_fullbatch_workspace_bytes(B, Hg, Wg, C, dtype)


def ttt_dwconv_fullbatch(q, k, v, w0, out, w_star=None, eta=1.0, workspace=None, stream=None):
    """q, k, v, out [B,Hg,Wg,C] channels-last; w0 [C,3,3] fp32; w_star [B,C,3,3] fp32 or None."""
    dt = _dtype(q, k, v, out)
    _weights(w0, w_star)
    B, Hg, Wg, C = q.shape
    ws, nbytes = _workspace(ttt_dwconv_fullbatch_workspace_bytes(B, Hg, Wg, C, dt), workspace, q.device)
    rc = lib().ttt_dwconv_fullbatch(_ptr(q), _ptr(k), _ptr(v), _ptr(w0), _ptr(out), _ptr(w_star), B, Hg, Wg,
                                    C, float(eta), dt, _ptr(ws), nbytes, _stream(stream))
    _check("ttt_dwconv_fullbatch", rc)
    return out


def ttt_mlp_fullbatch_workspace_bytes(B, H, N, d, hidden, dtype):
    return lib().ttt_mlp_fullbatch_workspace_bytes(B, H, N, d, hidden, dtype)


def ttt_mlp_fullbatch(q, k, v, w1, w2, out, w1_star=None, w2_star=None, eta=1.0, workspace=None,
                      stream=None):
    """q, k, v, out [B,H,N,d]; w1 [H,d,h], w2 [H,h,d] fp32; optional fp32 updated weights."""
    dt = _dtype(q, k, v, out)
    _weights(w1, w2, w1_star, w2_star)
    B, H, N, d = q.shape
    hidden = w1.shape[2]
    ws, nbytes = _workspace(ttt_mlp_fullbatch_workspace_bytes(B, H, N, d, hidden, dt), workspace, q.device)
    rc = lib().ttt_mlp_fullbatch(_ptr(q), _ptr(k), _ptr(v), _ptr(w1), _ptr(w2), _ptr(out), _ptr(w1_star),
                                 _ptr(w2_star), B, H, N, d, hidden, float(eta), dt, _ptr(ws), nbytes,
                                 _stream(stream))
    _check("ttt_mlp_fullbatch", rc)
    return out


def ttt_linear_chunked_bidir_workspace_bytes(B, H, N, d, chunk, dtype):
    return lib().ttt_linear_chunked_bidir_workspace_bytes(B, H, N, d, chunk, dtype)


def ttt_linear_chunked_bidir(q, k, v, w0, out, chunk, eta=1.0, workspace=None, stream=None):
    """q, k, v, out [B,H,N,d]; w0 [H,d,d] fp32; N % chunk == 0."""
    dt = _dtype(q, k, v, out)
    _weights(w0)
    B, H, N, d = q.shape
    ws, nbytes = _workspace(ttt_linear_chunked_bidir_workspace_bytes(B, H, N, d, chunk, dt), workspace,
                            q.device)
    rc = lib().ttt_linear_chunked_bidir(_ptr(q), _ptr(k), _ptr(v), _ptr(w0), _ptr(out), B, H, N, d,
                                        int(chunk), float(eta), dt, _ptr(ws), nbytes, _stream(stream))
    _check("ttt_linear_chunked_bidir", rc)
    return out


def ttt_linear_chunked_workspace_bytes(B, H, N, d, chunk, direction, dtype):
    return lib().ttt_linear_chunked_workspace_bytes(B, H, N, d, chunk, direction, dtype)


def ttt_linear_chunked(q, k, v, w0, out, chunk, eta=1.0, direction=0, workspace=None, stream=None):
    """One-way (direction +1 raster, -1 reverse) or bidirectional (0) chunked scan."""
    dt = _dtype(q, k, v, out)
    _weights(w0)
    B, H, N, d = q.shape
    ws, nbytes = _workspace(ttt_linear_chunked_workspace_bytes(B, H, N, d, chunk, direction, dt), workspace,
                            q.device)
    rc = lib().ttt_linear_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(w0), _ptr(out), B, H, N, d, int(chunk),
                                  float(eta), int(direction), dt, _ptr(ws), nbytes, _stream(stream))
    _check("ttt_linear_chunked", rc)
    return out


def ttt_linear_minibatch_workspace_bytes(B, H, N, d, chunk, epochs, dtype):
    return lib().ttt_linear_minibatch_workspace_bytes(B, H, N, d, chunk, epochs, dtype)


def ttt_linear_minibatch(q, k, v, w0, out, chunk, epochs=1, w_final=None, eta=1.0, workspace=None, stream=None):
    """`epochs` epochs of mini-batch inner training (chunks of `chunk` tokens), then out = Q W_final."""
    dt = _dtype(q, k, v, out)
    _weights(w0, w_final)
    B, H, N, d = q.shape
    ws, nbytes = _workspace(ttt_linear_minibatch_workspace_bytes(B, H, N, d, chunk, epochs, dt), workspace,
                            q.device)
    rc = lib().ttt_linear_minibatch(_ptr(q), _ptr(k), _ptr(v), _ptr(w0), _ptr(out), _ptr(w_final), B, H, N, d,
                                    int(chunk), int(epochs), float(eta), dt, _ptr(ws), nbytes, _stream(stream))
    _check("ttt_linear_minibatch", rc)
    return out


def ttt_linear_chunked_conv_workspace_bytes(B, H, Hg, Wg, d, chunk, direction, dtype):
    return lib().ttt_linear_chunked_conv_workspace_bytes(B, H, Hg, Wg, d, chunk, direction, dtype)


def ttt_linear_chunked_conv(q, k, v, w0, wk, wv, out, Hg, Wg, chunk, eta=1.0, direction=0, workspace=None,
                            stream=None):
    """Chunked scan on (Q, conv3x3(K; wk), conv3x3(V; wv)) over the Hg x Wg token grid."""
    dt = _dtype(q, k, v, out)
    _weights(w0, wk, wv)
    B, H, N, d = q.shape
    if N != Hg * Wg:
        raise ValueError("N must equal Hg * Wg")
    ws, nbytes = _workspace(ttt_linear_chunked_conv_workspace_bytes(B, H, Hg, Wg, d, chunk, direction, dt),
                            workspace, q.device)
    rc = lib().ttt_linear_chunked_conv(_ptr(q), _ptr(k), _ptr(v), _ptr(w0), _ptr(wk), _ptr(wv), _ptr(out), B, H,
                                       Hg, Wg, d, int(chunk), float(eta), int(direction), dt, _ptr(ws), nbytes,
                                       _stream(stream))
    _check("ttt_linear_chunked_conv", rc)
    return out


def ttt_linear_chunked_bidir_noalloc(q, k, v, w0, out, chunk, eta=1.0, stream=None):
    """The chunked scan without a workspace argument: for callers that may not allocate
    device memory at call time.  Its scratch is a fixed array inside the library's device
    image (ttt_linear_chunked_bidir_noalloc_max_bytes() long); calls that overlap on the GPU
    race on it."""
    dt = _dtype(q, k, v, out)
    _weights(w0)
    B, H, N, d = q.shape
    rc = lib().ttt_linear_chunked_bidir_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(w0), _ptr(out), B, H, N, d,
                                                int(chunk), float(eta), dt, _stream(stream))
    _check("ttt_linear_chunked_bidir_noalloc", rc)
    return out


TTT_FAULT_SKIP_LOAD = 0x1


def debug_set_wait_limit(cycles: int) -> None:
    """Bounded-wait limit (SM cycles) of kernels launched afterwards; <= 0 restores the default."""
    _check("ttt_debug_set_wait_limit", lib().ttt_debug_set_wait_limit(int(cycles)))


def debug_arm_fault(bits: int) -> None:
    """Arm (bits != 0) or clear (0) the simulated lost-transfer test hook."""
    _check("ttt_debug_arm_fault", lib().ttt_debug_arm_fault(int(bits)))


def kernel_launch_count() -> int:
    return int(lib().ttt_kernel_launch_count())


def device_error() -> int:
    """Synchronise and return (and clear) the device error bits; raises on a timeout."""
    bits = ctypes.c_uint(0)
    rc = lib().ttt_device_error(ctypes.byref(bits))
    if rc != 0:
        raise TTTError("ttt_device_error", rc)
    return bits.value


# ----------------------------------------------------------------------- conveniences --
def linear_fullbatch(q, k, v, w0, eta=1.0, with_w_star=False):
    out = torch.empty_like(q)
    ws = torch.empty((q.shape[0], q.shape[1], q.shape[3], q.shape[3]), dtype=torch.float32,
                     device=q.device) if with_w_star else None
    ttt_linear_fullbatch(q, k, v, w0, out, ws, eta)
    return (out, ws) if with_w_star else out


def linear_fullbatch_bwd(q, k, v, w0, dout, eta=1.0):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dw0 = torch.empty_like(w0)
    return ttt_linear_fullbatch_bwd(q, k, v, w0, dout, dq, dk, dv, dw0, eta)


def dwconv_fullbatch(q, k, v, w0, eta=1.0, with_w_star=False):
    out = torch.empty_like(q)
    ws = torch.empty((q.shape[0], q.shape[3], 3, 3), dtype=torch.float32,
                     device=q.device) if with_w_star else None
    ttt_dwconv_fullbatch(q, k, v, w0, out, ws, eta)
    return (out, ws) if with_w_star else out


def mlp_fullbatch(q, k, v, w1, w2, eta=1.0, with_w_star=False):
    out = torch.empty_like(q)
    B, H, _, d = q.shape
    h = w1.shape[2]
    w1s = torch.empty((B, H, d, h), dtype=torch.float32, device=q.device) if with_w_star else None
    w2s = torch.empty((B, H, h, d), dtype=torch.float32, device=q.device) if with_w_star else None
    ttt_mlp_fullbatch(q, k, v, w1, w2, out, w1s, w2s, eta)
    return (out, w1s, w2s) if with_w_star else out


def linear_chunked(q, k, v, w0, chunk, eta=1.0, direction=0):
    out = torch.empty_like(q)
    ttt_linear_chunked(q, k, v, w0, out, chunk, eta, direction)
    return out


def linear_minibatch(q, k, v, w0, chunk, epochs=1, eta=1.0, with_w_final=False):
    out = torch.empty_like(q)
    wf = torch.empty((q.shape[0], q.shape[1], q.shape[3], q.shape[3]), dtype=torch.float32,
                     device=q.device) if with_w_final else None
    ttt_linear_minibatch(q, k, v, w0, out, chunk, epochs, wf, eta)
    return (out, wf) if with_w_final else out


def linear_chunked_conv(q, k, v, w0, wk, wv, Hg, Wg, chunk, eta=1.0, direction=0):
    out = torch.empty_like(q)
    ttt_linear_chunked_conv(q, k, v, w0, wk, wv, out, Hg, Wg, chunk, eta, direction)
    return out


def linear_chunked_bidir(q, k, v, w0, chunk, eta=1.0):
    out = torch.empty_like(q)
    ttt_linear_chunked_bidir(q, k, v, w0, out, chunk, eta)
    return out
