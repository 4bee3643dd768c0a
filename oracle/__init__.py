"""ctypes front end of the fp64 CPU oracle for the TTT layer.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's CPU-baseline /
reference leg import this package.  The product (the CUDA library and its binding) never
does.  Inputs are converted to float64 exactly (bf16 and fp32 values widen without
rounding), so the oracle sees the same numbers the GPU sees.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        d, i, p = ctypes.c_double, ctypes.c_int, ctypes.c_void_p
        _lib.ttt_oracle_linear_loss.restype = d
        _lib.ttt_oracle_linear_loss.argtypes = [p, p, p, i, i]
        _lib.ttt_oracle_linear_grad.restype = None
        _lib.ttt_oracle_linear_grad.argtypes = [p, p, p, i, i, p]
        _lib.ttt_oracle_linear_fullbatch.restype = i
        _lib.ttt_oracle_linear_fullbatch.argtypes = [p, p, p, p, p, p, i, i, i, i, d, i]
        _lib.ttt_oracle_dwconv_loss.restype = d
        _lib.ttt_oracle_dwconv_loss.argtypes = [p, p, p, i, i, i]
        _lib.ttt_oracle_dwconv_grad.restype = None
        _lib.ttt_oracle_dwconv_grad.argtypes = [p, p, p, i, i, i, p]
        _lib.ttt_oracle_dwconv_fullbatch.restype = i
        _lib.ttt_oracle_dwconv_fullbatch.argtypes = [p, p, p, p, p, p, i, i, i, i, d, i]
        _lib.ttt_oracle_gelu_tanh.restype = d
        _lib.ttt_oracle_gelu_tanh.argtypes = [d]
        _lib.ttt_oracle_gelu_tanh_grad.restype = d
        _lib.ttt_oracle_gelu_tanh_grad.argtypes = [d]
        _lib.ttt_oracle_mlp_loss.restype = d
        _lib.ttt_oracle_mlp_loss.argtypes = [p, p, p, p, i, i, i]
        _lib.ttt_oracle_mlp_grad.restype = None
        _lib.ttt_oracle_mlp_grad.argtypes = [p, p, p, p, i, i, i, p, p]
        _lib.ttt_oracle_mlp_fullbatch.restype = i
        _lib.ttt_oracle_mlp_fullbatch.argtypes = [p, p, p, p, p, p, p, p, i, i, i, i, i, d, i]
        _lib.ttt_oracle_linear_chunked.restype = i
        _lib.ttt_oracle_linear_chunked.argtypes = [p, p, p, p, p, i, i, i, i, i, d, i, i]
        _lib.ttt_oracle_linear_fullbatch_bwd.restype = i
        _lib.ttt_oracle_linear_fullbatch_bwd.argtypes = [p, p, p, p, p, p, p, p, p, i, i, i, i, d, i]
        _lib.ttt_oracle_linear_minibatch.restype = i
        _lib.ttt_oracle_linear_minibatch.argtypes = [p, p, p, p, p, p, i, i, i, i, i, i, d, i]
        _lib.ttt_oracle_dwconv_prep.restype = None
        _lib.ttt_oracle_dwconv_prep.argtypes = [p, p, p, i, i, i, i, i]
        _lib.ttt_oracle_vit3_block.restype = i
        _lib.ttt_oracle_vit3_block.argtypes = [p, p, p, p, p, p, i, i, i, i, i, d, i]
        _lib.ttt_oracle_linear_chunked_prep.restype = i
        _lib.ttt_oracle_linear_chunked_prep.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, i, d, i, i]
    return _lib


def default_threads() -> int:
    return os.cpu_count() or 1


def _f64(x) -> np.ndarray:
    """Exact widening to a contiguous float64 numpy array (accepts numpy or torch CPU)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- TTT-Linear ---------
def linear_loss(k, v, w) -> float:
    k, v, w = _f64(k), _f64(v), _f64(w)
    N, d = k.shape
    return lib().ttt_oracle_linear_loss(_p(k), _p(v), _p(w), N, d)


def linear_grad(k, v, w) -> np.ndarray:
    k, v, w = _f64(k), _f64(v), _f64(w)
    N, d = k.shape
    g = np.empty((d, d))
    lib().ttt_oracle_linear_grad(_p(k), _p(v), _p(w), N, d, _p(g))
    return g


def linear_fullbatch(q, k, v, w0, eta=1.0, threads=None):
    """q,k,v [B,H,N,d]; w0 [H,d,d] -> (out [B,H,N,d], w_star [B,H,d,d]) in float64."""
    q, k, v, w0 = _f64(q), _f64(k), _f64(v), _f64(w0)
    B, H, N, d = q.shape
    out = np.empty_like(q)
    ws = np.empty((B, H, d, d))
    rc = lib().ttt_oracle_linear_fullbatch(_p(q), _p(k), _p(v), _p(w0), _p(out), _p(ws),
                                           B, H, N, d, float(eta), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out, ws


# ---------------------------------------------------------------- 3x3 depthwise conv ---
def dwconv_loss(k, v, w) -> float:
    """k, v [Hg, Wg, C] one image; w [C, 3, 3]."""
    k, v, w = _f64(k), _f64(v), _f64(w)
    Hg, Wg, C = k.shape
    return lib().ttt_oracle_dwconv_loss(_p(k), _p(v), _p(w), Hg, Wg, C)


def dwconv_grad(k, v, w) -> np.ndarray:
    k, v, w = _f64(k), _f64(v), _f64(w)
    Hg, Wg, C = k.shape
    g = np.empty((C, 3, 3))
    lib().ttt_oracle_dwconv_grad(_p(k), _p(v), _p(w), Hg, Wg, C, _p(g))
    return g


def dwconv_fullbatch(q, k, v, w0, eta=1.0, threads=None):
    """q,k,v [B,Hg,Wg,C]; w0 [C,3,3] -> (out [B,Hg,Wg,C], w_star [B,C,3,3])."""
    q, k, v, w0 = _f64(q), _f64(k), _f64(v), _f64(w0)
    B, Hg, Wg, C = q.shape
    out = np.empty_like(q)
    ws = np.empty((B, C, 3, 3))
    rc = lib().ttt_oracle_dwconv_fullbatch(_p(q), _p(k), _p(v), _p(w0), _p(out), _p(ws),
                                           B, Hg, Wg, C, float(eta), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out, ws


# ---------------------------------------------------------------- TTT-MLP ---------------
def gelu_tanh(u: float) -> float:
    return lib().ttt_oracle_gelu_tanh(float(u))


def gelu_tanh_grad(u: float) -> float:
    return lib().ttt_oracle_gelu_tanh_grad(float(u))


def mlp_loss(k, v, w1, w2) -> float:
    k, v, w1, w2 = _f64(k), _f64(v), _f64(w1), _f64(w2)
    N, d = k.shape
    h = w1.shape[1]
    return lib().ttt_oracle_mlp_loss(_p(k), _p(v), _p(w1), _p(w2), N, d, h)


def mlp_grad(k, v, w1, w2):
    k, v, w1, w2 = _f64(k), _f64(v), _f64(w1), _f64(w2)
    N, d = k.shape
    h = w1.shape[1]
    g1 = np.empty((d, h))
    g2 = np.empty((h, d))
    lib().ttt_oracle_mlp_grad(_p(k), _p(v), _p(w1), _p(w2), N, d, h, _p(g1), _p(g2))
    return g1, g2


def mlp_fullbatch(q, k, v, w1, w2, eta=1.0, threads=None):
    """q,k,v [B,H,N,d]; w1 [H,d,h]; w2 [H,h,d] -> (out, w1_star [B,H,d,h], w2_star [B,H,h,d])."""
    q, k, v, w1, w2 = _f64(q), _f64(k), _f64(v), _f64(w1), _f64(w2)
    B, H, N, d = q.shape
    h = w1.shape[2]
    out = np.empty_like(q)
    w1s = np.empty((B, H, d, h))
    w2s = np.empty((B, H, h, d))
    rc = lib().ttt_oracle_mlp_fullbatch(_p(q), _p(k), _p(v), _p(w1), _p(w2), _p(out), _p(w1s),
                                        _p(w2s), B, H, N, d, h, float(eta),
                                        threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out, w1s, w2s


# ---------------------------------------------------------------- chunked scan ---------
def linear_chunked(q, k, v, w0, chunk, eta=1.0, direction=0, threads=None) -> np.ndarray:
    """direction +1 raster, -1 reverse raster, 0 both summed.  -> out [B,H,N,d]."""
    q, k, v, w0 = _f64(q), _f64(k), _f64(v), _f64(w0)
    B, H, N, d = q.shape
    out = np.empty_like(q)
    rc = lib().ttt_oracle_linear_chunked(_p(q), _p(k), _p(v), _p(w0), _p(out), B, H, N, d,
                                         int(chunk), float(eta), int(direction),
                                         threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out


# ---------------------------------------------------------------- backward --------------
def linear_fullbatch_bwd(q, k, v, w0, dout, eta=1.0, threads=None):
    """Gradients of the full-batch TTT-Linear layer for the upstream gradient `dout`:
    q,k,v,dout [B,H,N,d]; w0 [H,d,d] -> (dq, dk, dv [B,H,N,d], dw0 [H,d,d] summed over B)."""
    q, k, v, w0, g = _f64(q), _f64(k), _f64(v), _f64(w0), _f64(dout)
    B, H, N, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    dw0 = np.empty((H, d, d))
    rc = lib().ttt_oracle_linear_fullbatch_bwd(_p(q), _p(k), _p(v), _p(w0), _p(g), _p(dq), _p(dk),
                                               _p(dv), _p(dw0), B, H, N, d, float(eta),
                                               threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return dq, dk, dv, dw0


# ---------------------------------------------------------------- mini-batch / epochs ---
def linear_minibatch(q, k, v, w0, chunk, epochs=1, eta=1.0, threads=None):
    """E epochs of mini-batch inner training in raster order, then out = Q W_final.
    -> (out [B,H,N,d], w_final [B,H,d,d])."""
    q, k, v, w0 = _f64(q), _f64(k), _f64(v), _f64(w0)
    B, H, N, d = q.shape
    out = np.empty_like(q)
    wf = np.empty((B, H, d, d))
    rc = lib().ttt_oracle_linear_minibatch(_p(q), _p(k), _p(v), _p(w0), _p(out), _p(wf), B, H, N, d,
                                           int(chunk), int(epochs), float(eta),
                                           threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out, wf


# ---------------------------------------------------------------- conv preprocessing ----
def dwconv_prep(x, w, Hg, Wg):
    """3x3 depthwise conv (zero padding) of x [B,H,Hg*Wg,d] with taps w [H,d,3,3]."""
    x, w = _f64(x), _f64(w)
    B, H, N, d = x.shape
    assert N == Hg * Wg
    out = np.empty_like(x)
    lib().ttt_oracle_dwconv_prep(_p(x), _p(w), _p(out), B, H, Hg, Wg, d)
    return out


def linear_chunked_prep(q, k, v, w0, wk, wv, Hg, Wg, chunk, eta=1.0, direction=0, threads=None):
    """Chunked scan on (Q, conv(K; wk), conv(V; wv)) over the Hg x Wg grid."""
    q, k, v, w0, wk, wv = _f64(q), _f64(k), _f64(v), _f64(w0), _f64(wk), _f64(wv)
    B, H, N, d = q.shape
    assert N == Hg * Wg
    out = np.empty_like(q)
    rc = lib().ttt_oracle_linear_chunked_prep(_p(q), _p(k), _p(v), _p(w0), _p(wk), _p(wv), _p(out),
                                              B, H, Hg, Wg, d, int(chunk), float(eta), int(direction),
                                              threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out


# ---------------------------------------------------------------- the ViT^3 block -------
def vit3_block(x, wqkvg, w0, wc, wo, Hg, Wg, H, eta=1.0, threads=None):
    """x [B, Hg*Wg, C] -> y [B, Hg*Wg, C] (projections, TTT-Linear core per head, GLU gate,
    3x3 depthwise-conv branch on x, concat, output projection)."""
    x, wqkvg, w0, wc, wo = _f64(x), _f64(wqkvg), _f64(w0), _f64(wc), _f64(wo)
    B, N, C = x.shape
    assert N == Hg * Wg
    y = np.empty_like(x)
    rc = lib().ttt_oracle_vit3_block(_p(x), _p(wqkvg), _p(w0), _p(wc), _p(wo), _p(y), B, Hg, Wg, C, H,
                                     float(eta), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return y
