"""Pins of the fp64 CPU oracle to facts other than itself.

Each test checks the oracle against something the definition or the mathematics fixes:
hand-worked examples (tests/golden), closed forms, finite differences, torch autograd of
library operators (an independent derivative of the same loss), library routines for
special cases (conv2d, gelu), invariants.  They are chosen so that a plausible slip in the
oracle (a dropped 1/N, a sign, a transposed operand, a convolution flipped into a
correlation, the chunk output taken before the update) fails at least one of them.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

RNG = np.random.default_rng(1234)


def rnd(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ============================================================== TTT-Linear ============
def test_linear_golden(golden_dir):
    g = load(golden_dir, "linear_d2_n2.json")
    k, v, w0, q = (np.array(g[x], float) for x in ("k", "v", "w0", "q"))
    assert oracle.linear_loss(k, v, w0) == pytest.approx(g["loss_w0"], abs=1e-15)
    np.testing.assert_allclose(oracle.linear_grad(k, v, w0), g["grad_w0"], atol=1e-15)
    out, ws = oracle.linear_fullbatch(q[None, None], k[None, None], v[None, None], w0[None],
                                      eta=g["eta"])
    np.testing.assert_allclose(ws[0, 0], g["w_star"], atol=1e-15)
    np.testing.assert_allclose(out[0, 0], g["out"], atol=1e-15)


def test_linear_gram_closed_form():
    """I1: the per-token-loop step equals W0 - (eta/N)(K^T K W0 - K^T V) (numpy matmul)."""
    B, H, N, d = 2, 3, 37, 8
    q, k, v = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
    w0 = rnd(H, d, d, scale=0.3)
    eta = 0.37
    out, ws = oracle.linear_fullbatch(q, k, v, w0, eta=eta)
    for b in range(B):
        for h in range(H):
            K, V = k[b, h], v[b, h]
            ref = w0[h] - (eta / N) * (K.T @ K @ w0[h] - K.T @ V)
            np.testing.assert_allclose(ws[b, h], ref, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(out[b, h], q[b, h] @ ref, rtol=1e-11, atol=1e-12)


def test_linear_grad_autograd():
    """The hand-derived gradient equals torch autograd of the loss built from torch ops."""
    N, d = 23, 6
    k, v, w = rnd(N, d), rnd(N, d), rnd(d, d)
    W = torch.tensor(w, requires_grad=True)
    loss = 0.5 * ((torch.tensor(k) @ W - torch.tensor(v)) ** 2).sum(dim=1).mean()
    loss.backward()
    np.testing.assert_allclose(oracle.linear_grad(k, v, w), W.grad.numpy(), rtol=1e-12,
                               atol=1e-13)
    assert oracle.linear_loss(k, v, w) == pytest.approx(loss.item(), rel=1e-13)


def fd_grad(loss_fn, w, eps=1e-6):
    g = np.zeros_like(w)
    flat = w.reshape(-1)
    for i in range(flat.size):
        wp, wm = flat.copy(), flat.copy()
        wp[i] += eps
        wm[i] -= eps
        g.reshape(-1)[i] = (loss_fn(wp.reshape(w.shape)) - loss_fn(wm.reshape(w.shape))) / (2 * eps)
    return g


def test_linear_finite_difference():
    """I2: central differences of l(W) match the analytic gradient."""
    N, d = 16, 4
    k, v, w = rnd(N, d), rnd(N, d), rnd(d, d)
    fd = fd_grad(lambda ww: oracle.linear_loss(k, v, ww), w)
    an = oracle.linear_grad(k, v, w)
    np.testing.assert_allclose(an, fd, rtol=1e-7, atol=1e-8)


def test_linear_eta_zero_and_fixed_point():
    """I3: eta = 0 gives O = Q W0.  I4: V = K W0 gives W* = W0 exactly."""
    B, H, N, d = 1, 2, 9, 5
    q, k = rnd(B, H, N, d), rnd(B, H, N, d)
    w0 = rnd(H, d, d)
    out, ws = oracle.linear_fullbatch(q, k, rnd(B, H, N, d), w0, eta=0.0)
    for h in range(H):
        np.testing.assert_allclose(out[0, h], q[0, h] @ w0[h], rtol=1e-12, atol=1e-12)
    # V = K W0 computed with integers so that the residual is exactly zero
    ki = RNG.integers(-3, 4, size=(B, H, N, d)).astype(float)
    wi = RNG.integers(-2, 3, size=(H, d, d)).astype(float)
    vi = np.einsum("bhnd,hde->bhne", ki, wi)
    _, ws = oracle.linear_fullbatch(q, ki, vi, wi, eta=1.0)
    for h in range(H):
        assert np.array_equal(ws[0, h], wi[h])


def test_linear_zero_init_is_linear_attention():
    """I5: W0 = 0 gives O = (eta/N) Q (K^T V), and (I10) O is linear in V."""
    B, H, N, d = 2, 1, 31, 7
    q, k, v = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
    w0 = np.zeros((H, d, d))
    eta = 1.0
    out, _ = oracle.linear_fullbatch(q, k, v, w0, eta=eta)
    for b in range(B):
        ref = (eta / N) * q[b, 0] @ (k[b, 0].T @ v[b, 0])
        np.testing.assert_allclose(out[b, 0], ref, rtol=1e-12, atol=1e-13)
    out2, _ = oracle.linear_fullbatch(q, k, -2.5 * v, w0, eta=eta)
    np.testing.assert_allclose(out2, -2.5 * out, rtol=1e-12, atol=1e-13)


# ============================================================== depthwise conv ========
def conv_torch(x_hwc, w_c33):
    """Library depthwise cross-correlation (torch conv2d, groups = C, zero padding 1)."""
    x = torch.tensor(x_hwc).permute(2, 0, 1)[None]
    w = torch.tensor(w_c33)[:, None]
    return F.conv2d(x, w, padding=1, groups=x.shape[1])[0].permute(1, 2, 0)


def test_dwconv_golden(golden_dir):
    g = load(golden_dir, "dwconv_2x2_c1.json")
    k, v, q = (np.array(g[x], float)[..., None] for x in ("k", "v", "q"))
    w0 = np.array(g["w0"], float)[None]
    assert oracle.dwconv_loss(k, v, w0) == pytest.approx(g["loss_w0"], abs=1e-15)
    np.testing.assert_allclose(oracle.dwconv_grad(k, v, w0)[0], g["grad_w0"], atol=1e-15)
    out, ws = oracle.dwconv_fullbatch(q[None], k[None], v[None], w0, eta=g["eta"])
    np.testing.assert_allclose(ws[0, 0], g["w_star"], atol=1e-15)
    np.testing.assert_allclose(out[0, :, :, 0], g["out"], atol=1e-15)


def test_dwconv_forward_is_library_correlation():
    """I3 with the library: eta = 0 gives O = conv2d(Q, w0) with an asymmetric kernel."""
    B, Hg, Wg, C = 2, 5, 7, 3
    q, k, v = rnd(B, Hg, Wg, C), rnd(B, Hg, Wg, C), rnd(B, Hg, Wg, C)
    w0 = rnd(C, 3, 3)
    out, ws = oracle.dwconv_fullbatch(q, k, v, w0, eta=0.0)
    for b in range(B):
        np.testing.assert_allclose(out[b], conv_torch(q[b], w0).numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(ws[b], w0)


def test_dwconv_grad_autograd_and_fd():
    Hg, Wg, C = 4, 3, 2
    k, v, w = rnd(Hg, Wg, C), rnd(Hg, Wg, C), rnd(C, 3, 3)
    W = torch.tensor(w, requires_grad=True)
    x = torch.tensor(k).permute(2, 0, 1)[None]
    f = F.conv2d(x, W[:, None], padding=1, groups=C)[0].permute(1, 2, 0)
    loss = 0.5 * ((f - torch.tensor(v)) ** 2).sum(dim=2).mean()
    loss.backward()
    an = oracle.dwconv_grad(k, v, w)
    np.testing.assert_allclose(an, W.grad.numpy(), rtol=1e-12, atol=1e-13)
    assert oracle.dwconv_loss(k, v, w) == pytest.approx(loss.item(), rel=1e-13)
    fd = fd_grad(lambda ww: oracle.dwconv_loss(k, v, ww), w)
    np.testing.assert_allclose(an, fd, rtol=1e-7, atol=1e-8)


def im2col(x_hw):
    """Phi [N, 9]: column a*3+b is the zero-padded image shifted by (a-1, b-1)."""
    Hg, Wg = x_hw.shape
    p = np.pad(x_hw, 1)
    cols = [p[a:a + Hg, b:b + Wg].reshape(-1) for a in range(3) for b in range(3)]
    return np.stack(cols, axis=1)


def test_dwconv_regression_closed_form():
    """I7: per channel the conv model is linear in its taps: w* = w0 - (eta/N)(Phi^T Phi w0 - Phi^T v)."""
    B, Hg, Wg, C = 2, 6, 5, 3
    q, k, v = rnd(B, Hg, Wg, C), rnd(B, Hg, Wg, C), rnd(B, Hg, Wg, C)
    w0 = rnd(C, 3, 3)
    eta = 0.8
    N = Hg * Wg
    out, ws = oracle.dwconv_fullbatch(q, k, v, w0, eta=eta)
    for b in range(B):
        for c in range(C):
            phi = im2col(k[b, :, :, c])
            ref = w0[c].reshape(-1) - (eta / N) * (phi.T @ phi @ w0[c].reshape(-1)
                                                   - phi.T @ v[b, :, :, c].reshape(-1))
            np.testing.assert_allclose(ws[b, c].reshape(-1), ref, rtol=1e-12, atol=1e-12)
            o_ref = im2col(q[b, :, :, c]) @ ref
            np.testing.assert_allclose(out[b, :, :, c].reshape(-1), o_ref, rtol=1e-11, atol=1e-12)


def test_dwconv_single_pixel_and_fixed_point():
    """A 1x1 grid is a scalar regression on the centre tap (other taps get zero gradient);
    V = conv(K, w0) gives w* = w0 exactly."""
    k, v, w = rnd(1, 1, 2), rnd(1, 1, 2), rnd(2, 3, 3)
    g = oracle.dwconv_grad(k, v, w)
    for c in range(2):
        mask = np.ones((3, 3), bool)
        mask[1, 1] = False
        assert np.all(g[c][mask] == 0.0)
        assert g[c, 1, 1] == pytest.approx((w[c, 1, 1] * k[0, 0, c] - v[0, 0, c]) * k[0, 0, c],
                                           rel=1e-14)
    ki = RNG.integers(-3, 4, size=(1, 4, 5, 2)).astype(float)
    wi = RNG.integers(-2, 3, size=(2, 3, 3)).astype(float)
    vi = conv_torch(ki[0], wi).numpy()[None]
    _, ws = oracle.dwconv_fullbatch(ki, ki, vi, wi, eta=1.0)
    assert np.array_equal(ws[0], wi)


# ============================================================== TTT-MLP ===============
def test_gelu_against_library():
    us = np.linspace(-6, 6, 241)
    x = torch.tensor(us, requires_grad=True)
    y = F.gelu(x, approximate="tanh")
    y.sum().backward()
    for i, u in enumerate(us):
        assert oracle.gelu_tanh(u) == pytest.approx(y[i].item(), rel=1e-13, abs=1e-15)
        assert oracle.gelu_tanh_grad(u) == pytest.approx(x.grad[i].item(), rel=1e-12, abs=1e-14)


def test_mlp_golden(golden_dir):
    g = load(golden_dir, "mlp_d1_h2.json")
    k, v, q, w1, w2 = (np.array(g[x], float) for x in ("k", "v", "q", "w1", "w2"))
    rt = g["rtol"]
    assert oracle.mlp_loss(k, v, w1, w2) == pytest.approx(g["loss_w0"], rel=rt)
    g1, g2 = oracle.mlp_grad(k, v, w1, w2)
    np.testing.assert_allclose(g1, g["grad_w1"], rtol=rt, atol=1e-15)
    np.testing.assert_allclose(g2, g["grad_w2"], rtol=rt, atol=1e-15)
    out, w1s, w2s = oracle.mlp_fullbatch(q[None, None], k[None, None], v[None, None], w1[None],
                                         w2[None], eta=g["eta"])
    np.testing.assert_allclose(w1s[0, 0], g["w1_star"], rtol=rt)
    np.testing.assert_allclose(w2s[0, 0], g["w2_star"], rtol=rt)
    np.testing.assert_allclose(out[0, 0], g["out"], rtol=rt)


def test_mlp_golden_regenerates(golden_dir):
    """The MLP fixture is reproduced bit for bit by its committed calculator program
    (Python math only, nothing from the oracle)."""
    import subprocess
    import sys
    script = os.path.join(golden_dir, "make_mlp_d1_h2.py")
    r = subprocess.run([sys.executable, script, "--check"], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


def mlp_torch_loss(k, v, W1, W2):
    a = F.gelu(torch.tensor(k) @ W1, approximate="tanh")
    return 0.5 * ((a @ W2 - torch.tensor(v)) ** 2).sum(dim=1).mean()


def test_mlp_grad_autograd_and_fd():
    N, d, h = 12, 3, 8
    k, v = rnd(N, d), rnd(N, d)
    w1, w2 = rnd(d, h, scale=0.7), rnd(h, d, scale=0.5)
    W1 = torch.tensor(w1, requires_grad=True)
    W2 = torch.tensor(w2, requires_grad=True)
    loss = mlp_torch_loss(k, v, W1, W2)
    loss.backward()
    g1, g2 = oracle.mlp_grad(k, v, w1, w2)
    np.testing.assert_allclose(g1, W1.grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(g2, W2.grad.numpy(), rtol=1e-11, atol=1e-13)
    assert oracle.mlp_loss(k, v, w1, w2) == pytest.approx(loss.item(), rel=1e-12)
    fd1 = fd_grad(lambda ww: oracle.mlp_loss(k, v, ww, w2), w1)
    fd2 = fd_grad(lambda ww: oracle.mlp_loss(k, v, w1, ww), w2)
    np.testing.assert_allclose(g1, fd1, rtol=1e-7, atol=1e-8)
    np.testing.assert_allclose(g2, fd2, rtol=1e-7, atol=1e-8)


def test_mlp_eta_zero_and_full_step():
    """I3: eta = 0 gives gelu(Q W1) W2.  The full step equals the step taken with autograd."""
    B, H, N, d, h = 2, 2, 10, 4, 16
    q, k, v = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
    w1, w2 = rnd(H, d, h, scale=0.5), rnd(H, h, d, scale=0.25)
    out, w1s, w2s = oracle.mlp_fullbatch(q, k, v, w1, w2, eta=0.0)
    for b in range(B):
        for hh in range(H):
            ref = F.gelu(torch.tensor(q[b, hh]) @ torch.tensor(w1[hh]), approximate="tanh") \
                @ torch.tensor(w2[hh])
            np.testing.assert_allclose(out[b, hh], ref.numpy(), rtol=1e-12, atol=1e-13)
    eta = 1.0
    out, w1s, w2s = oracle.mlp_fullbatch(q, k, v, w1, w2, eta=eta)
    for b in range(B):
        for hh in range(H):
            W1 = torch.tensor(w1[hh], requires_grad=True)
            W2 = torch.tensor(w2[hh], requires_grad=True)
            mlp_torch_loss(k[b, hh], v[b, hh], W1, W2).backward()
            W1s = W1.detach() - eta * W1.grad
            W2s = W2.detach() - eta * W2.grad
            np.testing.assert_allclose(w1s[b, hh], W1s.numpy(), rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(w2s[b, hh], W2s.numpy(), rtol=1e-11, atol=1e-13)
            o = F.gelu(torch.tensor(q[b, hh]) @ W1s, approximate="tanh") @ W2s
            np.testing.assert_allclose(out[b, hh], o.numpy(), rtol=1e-11, atol=1e-13)


def test_mlp_zero_w2_is_kernelised_linear_attention():
    """I8: W2 = 0 gives W1* = W1, W2* = (eta/N) gelu(K W1)^T V, O = (eta/N) gelu(Q W1) gelu(K W1)^T V."""
    N, d, h = 13, 3, 12
    q, k, v = rnd(1, 1, N, d), rnd(1, 1, N, d), rnd(1, 1, N, d)
    w1, w2 = rnd(1, d, h), np.zeros((1, h, d))
    eta = 0.9
    out, w1s, w2s = oracle.mlp_fullbatch(q, k, v, w1, w2, eta=eta)
    gk = F.gelu(torch.tensor(k[0, 0] @ w1[0]), approximate="tanh").numpy()
    gq = F.gelu(torch.tensor(q[0, 0] @ w1[0]), approximate="tanh").numpy()
    np.testing.assert_array_equal(w1s[0, 0], w1[0])
    np.testing.assert_allclose(w2s[0, 0], (eta / N) * gk.T @ v[0, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out[0, 0], (eta / N) * gq @ (gk.T @ v[0, 0]), rtol=1e-11,
                               atol=1e-13)


def test_mlp_fixed_point():
    """I4: V = F_W(K) gives a zero residual, so W* = W exactly."""
    N, d, h = 6, 2, 4
    k = rnd(1, 1, N, d)
    w1, w2 = rnd(1, d, h), rnd(1, h, d)
    a = F.gelu(torch.tensor(k[0, 0] @ w1[0]), approximate="tanh").numpy()
    v = (a @ w2[0])[None, None]
    # the oracle's own forward must reproduce v to the last bit for an exact fixed point,
    # so compare with a tolerance at rounding level instead
    _, w1s, w2s = oracle.mlp_fullbatch(k, k, v, w1, w2, eta=1.0)
    np.testing.assert_allclose(w1s[0, 0], w1[0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(w2s[0, 0], w2[0], rtol=0, atol=1e-14)


# ============================================================== chunked bidirectional ==
def test_chunked_golden(golden_dir):
    g = load(golden_dir, "chunked_d1_n2.json")
    q, k, v = (np.array(g[x], float).reshape(1, 1, 2, 1) for x in ("q", "k", "v"))
    w0 = np.full((1, 1, 1), float(g["w0"]))
    for direction, key in ((1, "chunk1_forward"), (-1, "chunk1_reverse"), (0, "chunk1_bidir")):
        o = oracle.linear_chunked(q, k, v, w0, chunk=1, eta=g["eta"], direction=direction)
        np.testing.assert_allclose(o.reshape(-1), g[key], atol=1e-15)
    o = oracle.linear_chunked(q, k, v, w0, chunk=2, eta=g["eta"], direction=0)
    np.testing.assert_allclose(o.reshape(-1), g["chunk2_bidir"], atol=1e-15)


def test_chunked_full_chunk_equals_fullbatch():
    """I6: one chunk of b = N equals the full-batch step; bidirectional gives twice that."""
    B, H, N, d = 2, 2, 24, 5
    q, k, v = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
    w0 = rnd(H, d, d, scale=0.4)
    full, _ = oracle.linear_fullbatch(q, k, v, w0, eta=0.7)
    for direction in (1, -1):
        o = oracle.linear_chunked(q, k, v, w0, chunk=N, eta=0.7, direction=direction)
        np.testing.assert_allclose(o, full, rtol=1e-11, atol=1e-12)
    o = oracle.linear_chunked(q, k, v, w0, chunk=N, eta=0.7, direction=0)
    np.testing.assert_allclose(o, 2 * full, rtol=1e-11, atol=1e-12)


def torch_chunked(q, k, v, w0, b, eta, reverse):
    """Literal recurrence with autograd: each chunk takes one gradient step of its own loss."""
    N = q.shape[0]
    order = list(range(N))[::-1] if reverse else list(range(N))
    W = torch.tensor(w0)
    out = np.zeros_like(q)
    for c0 in range(0, N, b):
        idx = order[c0:c0 + b]
        Wv = W.clone().requires_grad_(True)
        loss = 0.5 * ((torch.tensor(k[idx]) @ Wv - torch.tensor(v[idx])) ** 2).sum(dim=1).mean()
        (gW,) = torch.autograd.grad(loss, Wv)
        W = W - eta * gW
        out[idx] = (torch.tensor(q[idx]) @ W).numpy()
    return out


def test_chunked_matches_autograd_recurrence():
    N, d, b = 20, 4, 4
    q, k, v = rnd(1, 1, N, d), rnd(1, 1, N, d), rnd(1, 1, N, d)
    w0 = rnd(1, d, d, scale=0.5)
    eta = 0.9
    fwd = torch_chunked(q[0, 0], k[0, 0], v[0, 0], w0[0], b, eta, reverse=False)
    rev = torch_chunked(q[0, 0], k[0, 0], v[0, 0], w0[0], b, eta, reverse=True)
    o_f = oracle.linear_chunked(q, k, v, w0, chunk=b, eta=eta, direction=1)[0, 0]
    o_r = oracle.linear_chunked(q, k, v, w0, chunk=b, eta=eta, direction=-1)[0, 0]
    o_b = oracle.linear_chunked(q, k, v, w0, chunk=b, eta=eta, direction=0)[0, 0]
    np.testing.assert_allclose(o_f, fwd, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(o_r, rev, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(o_b, fwd + rev, rtol=1e-11, atol=1e-12)


def test_chunked_reversal_symmetry_and_eta_zero():
    """I9: reversing the token order of Q, K, V reverses the bidirectional output.
    I3: eta = 0 gives 2 Q W0.  I10: W0 = 0 makes O linear in V."""
    B, H, N, d, b = 1, 2, 16, 3, 4
    q, k, v = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
    w0 = rnd(H, d, d, scale=0.5)
    o = oracle.linear_chunked(q, k, v, w0, chunk=b, eta=1.0)
    orv = oracle.linear_chunked(q[:, :, ::-1], k[:, :, ::-1], v[:, :, ::-1], w0, chunk=b, eta=1.0)
    np.testing.assert_allclose(orv[:, :, ::-1], o, rtol=1e-12, atol=1e-13)
    o0 = oracle.linear_chunked(q, k, v, w0, chunk=b, eta=0.0)
    for h in range(H):
        np.testing.assert_allclose(o0[0, h], 2 * q[0, h] @ w0[h], rtol=1e-12, atol=1e-13)
    z = np.zeros_like(w0)
    o1 = oracle.linear_chunked(q, k, v, z, chunk=b, eta=1.0)
    o2 = oracle.linear_chunked(q, k, 3.0 * v, z, chunk=b, eta=1.0)
    np.testing.assert_allclose(o2, 3.0 * o1, rtol=1e-12, atol=1e-13)


def test_chunk_output_uses_updated_weights():
    """The chunk output uses W after that chunk's update: with b = 1, d = 1, W0 = 0 the first
    output is q0 * eta * k0 * v0, not 0 (which the before-update reading would give)."""
    q, k, v = (np.array(x, float).reshape(1, 1, 3, 1) for x in ([2, 1, 1], [3, 1, 1], [5, 1, 1]))
    o = oracle.linear_chunked(q, k, v, np.zeros((1, 1, 1)), chunk=1, eta=0.1, direction=1)
    assert o[0, 0, 0, 0] == pytest.approx(2 * 0.1 * 3 * 5, rel=1e-14)
