"""Pins of the oracle's backward, mini-batch / multi-epoch, conv-preprocessing and ViT^3 block
functions (CPU only).  Each is tied to something other than itself: hand-worked fixtures
(tests/golden), finite differences of the pinned forward oracle, torch autograd of a
re-statement built from library matmuls, closed forms of the linear model's affine updates,
special cases, and torch's conv2d."""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from linear_attention_split_b200 import inputs

RNG = np.random.default_rng(1234)


def rnd(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ====================================================================== backward ========
def test_bwd_golden(golden_dir):
    g = load(golden_dir, "linear_bwd_d1_n2.json")
    arr = {x: np.array(g[x], float)[None, None] for x in ("q", "k", "v", "dout")}
    dq, dk, dv, dw0 = oracle.linear_fullbatch_bwd(arr["q"], arr["k"], arr["v"],
                                                  np.array(g["w0"], float)[None], arr["dout"],
                                                  eta=g["eta"])
    np.testing.assert_allclose(dq[0, 0], g["dq"], rtol=1e-13)
    np.testing.assert_allclose(dk[0, 0], g["dk"], rtol=1e-13)
    np.testing.assert_allclose(dv[0, 0], g["dv"], rtol=1e-13)
    np.testing.assert_allclose(dw0[0], g["dw0"], rtol=1e-13)


def outer_loss(q, k, v, w0, dout, eta):
    out, _ = oracle.linear_fullbatch(q, k, v, w0, eta=eta, threads=1)
    return float(np.sum(out * dout))


def test_bwd_finite_differences():
    """Central differences of L = sum dout * O through the forward oracle, every input."""
    B, H, N, d, eta = 2, 2, 5, 3, 0.7
    q, k, v, dout = (rnd(B, H, N, d) for _ in range(4))
    w0 = rnd(H, d, d, scale=0.5)
    dq, dk, dv, dw0 = oracle.linear_fullbatch_bwd(q, k, v, w0, dout, eta=eta)
    eps = 1e-6
    args = {"q": q, "k": k, "v": v, "w0": w0}
    got = {"q": dq, "k": dk, "v": dv, "w0": dw0}
    for name, x in args.items():
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[i] += eps
            xm[i] -= eps
            a = dict(args, **{name: xp})
            b = dict(args, **{name: xm})
            num[i] = (outer_loss(a["q"], a["k"], a["v"], a["w0"], dout, eta) -
                      outer_loss(b["q"], b["k"], b["v"], b["w0"], dout, eta)) / (2 * eps)
        np.testing.assert_allclose(got[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_bwd_autograd_of_restatement():
    """torch autograd through O = Q (W0 - (eta/N) K^T (K W0 - V)), W0 shared per head."""
    B, H, N, d, eta = 3, 2, 17, 4, 1.0
    q, k, v, dout = (rnd(B, H, N, d) for _ in range(4))
    w0 = rnd(H, d, d, scale=0.5)
    tq, tk, tv, tw = (torch.tensor(x, requires_grad=True) for x in (q, k, v, w0))
    ws = tw[None] - (eta / N) * tk.transpose(-1, -2) @ (tk @ tw[None] - tv)
    (tq @ ws * torch.tensor(dout)).sum().backward()
    dq, dk, dv, dw0 = oracle.linear_fullbatch_bwd(q, k, v, w0, dout, eta=eta)
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad), (dw0, tw.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_bwd_eta_zero():
    """eta = 0: O = Q W0, so dQ = dout W0^T, dK = dV = 0, dW0 = sum_b Q_b^T dout_b."""
    B, H, N, d = 3, 2, 9, 5
    q, k, v, dout = (rnd(B, H, N, d) for _ in range(4))
    w0 = rnd(H, d, d)
    dq, dk, dv, dw0 = oracle.linear_fullbatch_bwd(q, k, v, w0, dout, eta=0.0)
    np.testing.assert_allclose(dq, dout @ np.swapaxes(w0, -1, -2)[None], rtol=1e-12, atol=1e-13)
    assert np.all(dk == 0.0) and np.all(dv == 0.0)
    np.testing.assert_allclose(dw0, np.einsum("bhna,bhnc->hac", q, dout), rtol=1e-12, atol=1e-13)


# ====================================================================== mini-batch ======
def test_minibatch_golden(golden_dir):
    g = load(golden_dir, "minibatch_d1_n2.json")
    arr = {x: np.array(g[x], float)[None, None] for x in ("q", "k", "v")}
    out, wf = oracle.linear_minibatch(arr["q"], arr["k"], arr["v"], np.array(g["w0"], float)[None],
                                      g["chunk"], g["epochs"], eta=g["eta"])
    np.testing.assert_allclose(wf[0, 0], g["w_final"], rtol=g["rtol"])
    np.testing.assert_allclose(out[0, 0], g["out"], rtol=g["rtol"])


def test_minibatch_full_batch_one_epoch_is_fullbatch():
    B, H, N, d = 2, 2, 24, 6
    q, k, v = (rnd(B, H, N, d) for _ in range(3))
    w0 = rnd(H, d, d)
    out, wf = oracle.linear_minibatch(q, k, v, w0, chunk=N, epochs=1, eta=0.8)
    ro, rw = oracle.linear_fullbatch(q, k, v, w0, eta=0.8)
    np.testing.assert_allclose(out, ro, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(wf, rw, rtol=1e-12, atol=1e-13)


def test_minibatch_full_batch_epochs_closed_form():
    """Full batch, E epochs: W_E = A^E W0 + (sum_{j<E} A^j)(eta/N) C with A = I - (eta/N) G."""
    N, d, eta, E = 30, 5, 0.9, 4
    q, k, v = rnd(N, d), rnd(N, d), rnd(N, d)
    w0 = rnd(d, d)
    G, C = k.T @ k, k.T @ v
    A = np.eye(d) - (eta / N) * G
    S = sum(np.linalg.matrix_power(A, j) for j in range(E))
    W = np.linalg.matrix_power(A, E) @ w0 + S @ ((eta / N) * C)
    out, wf = oracle.linear_minibatch(q[None, None], k[None, None], v[None, None], w0[None], chunk=N,
                                      epochs=E, eta=eta)
    np.testing.assert_allclose(wf[0, 0], W, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out[0, 0], q @ W, rtol=1e-10, atol=1e-12)


def test_minibatch_chunks_affine_composition():
    """chunk b < N, E = 2: each mini-batch is the affine map W -> (I - (eta/b) K_c^T K_c) W
    + (eta/b) K_c^T V_c, composed in raster order."""
    N, d, b, E, eta = 48, 4, 8, 2, 0.6
    q, k, v = rnd(N, d), rnd(N, d), rnd(N, d)
    w0 = rnd(d, d)
    W = w0.copy()
    for _ in range(E):
        for c0 in range(0, N, b):
            kc, vc = k[c0:c0 + b], v[c0:c0 + b]
            W = (np.eye(d) - (eta / b) * kc.T @ kc) @ W + (eta / b) * kc.T @ vc
    out, wf = oracle.linear_minibatch(q[None, None], k[None, None], v[None, None], w0[None], chunk=b,
                                      epochs=E, eta=eta)
    np.testing.assert_allclose(wf[0, 0], W, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out[0, 0], q @ W, rtol=1e-10, atol=1e-12)


def test_minibatch_eta_zero_and_bad_args():
    q, k, v = (rnd(1, 2, 16, 3) for _ in range(3))
    w0 = rnd(2, 3, 3)
    out, wf = oracle.linear_minibatch(q, k, v, w0, chunk=4, epochs=3, eta=0.0)
    np.testing.assert_allclose(out, q @ w0[None], rtol=1e-13)
    with pytest.raises(ValueError):
        oracle.linear_minibatch(q, k, v, w0, chunk=5, epochs=1)  # 16 % 5 != 0
    with pytest.raises(ValueError):
        oracle.linear_minibatch(q, k, v, w0, chunk=4, epochs=0)


# ====================================================================== conv preprocessing
def test_dwconv_prep_is_library_depthwise_conv():
    B, H, Hg, Wg, d = 2, 3, 5, 7, 4
    x = rnd(B, H, Hg * Wg, d)
    w = rnd(H, d, 3, 3)
    got = oracle.dwconv_prep(x, w, Hg, Wg)
    # torch: channels = H*d, layout [B, C, Hg, Wg]; conv2d is cross-correlation
    xt = torch.tensor(x).reshape(B, H, Hg, Wg, d).permute(0, 1, 4, 2, 3).reshape(B, H * d, Hg, Wg)
    ref = F.conv2d(xt, torch.tensor(w).reshape(H * d, 1, 3, 3), padding=1, groups=H * d)
    ref = ref.reshape(B, H, d, Hg, Wg).permute(0, 1, 3, 4, 2).reshape(B, H, Hg * Wg, d)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_chunked_prep_identity_taps_is_plain_scan():
    B, H, Hg, Wg, d, b = 2, 2, 4, 6, 3, 4
    q, k, v = (rnd(B, H, Hg * Wg, d) for _ in range(3))
    w0 = rnd(H, d, d, scale=0.5)
    ident = np.zeros((H, d, 3, 3))
    ident[:, :, 1, 1] = 1.0
    for direction in (-1, 0, 1):
        got = oracle.linear_chunked_prep(q, k, v, w0, ident, ident, Hg, Wg, b, eta=0.7,
                                         direction=direction)
        ref = oracle.linear_chunked(q, k, v, w0, b, eta=0.7, direction=direction)
        np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-14)


def test_chunked_prep_is_scan_of_convolved_dataset():
    """The layer is the composition: conv of K and V (torch conv2d), then the pinned scan."""
    B, H, Hg, Wg, d, b = 1, 2, 5, 4, 3, 5
    q, k, v = (rnd(B, H, Hg * Wg, d) for _ in range(3))
    w0 = rnd(H, d, d, scale=0.5)
    wk, wv = rnd(H, d, 3, 3, scale=0.4), rnd(H, d, 3, 3, scale=0.4)

    def conv(x, w):
        xt = torch.tensor(x).reshape(B, H, Hg, Wg, d).permute(0, 1, 4, 2, 3).reshape(B, H * d, Hg, Wg)
        y = F.conv2d(xt, torch.tensor(w).reshape(H * d, 1, 3, 3), padding=1, groups=H * d)
        return y.reshape(B, H, d, Hg, Wg).permute(0, 1, 3, 4, 2).reshape(B, H, Hg * Wg, d).numpy()

    got = oracle.linear_chunked_prep(q, k, v, w0, wk, wv, Hg, Wg, b, direction=0)
    ref = oracle.linear_chunked(q, conv(k, wk), conv(v, wv), w0, b, direction=0)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_chunked_unidirectional_sums_to_bidirectional():
    """The scan directions are independent: forward + reverse = the bidirectional layer."""
    q, k, v = (rnd(2, 2, 32, 4) for _ in range(3))
    w0 = rnd(2, 4, 4, scale=0.5)
    f = oracle.linear_chunked(q, k, v, w0, 8, direction=1)
    r = oracle.linear_chunked(q, k, v, w0, 8, direction=-1)
    both = oracle.linear_chunked(q, k, v, w0, 8, direction=0)
    np.testing.assert_allclose(f + r, both, rtol=1e-12, atol=1e-13)


# ====================================================================== the ViT^3 block ==
def torch_block(x, wqkvg, w0, wc, wo, Hg, Wg, H, eta):
    """The block composed from library operators (matmul, conv2d, sigmoid) around the
    pinned TTT-Linear core of the oracle."""
    B, N, C = x.shape
    d = C // H
    xt = torch.tensor(x)
    p = xt @ torch.tensor(wqkvg)
    q, k, v, g = p[..., :C], p[..., C:2 * C], p[..., 2 * C:3 * C], p[..., 3 * C:]
    split = lambda t: t.reshape(B, N, H, d).permute(0, 2, 1, 3).numpy()
    o, _ = oracle.linear_fullbatch(split(q), split(k), split(v), w0, eta=eta)
    o = torch.tensor(o).permute(0, 2, 1, 3).reshape(B, N, C)
    m = o * torch.sigmoid(g)
    xi = xt.reshape(B, Hg, Wg, C).permute(0, 3, 1, 2)
    dc = F.conv2d(xi, torch.tensor(wc).reshape(C, 1, 3, 3), padding=1, groups=C)
    dc = dc.permute(0, 2, 3, 1).reshape(B, N, C)
    return (torch.cat([m, dc], dim=-1) @ torch.tensor(wo)).numpy()


def test_block_is_composition_of_library_operators():
    B, Hg, Wg, C, H = 2, 5, 6, 8, 2
    inp = {k: v.double().numpy() for k, v in inputs.block_inputs(B, Hg, Wg, C, H, dtype="f32", seed=3).items()}
    for eta in (1.0, 0.4):
        got = oracle.vit3_block(inp["x"], inp["wqkvg"], inp["w0"], inp["wc"], inp["wo"], Hg, Wg, H, eta=eta)
        ref = torch_block(inp["x"], inp["wqkvg"], inp["w0"], inp["wc"], inp["wo"], Hg, Wg, H, eta)
        np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_block_special_cases():
    """Zero gate columns give sigmoid(0) = 1/2 exactly; a Wo that keeps only the conv half
    leaves the 3x3 depthwise conv of x (torch conv2d) times that half."""
    B, Hg, Wg, C, H = 1, 4, 4, 4, 1
    x = rnd(B, Hg * Wg, C)
    wqkvg = rnd(C, 4 * C, scale=0.3)
    w0 = rnd(H, C, C, scale=0.5)
    wc = rnd(C, 3, 3)
    wo = np.zeros((2 * C, C))
    wo[C:, :] = np.eye(C)
    y = oracle.vit3_block(x, wqkvg, w0, wc, wo, Hg, Wg, H)
    xi = torch.tensor(x).reshape(B, Hg, Wg, C).permute(0, 3, 1, 2)
    dc = F.conv2d(xi, torch.tensor(wc).reshape(C, 1, 3, 3), padding=1, groups=C)
    np.testing.assert_allclose(y, dc.permute(0, 2, 3, 1).reshape(B, Hg * Wg, C).numpy(), rtol=1e-12, atol=1e-13)
    wq = wqkvg.copy()
    wq[:, 3 * C:] = 0.0
    wo2 = np.zeros((2 * C, C))
    wo2[:C, :] = np.eye(C)
    y2 = oracle.vit3_block(x, wq, w0, wc, wo2, Hg, Wg, H)
    q = x @ wq[:, :C]
    k = x @ wq[:, C:2 * C]
    v = x @ wq[:, 2 * C:3 * C]
    o, _ = oracle.linear_fullbatch(q[:, None], k[:, None], v[:, None], w0)
    np.testing.assert_allclose(y2, 0.5 * o[:, 0], rtol=1e-12, atol=1e-13)
