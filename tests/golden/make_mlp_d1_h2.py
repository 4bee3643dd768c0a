"""Writes tests/golden/mlp_d1_h2.json: a TTT-MLP full-batch step worked out by hand.

This is the calculator program behind that fixture.  It uses Python's `math` module only and
imports nothing from the oracle or the library, so the fixture pins the oracle from outside.

Source of the operation: TTT-MLP (hidden state a two-layer MLP) in the TTT abstract of Sun et
al. on the scholarfeed author page of Jiarui Xu; the full-batch step W* = W0 - eta grad l(W0)
with l(W) = (1/N) sum_i 1/2 ||F_W(k_i) - v_i||^2 (ViT^3 blog, online-learning rewrite of
attention, steps 1-3); F(x) = gelu_tanh(x W1) W2 without biases, gelu in its published tanh
form (Hendrycks & Gimpel).  The chain rule is written out below for d = 1, hidden = 2, N = 2.

Usage: ``python tests/golden/make_mlp_d1_h2.py`` (rewrites the file; ``--check`` only
compares and exits non-zero on any difference).
"""
import json
import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PATH = os.path.join(HERE, "mlp_d1_h2.json")

S = math.sqrt(2.0 / math.pi)
A = 0.044715


def gelu(u):
    return 0.5 * u * (1.0 + math.tanh(S * (u + A * u ** 3)))


def dgelu(u):
    t = math.tanh(S * (u + A * u ** 3))
    return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * S * (1.0 + 3.0 * A * u * u)


def compute(q, k, v, w1, w2, eta):
    """d = 1: q, k, v are lists of [x]; w1 = [[a, b]] (1 x 2); w2 = [[c], [e]] (2 x 1)."""
    N = len(k)
    h = len(w1[0])
    loss = 0.0
    g1 = [0.0] * h
    g2 = [0.0] * h
    for (kx,), (vx,) in zip(k, v):
        z = [kx * w1[0][j] for j in range(h)]
        a = [gelu(zj) for zj in z]
        p = sum(a[j] * w2[j][0] for j in range(h))
        r = p - vx
        loss += 0.5 * r * r / N
        for j in range(h):
            g2[j] += a[j] * r / N                        # dl/dW2[j] = a_j r
            g1[j] += kx * (r * w2[j][0]) * dgelu(z[j]) / N  # dl/dW1[j] = k (r W2[j]) gelu'(z_j)
    w1s = [w1[0][j] - eta * g1[j] for j in range(h)]
    w2s = [w2[j][0] - eta * g2[j] for j in range(h)]
    out = [[sum(gelu(qx * w1s[j]) * w2s[j] for j in range(h))] for (qx,) in q]
    return {"loss_w0": loss, "grad_w1": [g1], "grad_w2": [[x] for x in g2],
            "w1_star": [w1s], "w2_star": [[x] for x in w2s], "out": out}


def main():
    with open(PATH) as fh:
        fix = json.load(fh)
    got = compute(fix["q"], fix["k"], fix["v"], fix["w1"], fix["w2"], fix["eta"])
    if "--check" in sys.argv:
        bad = [key for key, val in got.items() if fix.get(key) != val]
        print("identical" if not bad else f"differs in {bad}")
        sys.exit(1 if bad else 0)
    fix.update(got)
    fix["citation"] = fix["citation"].replace(
        "evaluated with a pocket-calculator program (Python math module), independent of the oracle",
        "evaluated by tests/golden/make_mlp_d1_h2.py (Python math module only), independent of the oracle")
    with open(PATH, "w") as fh:
        json.dump(fix, fh, indent=2)
        fh.write("\n")


if __name__ == "__main__":
    main()
