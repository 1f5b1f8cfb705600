"""Pins for the MLP oracle: facts the pages and the mathematics fix, independent of the oracle.

Each test names the passage it follows.  None of these re-types the oracle's own formula: they
use printed values, closed forms, library routines with a different formulation, brute-force
loops with exact summation, finite differences, and the sharding invariants the pages state.
"""

import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit
from scipy.stats import norm

from oracle import mlp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = (s.strip() for s in line.split("=", 1))
            vals[k] = [float(t) for t in v.split()]
    return vals


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _rng_case(T, d, F, seed=0):
    r = np.random.default_rng(seed)
    return (r.standard_normal((T, d)), r.standard_normal((d, F)) / math.sqrt(d),
            r.standard_normal((d, F)) / math.sqrt(d), r.standard_normal((F, d)) / math.sqrt(F),
            r.standard_normal((T, d)))


# --- worked example: "Why tensor parallelism has to stay in scale-up", "What is Tensor Parallel"

def test_worked_example_values():
    g = _read_golden("worked_example_h2_dff3.txt")
    x = np.array([g["x"]])
    A = np.array([g["A_row0"], g["A_row1"]])
    B = np.array([g["B_row0"], g["B_row1"], g["B_row2"]])
    assert np.array_equal(mlp.hidden(x, A, "identity"), np.array([g["y"]]))
    assert np.array_equal(mlp.mlp_forward(x, A, B, "identity"), np.array([g["z"]]))


def test_worked_example_tp3_one_reduction():
    g = _read_golden("worked_example_h2_dff3.txt")
    x = np.array([g["x"]])
    A = np.array([g["A_row0"], g["A_row1"]])
    B = np.array([g["B_row0"], g["B_row1"], g["B_row2"]])
    tp = int(g["tp"][0])
    y, partials = mlp.mlp_forward_sharded(x, A, B, "identity", tp)
    assert len(partials) == 3
    # each GPU owns one column of A and one row of B: its partial is y_j * B[j]
    for j in range(3):
        assert np.array_equal(partials[j], g["y"][j] * B[j][None, :])
    assert np.array_equal(y, np.array([g["z"]]))


# --- activations: closed forms and library routines with another formulation

def test_gelu_closed_forms():
    assert mlp.gelu(0.0) == 0.0
    # GELU(1) = Phi(1) = 0.841344746068542948585232545632...
    assert abs(mlp.gelu(1.0) - 0.8413447460685429) < 1e-15
    z = np.linspace(-8, 8, 1001)
    np.testing.assert_allclose(mlp.gelu(z), z * norm.cdf(z), rtol=1e-13, atol=1e-15)
    # odd-part identity: GELU(z) - GELU(-z) = z
    np.testing.assert_allclose(mlp.gelu(z) - mlp.gelu(-z), z, atol=1e-13)


def test_silu_closed_forms():
    assert mlp.silu(0.0) == 0.0
    assert abs(mlp.silu(1.0) - 0.7310585786300049) < 1e-15  # 1 / (1 + e^-1)
    z = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(mlp.silu(z), z * expit(z), rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(mlp.silu(z) - mlp.silu(-z), z, atol=1e-12)


def test_relu_and_identity():
    z = np.array([-2.0, -0.0, 0.0, 3.5])
    assert np.array_equal(mlp.act(z, "relu"), np.array([0.0, 0.0, 0.0, 3.5]))
    assert np.array_equal(mlp.act(z, "identity"), z)


@pytest.mark.parametrize("kind", ["gelu", "relu", "identity"])
def test_act_grad_finite_difference(kind):
    z = np.linspace(-4, 4, 81) + 0.013  # avoid the ReLU kink at 0
    e = 1e-6
    fd = (mlp.act(z + e, kind) - mlp.act(z - e, kind)) / (2 * e)
    np.testing.assert_allclose(mlp.act_grad(z, kind), fd, rtol=1e-7, atol=1e-8)


def test_silu_grad_finite_difference():
    z = np.linspace(-6, 6, 121)
    e = 1e-6
    fd = (mlp.silu(z + e) - mlp.silu(z - e)) / (2 * e)
    np.testing.assert_allclose(mlp.silu_grad(z), fd, rtol=1e-7, atol=1e-9)


# --- brute force on tiny inputs (exact summation, scalar math library)

def _brute_forward(x, w1, w2, kind, wu=None):
    T, d = x.shape
    F = w1.shape[1]
    y = np.zeros((T, w2.shape[1]))
    for t in range(T):
        h = []
        for f in range(F):
            z = math.fsum(x[t, k] * w1[k, f] for k in range(d))
            if kind == "swiglu":
                u = math.fsum(x[t, k] * wu[k, f] for k in range(d))
                h.append(z / (1.0 + math.exp(-z)) * u)
            elif kind == "gelu":
                h.append(0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0))))
            elif kind == "relu":
                h.append(z if z > 0 else 0.0)
            else:
                h.append(z)
        for n in range(w2.shape[1]):
            y[t, n] = math.fsum(h[f] * w2[f, n] for f in range(F))
    return y


@pytest.mark.parametrize("kind", mlp.ACTS)
def test_forward_brute_force(kind):
    x, w1, wu, w2, _ = _rng_case(3, 5, 12, seed=1)
    wu = wu if kind == "swiglu" else None
    got = mlp.mlp_forward(x, w1, w2, kind, wu)
    ref = _brute_forward(x, w1, w2, kind, wu)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_forward_is_not_transposed():
    # rectangular shapes catch a transposed operand: x (2,3), W1 (3,5), W2 (5,3)
    x = np.arange(6.0).reshape(2, 3)
    w1 = np.arange(15.0).reshape(3, 5) - 7.0  # integers: every product and sum is exact
    w2 = np.arange(15.0).reshape(5, 3) - 4.0
    ref = _brute_forward(x, w1, w2, "identity")
    assert np.array_equal(mlp.mlp_forward(x, w1, w2, "identity"), ref)


# --- closed form: the linear special case

def test_identity_activation_is_one_matrix():
    x, w1, _, w2, _ = _rng_case(6, 8, 32, seed=2)
    np.testing.assert_allclose(mlp.mlp_forward(x, w1, w2, "identity"), x @ (w1 @ w2),
                               rtol=1e-12, atol=1e-13)


# --- sharding invariants ("Second matmul, row-parallel": the true y is the sum of the y_i)

@pytest.mark.parametrize("kind", mlp.ACTS)
def test_sharded_sum_equals_unsharded_every_p(kind):
    # the tiny configuration: T=4, d=8, d_ff=32
    x, w1, wu, w2, _ = _rng_case(4, 8, 32, seed=3)
    wu = wu if kind == "swiglu" else None
    ref = mlp.mlp_forward(x, w1, w2, kind, wu)
    for p in (1, 2, 4, 8, 16, 32):
        y, parts = mlp.mlp_forward_sharded(x, w1, w2, kind, p, wu)
        assert len(parts) == p and all(pt.shape == ref.shape for pt in parts)
        assert _rel(y, ref) <= 1e-13, p


def test_non_power_of_two_shards():
    # "What is Tensor Parallel" uses TP=3
    x, w1, wu, w2, _ = _rng_case(5, 6, 24, seed=4)
    ref = mlp.mlp_forward(x, w1, w2, "swiglu", wu)
    for p in (3, 6, 12, 24):
        y, _ = mlp.mlp_forward_sharded(x, w1, w2, "swiglu", p, wu)
        assert _rel(y, ref) <= 1e-13


def test_sharded_rejects_p_not_dividing():
    x, w1, _, w2, _ = _rng_case(2, 4, 10, seed=5)
    with pytest.raises(ValueError):
        mlp.mlp_forward_sharded(x, w1, w2, "gelu", 3)


def test_activation_commutes_with_column_split():
    # "The nonlinearity is free": act(x W1)[:, shard i] is act(x W1_i)
    x, w1, wu, _, _ = _rng_case(4, 8, 32, seed=6)
    for kind in mlp.ACTS:
        full = mlp.hidden(x, w1, kind, wu if kind == "swiglu" else None)
        for i in range(4):
            c = slice(8 * i, 8 * i + 8)
            part = mlp.hidden(x, w1[:, c], kind, wu[:, c] if kind == "swiglu" else None)
            np.testing.assert_allclose(part, full[:, c], rtol=1e-14, atol=1e-15)


def test_activation_does_not_commute_with_row_split():
    # "Had you split the first matmul by rows instead ... reduce them before the nonlinearity"
    x, w1, _, _, _ = _rng_case(4, 8, 32, seed=7)
    p = 4
    rows = [slice(2 * i, 2 * i + 2) for i in range(p)]
    full = mlp.act(x @ w1, "gelu")
    wrong = sum(mlp.act(x[:, r] @ w1[r, :], "gelu") for r in rows)
    assert _rel(wrong, full) > 1e-2
    # ... unless the activation is the identity (a linear map commutes with the sum)
    lin = sum(x[:, r] @ w1[r, :] for r in rows)
    np.testing.assert_allclose(lin, x @ w1, rtol=1e-13, atol=1e-13)


def test_mismatched_pairing_is_wrong():
    # "Common failure": the row slice of W2 must be exactly the one that pairs with the columns
    x, w1, wu, w2, _ = _rng_case(4, 8, 32, seed=8)
    ref = mlp.mlp_forward(x, w1, w2, "gelu")
    p, fs = 4, 8
    wrong = sum(mlp.act(x @ w1[:, fs * i:fs * i + fs], "gelu") @ w2[fs * ((i + 1) % p):fs * ((i + 1) % p) + fs]
                for i in range(p))
    assert _rel(wrong, ref) > 0.1
    # SwiGLU: gate slice i with up slice i+1 is wrong too
    ref = mlp.mlp_forward(x, w1, w2, "swiglu", wu)
    wrong = sum((mlp.silu(x @ w1[:, fs * i:fs * i + fs]) * (x @ wu[:, fs * ((i + 1) % p):fs * ((i + 1) % p) + fs]))
                @ w2[fs * i:fs * i + fs] for i in range(p))
    assert _rel(wrong, ref) > 0.1


# --- backward: central finite differences on the forward, and the sharding invariants

def _fd_grad(f, a, e=1e-6):
    g = np.zeros_like(a)
    it = np.nditer(a, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = a[i]
        a[i] = old + e
        fp = f()
        a[i] = old - e
        fm = f()
        a[i] = old
        g[i] = (fp - fm) / (2 * e)
    return g


@pytest.mark.parametrize("kind", mlp.ACTS)
def test_backward_finite_differences(kind):
    # tiny shape T=3, d=4, F=8
    x, w1, wu, w2, dy = _rng_case(3, 4, 8, seed=9)
    wu = wu if kind == "swiglu" else None
    if kind == "relu":
        x = x + 0.0  # keep the kink away: checked below
        assert np.min(np.abs(x @ w1)) > 1e-4
    loss = lambda: float(np.sum(mlp.mlp_forward(x, w1, w2, kind, wu) * dy))
    g = mlp.mlp_backward(x, w1, w2, dy, kind, wu)
    assert _rel(g["dx"], _fd_grad(loss, x)) <= 1e-6
    assert _rel(g["dw1"], _fd_grad(loss, w1)) <= 1e-6
    assert _rel(g["dw2"], _fd_grad(loss, w2)) <= 1e-6
    if kind == "swiglu":
        assert _rel(g["dw_up"], _fd_grad(loss, wu)) <= 1e-6


def test_backward_matches_torch_autograd():
    # a library routine (reverse-mode AD) on the unsharded SwiGLU block
    x, w1, wu, w2, dy = _rng_case(5, 6, 16, seed=10)
    tx, t1, tu, t2 = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (x, w1, wu, w2))
    y = (torch.nn.functional.silu(tx @ t1) * (tx @ tu)) @ t2
    y.backward(torch.tensor(dy, dtype=torch.float64))
    g = mlp.mlp_backward(x, w1, w2, dy, "swiglu", wu)
    for mine, ref in ((g["dx"], tx.grad), (g["dw1"], t1.grad), (g["dw_up"], tu.grad), (g["dw2"], t2.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", mlp.ACTS)
def test_backward_sharded_invariants(kind):
    # "The backward pass": dx is the sum of per-shard partials; weight gradients need no exchange
    x, w1, wu, w2, dy = _rng_case(3, 4, 8, seed=11)
    wu = wu if kind == "swiglu" else None
    full = mlp.mlp_backward(x, w1, w2, dy, kind, wu)
    p, fs = 2, 4
    dx, shards = mlp.mlp_backward_sharded(x, w1, w2, dy, kind, p, wu)
    assert _rel(dx, full["dx"]) <= 1e-13
    for i, g in enumerate(shards):
        c = slice(fs * i, fs * i + fs)
        np.testing.assert_allclose(g["dw1"], full["dw1"][:, c], rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(g["dw2"], full["dw2"][c, :], rtol=1e-14, atol=1e-15)
        if kind == "swiglu":
            np.testing.assert_allclose(g["dw_up"], full["dw_up"][:, c], rtol=1e-14, atol=1e-15)
        # a single shard's dx is only a partial: it differs from the full dx
        assert _rel(g["dx"], full["dx"]) > 1e-3


def test_samples_match_full_results():
    x, w1, wu, w2, dy = _rng_case(7, 8, 16, seed=12)
    rows, cols, w2r = [0, 3, 6], [1, 5, 15], [0, 9]
    for kind in mlp.ACTS:
        w = wu if kind == "swiglu" else None
        full = mlp.mlp_backward(x, w1, w2, dy, kind, w)
        s = mlp.mlp_backward_samples(x, w1, w2, dy, kind, rows, cols, w2r, w)
        np.testing.assert_allclose(s["dx"], full["dx"][rows], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(s["dw1_cols"], full["dw1"][:, cols], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(s["dw2_rows"], full["dw2"][w2r], rtol=1e-13, atol=1e-14)
        if kind == "swiglu":
            np.testing.assert_allclose(s["dw_up_cols"], full["dw_up"][:, cols], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(mlp.mlp_forward_rows(x, w1, w2, kind, rows, w),
                                   mlp.mlp_forward(x, w1, w2, kind, w)[rows], rtol=1e-13, atol=1e-14)
