"""Oracle for the position-wise feed-forward block, forward and backward (float64, CPU).

Test infrastructure only (see the package docstring).

Sources (page title, section):

* "How does tensor parallelism split a transformer feed-forward block's two matmuls across
  devices?" -- "The shape of the block": h = act(x W1), y = h W2, x of shape (T, d), W1 of shape
  (d, F), W2 of shape (F, d).  "The nonlinearity is free": the activation is elementwise (GELU,
  ReLU, or a gated variant computed from the same slice).  "Second matmul, row-parallel": the
  true y equals the sum over shards of y_i = h_i W2_i.  "The backward pass": the weight gradient
  of each shard is that shard's slice of the full weight gradient; the input gradient is the sum
  of the per-shard partial input gradients.
* "Tensor Parallelism" (klaylearn), Notes: Y = XW, column split W = [W_1..W_p] along the output
  dimension, row split along the input dimension with X split to match, Y = sum_i Z_i; "shard the
  up/gate projections column-wise".

Readings where the pages leave a step open:

* GELU is the exact form 0.5 z (1 + erf(z / sqrt 2)).
* The gated variant is SwiGLU: h = silu(x Wg) * (x Wu), silu(z) = z * sigmoid(z); gate and up
  share the same column slice in every shard.
* Weights are stored input-major, W[in, out], so that Y = X W as the pages write it.

``act`` names: "identity", "relu", "gelu", "swiglu".  For "swiglu" ``w1`` is the gate matrix Wg
and ``w_up`` the up matrix Wu; for the other activations ``w_up`` is None.
"""

import numpy as np
from scipy.special import erf

ACTS = ("identity", "relu", "gelu", "swiglu")


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def sigmoid(z):
    z = _f64(z)
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    """silu(z) = z * sigmoid(z)."""
    z = _f64(z)
    return z * sigmoid(z)


def silu_grad(z):
    """d/dz silu(z) = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    z = _f64(z)
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def gelu(z):
    """Exact GELU, 0.5 z (1 + erf(z / sqrt(2)))."""
    z = _f64(z)
    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def gelu_grad(z):
    """d/dz GELU(z) = Phi(z) + z phi(z)."""
    z = _f64(z)
    cdf = 0.5 * (1.0 + erf(z / np.sqrt(2.0)))
    pdf = np.exp(-0.5 * z * z) / np.sqrt(2.0 * np.pi)
    return cdf + z * pdf


def act(z, kind):
    """The elementwise nonlinearity of the single-matrix forms."""
    z = _f64(z)
    if kind == "identity":
        return z
    if kind == "relu":
        return np.maximum(z, 0.0)
    if kind == "gelu":
        return gelu(z)
    raise ValueError(f"unknown activation {kind!r}")


def act_grad(z, kind):
    z = _f64(z)
    if kind == "identity":
        return np.ones_like(z)
    if kind == "relu":
        return (z > 0.0).astype(np.float64)
    if kind == "gelu":
        return gelu_grad(z)
    raise ValueError(f"unknown activation {kind!r}")


def hidden(x, w1, kind, w_up=None):
    """The widened activation h (T, F): act(x W1), or silu(x Wg) * (x Wu) for SwiGLU."""
    x, w1 = _f64(x), _f64(w1)
    if kind == "swiglu":
        return silu(x @ w1) * (x @ _f64(w_up))
    return act(x @ w1, kind)


def mlp_forward(x, w1, w2, kind, w_up=None):
    """Unsharded block: y = h W2 with h = hidden(x, ...).  Shapes: x (T,d) -> y (T,d)."""
    return hidden(x, w1, kind, w_up) @ _f64(w2)


def mlp_forward_sharded(x, w1, w2, kind, p, w_up=None):
    """Sharded reference mode (for invariant tests only).

    Shard i owns columns [i F/p, (i+1) F/p) of W1 (and of Wu) and the matching rows of W2
    (column-parallel then row-parallel).  Returns (y, partials) where partials[i] = h_i W2_i and
    y is their sum taken in the fixed order i = 0 .. p-1.
    """
    x, w1, w2 = _f64(x), _f64(w1), _f64(w2)
    F = w1.shape[1]
    if p < 1 or F % p:
        raise ValueError("p must divide d_ff")
    fs = F // p
    partials = []
    for i in range(p):
        cols = slice(i * fs, (i + 1) * fs)
        wu_i = None if w_up is None else _f64(w_up)[:, cols]
        h_i = hidden(x, w1[:, cols], kind, wu_i)
        partials.append(h_i @ w2[cols, :])
    y = np.zeros_like(partials[0])
    for part in partials:
        y = y + part
    return y, partials


def mlp_backward(x, w1, w2, dy, kind, w_up=None):
    """Chain rule through the unsharded block.

    Returns a dict with dx (T,d), dw1 (d,F), dw2 (F,d) and, for SwiGLU, dw_up (d,F).
    With z = x W1 (gate pre-activation for SwiGLU) and u = x Wu:
      dh  = dy W2^T
      dw2 = h^T dy
      non-gated: dz = dh * act'(z);                dx = dz W1^T
      SwiGLU:    dz = dh * u * silu'(z), du = dh * silu(z);  dx = dz Wg^T + du Wu^T
      dw1 = x^T dz,  dw_up = x^T du
    """
    x, w1, w2, dy = _f64(x), _f64(w1), _f64(w2), _f64(dy)
    z = x @ w1
    dh = dy @ w2.T
    out = {}
    if kind == "swiglu":
        wu = _f64(w_up)
        u = x @ wu
        s = silu(z)
        h = s * u
        dz = dh * u * silu_grad(z)
        du = dh * s
        out["dw_up"] = x.T @ du
        out["dx"] = dz @ w1.T + du @ wu.T
    else:
        h = act(z, kind)
        dz = dh * act_grad(z, kind)
        out["dx"] = dz @ w1.T
    out["dw1"] = x.T @ dz
    out["dw2"] = h.T @ dy
    return out


def mlp_backward_sharded(x, w1, w2, dy, kind, p, w_up=None):
    """Sharded reference mode of the backward pass (invariant tests only).

    Each shard runs the chain rule on its own column slice of W1/Wu and row slice of W2 with the
    replicated dy (the exit's backward is the identity).  Returns per-shard weight gradients (no
    exchange) and the input gradient as the in-order sum of the per-shard partial dx_i (the
    entry's backward is the all-reduce).
    """
    x, w1, w2, dy = _f64(x), _f64(w1), _f64(w2), _f64(dy)
    F = w1.shape[1]
    if p < 1 or F % p:
        raise ValueError("p must divide d_ff")
    fs = F // p
    shards = []
    for i in range(p):
        cols = slice(i * fs, (i + 1) * fs)
        wu_i = None if w_up is None else _f64(w_up)[:, cols]
        shards.append(mlp_backward(x, w1[:, cols], w2[cols, :], dy, kind, wu_i))
    dx = np.zeros_like(shards[0]["dx"])
    for g in shards:
        dx = dx + g["dx"]
    return dx, shards


def mlp_forward_rows(x, w1, w2, kind, rows, w_up=None):
    """Rows ``rows`` of the unsharded y: each output row depends only on the same input row."""
    return mlp_forward(_f64(x)[rows], w1, w2, kind, w_up)


def mlp_backward_samples(x, w1, w2, dy, kind, dx_rows, feat_cols, w2_rows, w_up=None):
    """Selected entries of the unsharded backward, each computed over its full contraction.

    * dx[dx_rows, :]            (every column of the chosen rows)
    * dw1[:, feat_cols] (and dw_up[:, feat_cols])  (whole columns = chosen hidden features)
    * dw2[w2_rows, :]           (whole rows = chosen hidden features)

    Used to check full-size results where the whole oracle would take too long.
    """
    x, w1, w2, dy = _f64(x), _f64(w1), _f64(w2), _f64(dy)
    out = {}
    # dx rows: needs the full hidden width for those tokens only.
    xr, dyr = x[dx_rows], dy[dx_rows]
    z = xr @ w1
    dh = dyr @ w2.T
    if kind == "swiglu":
        wu = _f64(w_up)
        u = xr @ wu
        dz = dh * u * silu_grad(z)
        du = dh * silu(z)
        out["dx"] = dz @ w1.T + du @ wu.T
    else:
        out["dx"] = (dh * act_grad(z, kind)) @ w1.T
    # dw1 / dw_up columns: needs every token but only the chosen hidden features.
    zc = x @ w1[:, feat_cols]
    dhc = dy @ w2[feat_cols, :].T
    if kind == "swiglu":
        wu = _f64(w_up)
        uc = x @ wu[:, feat_cols]
        out["dw1_cols"] = x.T @ (dhc * uc * silu_grad(zc))
        out["dw_up_cols"] = x.T @ (dhc * silu(zc))
    else:
        out["dw1_cols"] = x.T @ (dhc * act_grad(zc, kind))
    # dw2 rows: h restricted to the chosen features, over every token.
    zr = x @ w1[:, w2_rows]
    if kind == "swiglu":
        hr = silu(zr) * (x @ _f64(w_up)[:, w2_rows])
    else:
        hr = act(zr, kind)
    out["dw2_rows"] = hr.T @ dy
    return out
