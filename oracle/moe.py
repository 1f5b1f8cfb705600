"""Oracle for the tensor-parallel mixture-of-experts block (float64, CPU).

Test infrastructure only (see the package docstring).

Source (page title, section): "Tensor-parallel all-reduce count per transformer layer in MLX
shard_linear" (llms-explorer), facts:
* a MoE layer shards its routed experts ("switch_mlp") and its shared expert in place and the
  MoE block makes one all_sum on its output;
* the router stays replicated (Qwen3-MoE);
* sharding the shared expert in place folds its output into the routed experts' sum, so routed
  plus shared experts need one all_sum, not two;
* the sharded-to-all linear adds its bias once, after the sum.

Readings where the pages leave a step open:

* Each expert is a SwiGLU feed-forward block, h = silu(x Wg) * (x Wu), y = h W2 (the block of
  the MLP oracle), with its intermediate width F_e split column-wise into p shards like the
  dense MLP ("shard in place").
* Router: logits = x Wr (Wr of shape (d, E)); each token takes the k experts with the largest
  logits (ties: the lower expert index first) and weights them by the softmax of those k logits
  (softmax over all experts renormalised over the chosen k -- the same numbers).
* The shared expert (optional) sees every token with weight 1; an optional bias is added once
  to the sum.
* Block output: y = sum_{j<k} w_j expert_{e_j}(x) + shared(x) + bias.  Shard i's partial is
  shared_i(x) + sum_j w_j expert_{e_j, i}(x); the block's one reduction adds the p partials.
"""

import numpy as np

from . import mlp


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def route(x, wr, k):
    """Top-k routing.  Returns (idx [T, k] int, weights [T, k]) with idx[t] in descending logit
    order (lower index first among equal logits) and weights[t] = softmax(logits[t, idx[t]])."""
    logits = _f64(x) @ _f64(wr)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("k must be in 1..E")
    idx = np.zeros((T, k), dtype=np.int64)
    w = np.zeros((T, k))
    for t in range(T):
        # stable sort on the negated logits: equal logits keep ascending expert order
        order = np.argsort(-logits[t], kind="stable")[:k]
        idx[t] = order
        sel = logits[t, order]
        e = np.exp(sel - sel.max())
        w[t] = e / e.sum()
    return idx, w


def weights_for(x, wr, idx):
    """The routing weights that go with a given choice of experts: for each token, the softmax of
    its logits at the chosen experts ``idx[t]`` (in the order given).  With idx from route() this
    equals route()'s weights; for another valid top-k set (a near tie broken the other way) it
    gives that set's weights from the exact logits."""
    logits = _f64(x) @ _f64(wr)
    idx = np.asarray(idx, dtype=np.int64)
    w = np.zeros(idx.shape)
    for t in range(idx.shape[0]):
        sel = logits[t, idx[t]]
        e = np.exp(sel - sel.max())
        w[t] = e / e.sum()
    return w


def topk_margin(x, wr, idx):
    """For each token, the smallest chosen logit minus the largest unchosen one (exact logits).

    ``idx[t]`` is a true top-k set exactly when the margin is >= 0.  A router that computes its
    logits with an error of at most eps per logit picks a set whose exact margin is >= -2 eps, so
    a caller checks a rounded router's choice against that bound.  With k = E every logit is
    chosen and the margin is +inf."""
    logits = _f64(x) @ _f64(wr)
    idx = np.asarray(idx, dtype=np.int64)
    T, E = logits.shape
    out = np.full(T, np.inf)
    for t in range(T):
        chosen = np.zeros(E, dtype=bool)
        chosen[idx[t]] = True
        if chosen.sum() != idx.shape[1]:
            out[t] = -np.inf          # an expert chosen twice is never a valid top-k set
            continue
        if chosen.all():
            continue
        out[t] = logits[t, chosen].min() - logits[t, ~chosen].max()
    return out


def moe_forward(x, wr, experts, k, shared=None, bias=None, routing=None):
    """Unsharded MoE block.  experts: list of (wg, wu, w2) per expert; shared: (wg, wu, w2) or
    None; routing: (idx, weights) to use instead of route(x, wr, k)."""
    x = _f64(x)
    idx, w = routing if routing is not None else route(x, wr, k)
    y = np.zeros((x.shape[0], x.shape[1]))
    for t in range(x.shape[0]):
        for j in range(idx.shape[1]):
            wg, wu, w2 = experts[int(idx[t, j])]
            y[t] += w[t, j] * mlp.mlp_forward(x[t:t + 1], wg, w2, "swiglu", wu)[0]
    if shared is not None:
        wg, wu, w2 = shared
        y = y + mlp.mlp_forward(x, wg, w2, "swiglu", wu)
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return y


def moe_forward_sharded(x, wr, experts, k, p, shared=None, bias=None, routing=None):
    """Sharded reference mode (invariant tests only).  Shard i runs every expert (and the shared
    expert) on its column slice of Wg/Wu and row slice of W2.  Returns (y, partials): partials[i]
    is shard i's output and y = sum of the partials in order i = 0..p-1, plus the bias once."""
    x = _f64(x)
    idx, w = routing if routing is not None else route(x, wr, k)
    T, d = x.shape
    partials = []
    for i in range(p):
        part = np.zeros((T, d))
        for t in range(T):
            for j in range(idx.shape[1]):
                wg, wu, w2 = experts[int(idx[t, j])]
                f = _f64(wg).shape[1]
                if f % p:
                    raise ValueError("p must divide every expert's width")
                c = slice(i * f // p, (i + 1) * f // p)
                part[t] += w[t, j] * mlp.mlp_forward(x[t:t + 1], _f64(wg)[:, c], _f64(w2)[c, :],
                                                     "swiglu", _f64(wu)[:, c])[0]
        if shared is not None:
            wg, wu, w2 = shared
            f = _f64(wg).shape[1]
            if f % p:
                raise ValueError("p must divide the shared expert's width")
            c = slice(i * f // p, (i + 1) * f // p)
            part += mlp.mlp_forward(x, _f64(wg)[:, c], _f64(w2)[c, :], "swiglu", _f64(wu)[:, c])
        partials.append(part)
    y = np.zeros((T, d))
    for part in partials:
        y = y + part
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return y, partials


def moe_backward(x, wr, experts, k, dy, shared=None, routing=None):
    """Gradients of moe_forward's output y against an upstream gradient dy, with the choice of
    experts held fixed (the top-k selection is constant wherever the k-th and (k+1)-th logits
    differ, so it carries no gradient there).  The residual and the bias pass dy through and are
    not part of the result.

    Chain rule, with l_t = x_t Wr, the chosen experts e_tj = idx[t, j], the routed outputs
    o_tj = expert_{e_tj}(x_t) and the weights w_t = softmax(l_t[idx_t]):
      y_t = sum_j w_tj o_tj + shared(x_t)
      d o_tj = w_tj dy_t           -> expert e_tj's MLP backward on row t
      dw_tj = <dy_t, o_tj>
      dl_t[e_tj] = w_tj (dw_tj - sum_i w_ti dw_ti), 0 at the experts not chosen
      dWr = x^T dl,  dx += dl Wr^T
      the shared expert: its MLP backward with dy.
    ``routing``: (idx, weights) as moe_forward takes them; else route(x, wr, k).
    Returns a dict: dx (T, d), dwr (d, E), experts (per expert a dict dwg, dwu, dw2; zeros for
    an expert no token chose) and shared (dwg, dwu, dw2, or None)."""
    x, wr, dy = _f64(x), _f64(wr), _f64(dy)
    idx, w = routing if routing is not None else route(x, wr, k)
    idx = np.asarray(idx, dtype=np.int64)
    w = _f64(w)
    T, d = x.shape
    E = wr.shape[1]
    dx = np.zeros((T, d))
    grads = [{"dwg": np.zeros_like(_f64(ex[0])), "dwu": np.zeros_like(_f64(ex[1])),
              "dw2": np.zeros_like(_f64(ex[2]))} for ex in experts]
    dl = np.zeros((T, E))
    for t in range(T):
        dwt = np.zeros(idx.shape[1])
        for j in range(idx.shape[1]):
            wg, wu, w2 = experts[int(idx[t, j])]
            xt = x[t:t + 1]
            o = mlp.mlp_forward(xt, wg, w2, "swiglu", wu)[0]
            dwt[j] = dy[t] @ o
            b = mlp.mlp_backward(xt, wg, w2, w[t, j] * dy[t:t + 1], "swiglu", wu)
            g = grads[int(idx[t, j])]
            g["dwg"] += b["dw1"]
            g["dwu"] += b["dw_up"]
            g["dw2"] += b["dw2"]
            dx[t] += b["dx"][0]
        s = w[t] @ dwt
        for j in range(idx.shape[1]):
            dl[t, int(idx[t, j])] = w[t, j] * (dwt[j] - s)
    dwr = x.T @ dl
    dx += dl @ wr.T
    out = {"dx": dx, "dwr": dwr, "experts": grads, "shared": None}
    if shared is not None:
        wg, wu, w2 = shared
        b = mlp.mlp_backward(x, wg, w2, dy, "swiglu", wu)
        out["dx"] = out["dx"] + b["dx"]
        out["shared"] = {"dwg": b["dw1"], "dwu": b["dw_up"], "dw2": b["dw2"]}
    return out
