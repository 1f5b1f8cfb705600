"""Oracle for the grouped-query attention block (float64, CPU).

Test infrastructure only (see the package docstring).

Sources (page title, section):

* "Tensor Parallelism" (klaylearn), Notes, the grouped-query attention paragraph: hidden size
  8192, 64 query heads, 8 KV heads, head dim 128; with p = 8 each rank owns 8 Q heads and 1 KV
  head (local Wq 8192x1024, Wk and Wv 8192x128), attention runs locally over the local heads, and
  the output projection turns the local 1024-wide result into a partial 8192-wide update that is
  summed across ranks.
* "How does tensor parallelism split a transformer feed-forward block's two matmuls", closing
  paragraph of "What it costs": Q/K/V column-parallel so each device owns whole heads, output
  projection row-parallel, one reduction; heads are never split.

Readings where the pages leave a step open:

* Plain scaled-dot-product attention with scale 1/sqrt(head_dim); no RoPE, no QK norm, no bias.
* Query head j reads KV head floor(j / (n_q / n_kv)) -- contiguous head groups, which is what
  "rank i owns 8 Q heads and 1 KV head" gives when heads are numbered in column order.
* Causal: a query at position t sees keys at positions <= t (diagonal included).
* Weights are input-major: Wq (h, n_q*hd), Wk and Wv (h, n_kv*hd), Wo (n_q*hd, h).
"""

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def softmax_rows(s):
    """Row-wise softmax; -inf entries get weight 0.  The row maximum is subtracted first."""
    s = _f64(s)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def kv_head_of(j, n_q, n_kv):
    return j // (n_q // n_kv)


def attend(q, k, v, causal, q_pos0=0):
    """Single-head attention.  q (Sq, hd), k and v (Sk, hd).

    Query row r sits at absolute position q_pos0 + r; key c at position c.  With ``causal`` a
    query sees keys at positions <= its own.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    hd = q.shape[-1]
    s = (q @ k.T) / np.sqrt(hd)
    if causal:
        qpos = q_pos0 + np.arange(q.shape[0])[:, None]
        kpos = np.arange(k.shape[0])[None, :]
        s = np.where(kpos <= qpos, s, -np.inf)
    return softmax_rows(s) @ v


def project_qkv(x, wq, wk, wv, n_q, n_kv, head_dim):
    """x (S, h) -> q (S, n_q, hd), k and v (S, n_kv, hd)."""
    x = _f64(x)
    S = x.shape[0]
    q = (x @ _f64(wq)).reshape(S, n_q, head_dim)
    k = (x @ _f64(wk)).reshape(S, n_kv, head_dim)
    v = (x @ _f64(wv)).reshape(S, n_kv, head_dim)
    return q, k, v


def attention_heads(q, k, v, n_q, n_kv, causal, q_pos0=0):
    """All query heads: o (Sq, n_q*hd), each head attending over its KV head."""
    Sq, _, hd = q.shape
    o = np.empty((Sq, n_q, hd))
    for j in range(n_q):
        g = kv_head_of(j, n_q, n_kv)
        o[:, j, :] = attend(q[:, j, :], k[:, g, :], v[:, g, :], causal, q_pos0)
    return o.reshape(Sq, n_q * hd)


def attention_forward(x, wq, wk, wv, wo, n_q, n_kv, head_dim, causal=True):
    """Unsharded block, x (b, s, h) -> y (b, s, h): y = Attn(x Wq, x Wk, x Wv) Wo."""
    x = _f64(x)
    if x.ndim == 2:
        x = x[None]
    ys = []
    for bi in range(x.shape[0]):
        q, k, v = project_qkv(x[bi], wq, wk, wv, n_q, n_kv, head_dim)
        ys.append(attention_heads(q, k, v, n_q, n_kv, causal) @ _f64(wo))
    return np.stack(ys)


def attention_forward_rows(x, wq, wk, wv, wo, n_q, n_kv, head_dim, rows, causal=True):
    """Rows ``rows`` (positions) of the unsharded block output for a single sequence x (s, h):
    keys and values over every position, queries only at the chosen rows.  Each sampled output
    row is computed over its full contraction, so it equals that row of attention_forward."""
    x = _f64(x)
    if x.ndim == 3:
        x = x[0]
    S = x.shape[0]
    k = (x @ _f64(wk)).reshape(S, n_kv, head_dim)
    v = (x @ _f64(wv)).reshape(S, n_kv, head_dim)
    out = []
    for r in rows:
        q = (x[r:r + 1] @ _f64(wq)).reshape(1, n_q, head_dim)
        o = attention_heads(q, k, v, n_q, n_kv, causal, q_pos0=r)
        out.append(o @ _f64(wo))
    return np.concatenate(out, axis=0)


def attention_forward_sharded(x, wq, wk, wv, wo, n_q, n_kv, head_dim, p, causal=True):
    """Sharded reference mode (invariant tests only).

    Shard i owns query heads [i n_q/p, (i+1) n_q/p), KV heads [i n_kv/p, (i+1) n_kv/p), the
    matching column slices of Wq/Wk/Wv and the matching row slice of Wo.  It computes its
    heads' attention locally and a full-width partial y_i = o_i Wo_i; y is the in-order sum.
    Returns (y, partials).
    """
    if n_q % p or n_kv % p:
        raise ValueError("p must divide both n_q and n_kv")
    x = _f64(x)
    if x.ndim == 2:
        x = x[None]
    wq, wk, wv, wo = _f64(wq), _f64(wk), _f64(wv), _f64(wo)
    qh, kh = n_q // p, n_kv // p
    partials = []
    for i in range(p):
        qc = slice(i * qh * head_dim, (i + 1) * qh * head_dim)
        kc = slice(i * kh * head_dim, (i + 1) * kh * head_dim)
        part = []
        for bi in range(x.shape[0]):
            q, k, v = project_qkv(x[bi], wq[:, qc], wk[:, kc], wv[:, kc], qh, kh, head_dim)
            part.append(attention_heads(q, k, v, qh, kh, causal) @ wo[qc, :])
        partials.append(np.stack(part))
    y = np.zeros_like(partials[0])
    for part in partials:
        y = y + part
    return y, partials


def attention_decode(x, wq, wk, wv, wo, k_cache, v_cache, n_q, n_kv, head_dim):
    """One decode step for a batch of single tokens.

    x (b, h) is the new token of each sequence; k_cache and v_cache (b, n_kv, L, hd) hold the
    keys and values of positions 0..L-1.  The new token sits at position L: its own key and
    value are appended, and it attends to all L+1 keys (causality is automatic).
    Returns (y (b, h), k_new (b, n_kv, hd), v_new (b, n_kv, hd)).
    """
    x = _f64(x)
    b = x.shape[0]
    ys, kn, vn = [], [], []
    for bi in range(b):
        q, k, v = project_qkv(x[bi:bi + 1], wq, wk, wv, n_q, n_kv, head_dim)
        keys = np.concatenate([_f64(k_cache[bi]), k.transpose(1, 0, 2)], axis=1)  # (n_kv, L+1, hd)
        vals = np.concatenate([_f64(v_cache[bi]), v.transpose(1, 0, 2)], axis=1)
        o = np.empty((n_q, head_dim))
        for j in range(n_q):
            g = kv_head_of(j, n_q, n_kv)
            o[j] = attend(q[0, j][None, :], keys[g], vals[g], causal=False)[0]
        ys.append(o.reshape(1, n_q * head_dim) @ _f64(wo))
        kn.append(k[0])
        vn.append(v[0])
    return np.concatenate(ys, axis=0), np.stack(kn), np.stack(vn)


# ----------------------------------------------------------------------------------- backward
# "Tensor Parallelism" (klaylearn), Notes: the attention block is column-parallel Q/K/V, local
# attention and a row-parallel output projection, so its backward has the same shape as the
# MLP's ("How does tensor parallelism split a transformer feed-forward block's two matmuls",
# "The backward pass"; the same page notes the pattern applies to multi-head attention): dY is
# replicated, each shard's weight gradients need no exchange, and dX is the sum of per-shard
# partials.  Here the block is unsharded; the chain rule is written out step by step.


def attend_backward(q, k, v, do, causal, q_pos0=0):
    """Gradients of one head's attention o = softmax(q k^T / sqrt(hd) [masked]) v.

    q (Sq, hd), k and v (Sk, hd), do (Sq, hd) = dL/do.  Returns dq, dk, dv.
      P = softmax(S), dV = P^T dO, dP = dO V^T,
      dS = P * (dP - D) with D = rowsum(dO * O) (= rowsum(P * dP)),
      dQ = dS K / sqrt(hd), dK = dS^T Q / sqrt(hd).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    hd = q.shape[-1]
    scale = 1.0 / np.sqrt(hd)
    s = (q @ k.T) * scale
    if causal:
        qpos = q_pos0 + np.arange(q.shape[0])[:, None]
        kpos = np.arange(k.shape[0])[None, :]
        s = np.where(kpos <= qpos, s, -np.inf)
    p = softmax_rows(s)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    d = np.sum(do * o, axis=-1, keepdims=True)
    ds = p * (dp - d)
    dq = (ds @ k) * scale
    dk = (ds.T @ q) * scale
    return dq, dk, dv


def attention_backward(x, wq, wk, wv, wo, dy, n_q, n_kv, head_dim, causal=True):
    """Unsharded block backward.  x and dy (b, s, h).  Returns dx (b, s, h) and the weight
    gradients dWq (h, n_q hd), dWk and dWv (h, n_kv hd), dWo (n_q hd, h), summed over the batch.

      O = attention(x Wq, x Wk, x Wv),  y = O Wo
      dWo = O^T dY,  dO = dY Wo^T,  (dQ, dK, dV) per head by attend_backward (a KV head collects
      the dK, dV of every query head that reads it),
      dWq = x^T dQ,  dWk = x^T dK,  dWv = x^T dV,  dx = dQ Wq^T + dK Wk^T + dV Wv^T.
    """
    x, dy = _f64(x), _f64(dy)
    if x.ndim == 2:
        x, dy = x[None], dy[None]
    wq, wk, wv, wo = _f64(wq), _f64(wk), _f64(wv), _f64(wo)
    dwq, dwk, dwv, dwo = (np.zeros_like(wq), np.zeros_like(wk), np.zeros_like(wv),
                          np.zeros_like(wo))
    dxs = []
    for bi in range(x.shape[0]):
        S = x.shape[1]
        q, k, v = project_qkv(x[bi], wq, wk, wv, n_q, n_kv, head_dim)
        o = attention_heads(q, k, v, n_q, n_kv, causal)               # (S, n_q hd)
        dwo += o.T @ dy[bi]
        do = (dy[bi] @ wo.T).reshape(S, n_q, head_dim)
        dq = np.zeros((S, n_q, head_dim))
        dk = np.zeros((S, n_kv, head_dim))
        dv = np.zeros((S, n_kv, head_dim))
        for j in range(n_q):
            g = kv_head_of(j, n_q, n_kv)
            a, b_, c = attend_backward(q[:, j], k[:, g], v[:, g], do[:, j], causal)
            dq[:, j] = a
            dk[:, g] += b_
            dv[:, g] += c
        dq, dk, dv = (t.reshape(S, -1) for t in (dq, dk, dv))
        dwq += x[bi].T @ dq
        dwk += x[bi].T @ dk
        dwv += x[bi].T @ dv
        dxs.append(dq @ wq.T + dk @ wk.T + dv @ wv.T)
    return np.stack(dxs), dwq, dwk, dwv, dwo
