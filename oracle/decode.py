"""Oracle for the decode layer stack (float64, CPU).

Test infrastructure only (see the package docstring).

Sources (page title, section):

* "How does tensor parallelism split a transformer feed-forward block's two matmuls",
  "One collective": after the reduction every device holds the full y, "ready for the residual
  add and the following normalization layer, both of which stay replicated".
* "Tensor Parallelism" (klaylearn), Notes: Llama-style attention block with grouped-query heads.
* Page 1 (llms-explorer, "Tensor-parallel all-reduce count per transformer layer"), facts on
  dense Llama in mlx-lm: o_proj and down_proj are the two reductions of a layer.

Reading where the pages leave a step open: a pre-norm Llama layer,
    x <- x + Attn(RMSNorm(x)) ;  x <- x + SwiGLU-MLP(RMSNorm(x)),
with RMSNorm(x) = x / sqrt(mean(x^2) + eps), unit weight, eps = 1e-5.
"""

import numpy as np

from . import attention, mlp

RMS_EPS = 1e-5


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def rmsnorm(x, eps=RMS_EPS):
    """x / sqrt(mean(x^2) + eps) over the last axis (unit weight)."""
    x = _f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def decode_layer(x, w, k_cache, v_cache, n_q, n_kv, head_dim):
    """One layer for a batch of single tokens.

    x (b, h); ``w`` maps "wq", "wk", "wv", "wo", "wg", "wu", "w2" to input-major matrices;
    caches (b, n_kv, L, hd).  Returns (x_out, k_new, v_new).
    """
    x = _f64(x)
    a = rmsnorm(x)
    attn_out, k_new, v_new = attention.attention_decode(
        a, w["wq"], w["wk"], w["wv"], w["wo"], k_cache, v_cache, n_q, n_kv, head_dim)
    x = x + attn_out
    m = rmsnorm(x)
    x = x + mlp.mlp_forward(m, w["wg"], w["w2"], "swiglu", w_up=w["wu"])
    return x, k_new, v_new


def decode_stack(x, layer_weights, layer_caches, n_q, n_kv, head_dim):
    """Run the layers in order.  ``layer_weights(l)`` returns layer l's weight dict and
    ``layer_caches(l)`` its (k_cache, v_cache); both are callables so that a caller can produce
    one layer at a time.  Returns the final x and the list of appended (k_new, v_new)."""
    appended = []
    l = 0
    while True:
        w = layer_weights(l)
        if w is None:
            break
        kc, vc = layer_caches(l)
        x, kn, vn = decode_layer(x, w, kc, vc, n_q, n_kv, head_dim)
        appended.append((kn, vn))
        l += 1
    return x, appended
