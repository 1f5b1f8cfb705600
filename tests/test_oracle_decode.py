"""Pins for the oracle's decode layer stack (a pre-norm Llama layer run layer after layer over a
KV cache per layer; "How does tensor parallelism split a transformer feed-forward block's two
matmuls", "One collective": the residual add and the following normalization stay replicated).

The stack is pinned against the causal multi-layer prefill of the same model (its last row, and
the keys and values each layer appends), which is built here from the attention and MLP oracles
(each pinned on its own); a stack that reused one layer's cache or weights, or did not pass x
from layer to layer, fails it.
"""

import numpy as np

from oracle import attention, decode, mlp

N_Q, N_KV, HD, H, F, L, LAYERS = 4, 2, 8, 16, 24, 6, 3


def _model(seed):
    r = np.random.default_rng(seed)
    shapes = (("wq", (H, N_Q * HD)), ("wk", (H, N_KV * HD)), ("wv", (H, N_KV * HD)),
              ("wo", (N_Q * HD, H)), ("wg", (H, F)), ("wu", (H, F)), ("w2", (F, H)))
    return [{k: 0.3 * r.standard_normal(s) for k, s in shapes} for _ in range(LAYERS)]


def _prefill(xs, layers):
    """Causal pre-norm prefill over the whole sequence xs (b, L+1, H); returns the final
    activations and, per layer, the normed input that the layer's keys and values come from."""
    x = xs
    normed = []
    for w in layers:
        a = decode.rmsnorm(x)
        normed.append(a)
        x = x + attention.attention_forward(a, w["wq"], w["wk"], w["wv"], w["wo"], N_Q, N_KV, HD,
                                            causal=True)
        x = x + np.stack([mlp.mlp_forward(decode.rmsnorm(x[b]), w["wg"], w["w2"], "swiglu",
                                          w["wu"]) for b in range(x.shape[0])])
    return x, normed


def _caches(normed, layers):
    """Layer l's cache: keys and values of positions 0..L-1 of that layer's normed input,
    laid out (b, n_kv, L, hd)."""
    out = []
    for a, w in zip(normed, layers):
        b = a.shape[0]
        kc = (a[:, :L] @ w["wk"]).reshape(b, L, N_KV, HD).transpose(0, 2, 1, 3)
        vc = (a[:, :L] @ w["wv"]).reshape(b, L, N_KV, HD).transpose(0, 2, 1, 3)
        out.append((kc, vc))
    return out


def test_decode_stack_equals_multilayer_prefill_last_row():
    layers = _model(1)
    xs = np.random.default_rng(2).standard_normal((2, L + 1, H))
    full, normed = _prefill(xs, layers)
    caches = _caches(normed, layers)
    out, appended = decode.decode_stack(xs[:, L], lambda l: layers[l] if l < LAYERS else None,
                                        lambda l: caches[l], N_Q, N_KV, HD)
    np.testing.assert_allclose(out, full[:, L], rtol=1e-11, atol=1e-12)
    assert len(appended) == LAYERS
    for l, (kn, vn) in enumerate(appended):
        a = normed[l][:, L]
        np.testing.assert_allclose(kn, (a @ layers[l]["wk"]).reshape(2, N_KV, HD), rtol=1e-12,
                                   atol=1e-13)
        np.testing.assert_allclose(vn, (a @ layers[l]["wv"]).reshape(2, N_KV, HD), rtol=1e-12,
                                   atol=1e-13)


def test_decode_stack_uses_each_layers_own_cache_and_weights():
    # the same model with layer 0's cache given to every layer, or with the layers' order
    # reversed, gives a different result: the prefill pin above has the power to see either
    layers = _model(3)
    xs = np.random.default_rng(4).standard_normal((1, L + 1, H))
    full, normed = _prefill(xs, layers)
    caches = _caches(normed, layers)
    ok, _ = decode.decode_stack(xs[:, L], lambda l: layers[l] if l < LAYERS else None,
                                lambda l: caches[l], N_Q, N_KV, HD)
    same_cache, _ = decode.decode_stack(xs[:, L], lambda l: layers[l] if l < LAYERS else None,
                                        lambda l: caches[0], N_Q, N_KV, HD)
    rev = layers[::-1]
    reversed_w, _ = decode.decode_stack(xs[:, L], lambda l: rev[l] if l < LAYERS else None,
                                        lambda l: caches[l], N_Q, N_KV, HD)
    np.testing.assert_allclose(ok, full[:, L], rtol=1e-11, atol=1e-12)
    for bad in (same_cache, reversed_w):
        assert np.linalg.norm(bad - full[:, L]) > 1e-3 * np.linalg.norm(full[:, L])


def test_one_layer_stack_is_the_decode_layer():
    layers = _model(5)[:1]
    xs = np.random.default_rng(6).standard_normal((1, L + 1, H))
    full, normed = _prefill(xs, layers)
    caches = _caches(normed, layers)
    out, _ = decode.decode_stack(xs[:, L], lambda l: layers[l] if l < 1 else None,
                                 lambda l: caches[l], N_Q, N_KV, HD)
    np.testing.assert_allclose(out, full[:, L], rtol=1e-11, atol=1e-12)
    assert np.array_equal(out, decode.decode_layer(xs[:, L], layers[0], *caches[0], N_Q, N_KV,
                                                   HD)[0])
