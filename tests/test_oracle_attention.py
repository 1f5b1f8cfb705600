"""Pins for the attention and decode oracles (closed forms, library routines, invariants)."""

import math

import numpy as np
import pytest
import torch

from oracle import attention, decode, mlp


def _rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300)


def _case(b, s, h, n_q, n_kv, hd, seed=0, std=0.2):
    r = np.random.default_rng(seed)
    return (r.standard_normal((b, s, h)), std * r.standard_normal((h, n_q * hd)),
            std * r.standard_normal((h, n_kv * hd)), std * r.standard_normal((h, n_kv * hd)),
            std * r.standard_normal((n_q * hd, h)))


def _torch_sdpa_block(x, wq, wk, wv, wo, n_q, n_kv, hd, causal):
    """Library routine: torch's scaled_dot_product_attention in float64 with KV heads repeated
    to the query heads (head j -> KV head j // (n_q/n_kv))."""
    b, s, h = x.shape
    tx = torch.tensor(x)
    q = (tx @ torch.tensor(wq)).view(b, s, n_q, hd).transpose(1, 2)
    k = (tx @ torch.tensor(wk)).view(b, s, n_kv, hd).transpose(1, 2)
    v = (tx @ torch.tensor(wv)).view(b, s, n_kv, hd).transpose(1, 2)
    k = k.repeat_interleave(n_q // n_kv, dim=1)
    v = v.repeat_interleave(n_q // n_kv, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal)
    return (o.transpose(1, 2).reshape(b, s, n_q * hd) @ torch.tensor(wo)).numpy()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n_q,n_kv", [(8, 2), (4, 4), (6, 1)])
def test_matches_torch_sdpa(causal, n_q, n_kv):
    hd = 8
    x, wq, wk, wv, wo = _case(2, 9, 16, n_q, n_kv, hd, seed=n_q + n_kv)
    got = attention.attention_forward(x, wq, wk, wv, wo, n_q, n_kv, hd, causal)
    ref = _torch_sdpa_block(x, wq, wk, wv, wo, n_q, n_kv, hd, causal)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_first_query_sees_only_first_key():
    # causal closed form: position 0 attends to key 0 alone, so o[0] = v[0]
    r = np.random.default_rng(1)
    q, k, v = r.standard_normal((5, 4)), r.standard_normal((5, 4)), r.standard_normal((5, 4))
    o = attention.attend(q, k, v, causal=True)
    np.testing.assert_array_equal(o[0], v[0])


def test_equal_keys_give_prefix_mean():
    # all keys equal -> uniform weights over the visible prefix
    r = np.random.default_rng(2)
    q, v = r.standard_normal((6, 4)), r.standard_normal((6, 4))
    k = np.tile(r.standard_normal((1, 4)), (6, 1))
    o = attention.attend(q, k, v, causal=True)
    for t in range(6):
        np.testing.assert_allclose(o[t], v[:t + 1].mean(axis=0), rtol=1e-13, atol=1e-14)


def test_single_key_returns_value_row():
    r = np.random.default_rng(3)
    q, k, v = r.standard_normal((3, 4)), r.standard_normal((1, 4)), r.standard_normal((1, 4))
    o = attention.attend(q, k, v, causal=False)
    np.testing.assert_allclose(o, np.tile(v, (3, 1)), rtol=1e-15)


def test_softmax_scale_is_inverse_sqrt_head_dim():
    # two keys with score gap g: weight ratio exp(g / sqrt(hd))
    hd = 16
    q = np.zeros((1, hd)); q[0, 0] = 1.0
    k = np.zeros((2, hd)); k[0, 0] = 3.0
    v = np.array([[1.0] + [0.0] * (hd - 1), [0.0] * hd])
    w0 = attention.attend(q, k, v, causal=False)[0, 0]
    expect = math.exp(3.0 / 4.0) / (math.exp(3.0 / 4.0) + 1.0)
    assert abs(w0 - expect) < 1e-15


@pytest.mark.parametrize("p", [1, 2, 4])
def test_sharded_heads_equal_unsharded(p):
    # "Tensor Parallelism", grouped-query paragraph: each rank owns whole Q heads with their KV
    # head, runs attention locally, and the output projections' partials sum to the block output
    n_q, n_kv, hd = 8, 4, 8
    x, wq, wk, wv, wo = _case(1, 7, 32, n_q, n_kv, hd, seed=5)
    ref = attention.attention_forward(x, wq, wk, wv, wo, n_q, n_kv, hd)
    y, parts = attention.attention_forward_sharded(x, wq, wk, wv, wo, n_q, n_kv, hd, p)
    assert len(parts) == p
    assert _rel(y, ref) <= 1e-13


def test_sharded_rejects_split_heads():
    x, wq, wk, wv, wo = _case(1, 3, 16, 8, 2, 4, seed=6)
    with pytest.raises(ValueError):
        attention.attention_forward_sharded(x, wq, wk, wv, wo, 8, 2, 4, p=4)


def test_70b_head_bookkeeping():
    # h=8192, 64 Q heads, 8 KV heads, hd=128, p=8: local Wq 8192x1024, Wk/Wv 8192x128, 8 Q + 1 KV
    h, n_q, n_kv, hd, p = 8192, 64, 8, 128, 8
    assert (h, n_q // p * hd) == (8192, 1024)
    assert (h, n_kv // p * hd) == (8192, 128)
    owners = [attention.kv_head_of(j, n_q, n_kv) for j in range(n_q)]
    for i in range(p):  # rank i's 8 query heads all read KV head i
        assert set(owners[8 * i:8 * i + 8]) == {i}


def test_decode_equals_last_row_of_causal_prefill():
    # a decode step over a cache built from the same tokens equals the last row of the causal
    # full-sequence computation
    n_q, n_kv, hd, h, L = 4, 2, 8, 16, 6
    x, wq, wk, wv, wo = _case(2, L + 1, h, n_q, n_kv, hd, seed=7)
    full = attention.attention_forward(x, wq, wk, wv, wo, n_q, n_kv, hd, causal=True)
    kc = np.stack([(x[bi, :L] @ wk).reshape(L, n_kv, hd).transpose(1, 0, 2) for bi in range(2)])
    vc = np.stack([(x[bi, :L] @ wv).reshape(L, n_kv, hd).transpose(1, 0, 2) for bi in range(2)])
    y, kn, vn = attention.attention_decode(x[:, L], wq, wk, wv, wo, kc, vc, n_q, n_kv, hd)
    np.testing.assert_allclose(y, full[:, L], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(kn, (x[:, L] @ wk).reshape(2, n_kv, hd), rtol=1e-14)


def test_rmsnorm_closed_form_and_library():
    c = np.full((1, 8), -3.0)
    np.testing.assert_allclose(decode.rmsnorm(c), -3.0 / np.sqrt(9.0 + 1e-5), rtol=1e-15)
    r = np.random.default_rng(8).standard_normal((3, 64))
    ref = torch.nn.functional.rms_norm(torch.tensor(r), (64,), eps=1e-5).numpy()
    np.testing.assert_allclose(decode.rmsnorm(r), ref, rtol=1e-13)


def test_decode_layer_equals_prefill_layer_last_row():
    # the decode layer (pre-norm attention + residual, pre-norm SwiGLU MLP + residual) on the
    # newest token equals the same layer applied causally to the whole sequence, last row
    n_q, n_kv, hd, h, F, L = 4, 2, 8, 16, 24, 5
    r = np.random.default_rng(9)
    xs = r.standard_normal((1, L + 1, h))
    w = {k: 0.2 * r.standard_normal(s) for k, s in
         (("wq", (h, n_q * hd)), ("wk", (h, n_kv * hd)), ("wv", (h, n_kv * hd)), ("wo", (n_q * hd, h)),
          ("wg", (h, F)), ("wu", (h, F)), ("w2", (F, h)))}
    a = decode.rmsnorm(xs)
    x1 = xs + attention.attention_forward(a, w["wq"], w["wk"], w["wv"], w["wo"], n_q, n_kv, hd, True)
    full = x1 + mlp.mlp_forward(decode.rmsnorm(x1[0]), w["wg"], w["w2"], "swiglu", w["wu"])[None]
    kc = (a[0, :L] @ w["wk"]).reshape(L, n_kv, hd).transpose(1, 0, 2)[None]
    vc = (a[0, :L] @ w["wv"]).reshape(L, n_kv, hd).transpose(1, 0, 2)[None]
    out, _, _ = decode.decode_layer(xs[:, L], w, kc, vc, n_q, n_kv, hd)
    np.testing.assert_allclose(out, full[:, L], rtol=1e-12, atol=1e-13)


def test_rows_match_full_forward():
    n_q, n_kv, hd = 8, 2, 8
    x, wq, wk, wv, wo = _case(1, 11, 32, n_q, n_kv, hd, seed=10)
    full = attention.attention_forward(x, wq, wk, wv, wo, n_q, n_kv, hd, causal=True)[0]
    rows = [0, 5, 10]
    got = attention.attention_forward_rows(x, wq, wk, wv, wo, n_q, n_kv, hd, rows, causal=True)
    np.testing.assert_allclose(got, full[rows], rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------------------ backward pins
def _torch_grads(x, wq, wk, wv, wo, dy, n_q, n_kv, hd, causal):
    """Library routine: torch autograd through SDPA in float64 with repeat-interleaved KV heads."""
    T = [torch.tensor(a, requires_grad=True) for a in (x, wq, wk, wv, wo)]
    X, Wq, Wk, Wv, Wo = T
    b, s, _ = x.shape
    Q = (X @ Wq).reshape(b, s, n_q, hd).transpose(1, 2)
    K = (X @ Wk).reshape(b, s, n_kv, hd).transpose(1, 2).repeat_interleave(n_q // n_kv, 1)
    V = (X @ Wv).reshape(b, s, n_kv, hd).transpose(1, 2).repeat_interleave(n_q // n_kv, 1)
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=causal)
    Y = O.transpose(1, 2).reshape(b, s, n_q * hd) @ Wo
    (Y * torch.tensor(dy)).sum().backward()
    return [t.grad.numpy() for t in T]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n_q,n_kv", [(4, 2), (4, 4), (8, 1)])
def test_backward_matches_torch_autograd(causal, n_q, n_kv):
    hd = 8
    x, wq, wk, wv, wo = _case(2, 9, 24, n_q, n_kv, hd, seed=20)
    dy = np.random.default_rng(21).standard_normal(x.shape)
    got = attention.attention_backward(x, wq, wk, wv, wo, dy, n_q, n_kv, hd, causal)
    ref = _torch_grads(x, wq, wk, wv, wo, dy, n_q, n_kv, hd, causal)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-12)


def test_backward_central_differences():
    # L = sum(y * dY); every gradient entry checked against (L(w+e) - L(w-e)) / 2e in float64
    n_q, n_kv, hd = 4, 2, 3
    x, wq, wk, wv, wo = _case(1, 5, 6, n_q, n_kv, hd, seed=22)
    dy = np.random.default_rng(23).standard_normal(x.shape)
    grads = attention.attention_backward(x, wq, wk, wv, wo, dy, n_q, n_kv, hd, True)
    args = [x, wq, wk, wv, wo]
    eps = 1e-6

    def loss(a):
        return float(np.sum(attention.attention_forward(*a, n_q, n_kv, hd, True) * dy))

    for which, g in enumerate(grads):
        base = args[which]
        for idx in np.ndindex(base.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd = (loss(plus) - loss(minus)) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (which, idx, fd, g[idx])


def test_backward_single_key_closed_form():
    # one position: the softmax has a single entry, so o = v and the scores get no gradient:
    # dq = dk = 0 and dv = do for every head (summed over the heads sharing a KV head)
    n_q, n_kv, hd = 4, 2, 5
    q, k, v = (np.random.default_rng(24 + i).standard_normal((1, hd)) for i in range(3))
    do = np.random.default_rng(27).standard_normal((1, hd))
    dq, dk, dv = attention.attend_backward(q, k, v, do, causal=True)
    # dS = P (dP - D) with dP = do.v and D = sum(do * o), o = v: zero up to summation order
    assert np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14
    np.testing.assert_allclose(dv, do, rtol=0, atol=0)
