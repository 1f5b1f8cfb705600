"""Pins for the MoE oracle ("Tensor-parallel all-reduce count per transformer layer in MLX
shard_linear", facts on MoE layers: experts and shared expert sharded in place, one block-level
sum, router replicated, bias added once after the sum).

They use hand-computed routing, scipy's softmax, the dense MLP oracle (pinned on its own), brute
force and the sharding invariants; none re-types the oracle's formulas.
"""
import math

import numpy as np
import pytest
from scipy.special import softmax

from oracle import mlp, moe


def _case(T=6, d=8, E=4, F=8, seed=0, shared=True):
    r = np.random.default_rng(seed)
    x = r.standard_normal((T, d))
    wr = r.standard_normal((d, E))
    experts = [tuple(r.standard_normal(s) / math.sqrt(s[0]) for s in ((d, F), (d, F), (F, d)))
               for _ in range(E)]
    sh = tuple(r.standard_normal(s) / math.sqrt(s[0]) for s in ((d, F), (d, F), (F, d))) if shared else None
    return x, wr, experts, sh


def test_routing_by_hand():
    # x picks rows of Wr: logits are known exactly
    wr = np.array([[1.0, 3.0, 2.0, 0.0],
                   [0.5, 0.5, 4.0, 1.0]])
    x = np.array([[1.0, 0.0], [0.0, 1.0]])
    idx, w = moe.route(x, wr, 2)
    assert idx.tolist() == [[1, 2], [2, 3]]
    # weights: softmax of the two chosen logits, e.g. e^3 / (e^3 + e^2)
    assert abs(w[0, 0] - math.exp(3) / (math.exp(3) + math.exp(2))) < 1e-15
    assert abs(w[1, 1] - math.exp(1) / (math.exp(4) + math.exp(1))) < 1e-15
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)


def test_routing_ties_take_lower_index():
    wr = np.array([[2.0, 5.0, 5.0, 5.0]])
    idx, w = moe.route(np.array([[1.0]]), wr, 2)
    assert idx.tolist() == [[1, 2]]
    assert w.tolist() == [[0.5, 0.5]]


def test_k_equals_E_is_full_softmax_mixture():
    x, wr, experts, _ = _case(shared=False)
    E = len(experts)
    y = moe.moe_forward(x, wr, experts, E)
    g = softmax(x @ wr, axis=1)
    want = sum(g[:, e:e + 1] * mlp.mlp_forward(x, ex[0], ex[2], "swiglu", ex[1])
               for e, ex in enumerate(experts))
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-13)


def test_one_expert_is_the_dense_mlp():
    x, wr, experts, _ = _case(E=1, shared=False)
    y = moe.moe_forward(x, wr, experts, 1)
    wg, wu, w2 = experts[0]
    np.testing.assert_allclose(y, mlp.mlp_forward(x, wg, w2, "swiglu", wu), rtol=1e-13)


def test_brute_force_top1():
    # k = 1: each token's output is exactly its arg-max expert's block (weight 1)
    x, wr, experts, _ = _case(shared=False, seed=3)
    y = moe.moe_forward(x, wr, experts, 1)
    for t in range(x.shape[0]):
        logits = [sum(x[t, i] * wr[i, e] for i in range(x.shape[1])) for e in range(wr.shape[1])]
        e = max(range(len(logits)), key=lambda j: (logits[j], -j))
        wg, wu, w2 = experts[e]
        np.testing.assert_allclose(y[t], mlp.mlp_forward(x[t:t + 1], wg, w2, "swiglu", wu)[0],
                                   rtol=1e-13)


@pytest.mark.parametrize("p", [1, 2, 4, 8])
def test_sharded_sum_equals_unsharded(p):
    x, wr, experts, sh = _case(seed=4)
    bias = np.arange(x.shape[1], dtype=np.float64)
    y, parts = moe.moe_forward_sharded(x, wr, experts, 2, p, shared=sh, bias=bias)
    assert len(parts) == p   # one partial per shard: one block-level reduction
    np.testing.assert_allclose(y, moe.moe_forward(x, wr, experts, 2, shared=sh, bias=bias),
                               rtol=1e-12, atol=1e-12)


def test_shared_expert_folds_into_the_one_sum():
    x, wr, experts, sh = _case(seed=5)
    routed = moe.moe_forward(x, wr, experts, 2)
    both = moe.moe_forward(x, wr, experts, 2, shared=sh)
    np.testing.assert_allclose(both - routed, mlp.mlp_forward(x, sh[0], sh[2], "swiglu", sh[1]),
                               rtol=1e-12, atol=1e-13)
    # sharded: the shared expert's slice is inside each shard's partial, no second sum
    _, parts = moe.moe_forward_sharded(x, wr, experts, 2, 2, shared=sh)
    _, parts_r = moe.moe_forward_sharded(x, wr, experts, 2, 2)
    shared_parts = [p_ - q_ for p_, q_ in zip(parts, parts_r)]
    np.testing.assert_allclose(sum(shared_parts), mlp.mlp_forward(x, sh[0], sh[2], "swiglu", sh[1]),
                               rtol=1e-12, atol=1e-13)


def test_bias_added_once_after_the_sum():
    x, wr, experts, sh = _case(seed=6)
    bias = np.full(x.shape[1], 0.25)
    y0, _ = moe.moe_forward_sharded(x, wr, experts, 2, 4, shared=sh)
    y1, _ = moe.moe_forward_sharded(x, wr, experts, 2, 4, shared=sh, bias=bias)
    np.testing.assert_allclose(y1 - y0, np.broadcast_to(bias, y0.shape), rtol=0, atol=1e-14)


def test_given_routing_is_used():
    x, wr, experts, _ = _case(seed=7)
    idx = np.tile(np.array([[3, 0]]), (x.shape[0], 1))
    w = np.tile(np.array([[0.75, 0.25]]), (x.shape[0], 1))
    y = moe.moe_forward(x, wr, experts, 2, routing=(idx, w))
    f = lambda e: mlp.mlp_forward(x, experts[e][0], experts[e][2], "swiglu", experts[e][1])
    np.testing.assert_allclose(y, 0.75 * f(3) + 0.25 * f(0), rtol=1e-13)


def test_weights_for_a_given_choice_by_hand():
    # the weights of a given expert set are the softmax of those logits, in the order given
    wr = np.array([[1.0, 3.0, 2.0, 0.0]])
    x = np.array([[1.0]])
    w = moe.weights_for(x, wr, np.array([[2, 0]]))
    assert abs(w[0, 0] - math.e / (math.e + 1.0)) < 1e-15
    assert abs(w[0, 1] - 1.0 / (math.e + 1.0)) < 1e-15
    idx, wref = moe.route(x, wr, 2)
    assert np.array_equal(moe.weights_for(x, wr, idx), wref)


def test_weights_for_route_equals_scipy_renormalised_softmax():
    # softmax over all experts, renormalised over the chosen k (scipy), for a random case
    x, wr, _, _ = _case(T=9, d=8, E=16, seed=7)
    idx, _ = moe.route(x, wr, 3)
    g = softmax(x @ wr, axis=1)
    want = np.take_along_axis(g, idx, axis=1)
    want = want / want.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(moe.weights_for(x, wr, idx), want, rtol=1e-13)


def test_topk_margin_by_hand():
    # logits [1, 3, 2, 0]: the top-2 set {1, 2} has margin 2 - 1 = 1; swapping in expert 0 for
    # expert 2 gives a set that is not a top-2 set, margin 1 - 2 = -1; a repeated expert is never
    # valid; k = E has nothing unchosen
    wr = np.array([[1.0, 3.0, 2.0, 0.0]])
    x = np.array([[1.0]])
    assert moe.topk_margin(x, wr, np.array([[1, 2]]))[0] == 1.0
    assert moe.topk_margin(x, wr, np.array([[2, 1]]))[0] == 1.0
    assert moe.topk_margin(x, wr, np.array([[1, 0]]))[0] == -1.0
    assert moe.topk_margin(x, wr, np.array([[1, 1]]))[0] == -np.inf
    assert moe.topk_margin(x, wr, np.array([[0, 1, 2, 3]]))[0] == np.inf


def test_topk_margin_of_route_is_the_logit_gap():
    # brute force: for the oracle's own choice the margin is the k-th minus the (k+1)-th largest
    # logit, >= 0 for every token
    x, wr, _, _ = _case(T=20, d=8, E=12, seed=8)
    k = 4
    idx, _ = moe.route(x, wr, k)
    srt = -np.sort(-(x @ wr), axis=1)
    np.testing.assert_allclose(moe.topk_margin(x, wr, idx), srt[:, k - 1] - srt[:, k], rtol=1e-14)
    assert (moe.topk_margin(x, wr, idx) >= 0).all()


# --- backward: central finite differences of the forward (itself pinned above), with the choice
# of experts held at the base point's and the weights recomputed from the perturbed logits

def _fd_case(seed=3, T=5, d=6, E=5, F=4, k=2):
    r = np.random.default_rng(seed)
    for _ in range(200):
        x = r.standard_normal((T, d))
        wr = r.standard_normal((d, E))
        idx, _ = moe.route(x, wr, k)
        if moe.topk_margin(x, wr, idx).min() > 0.3:   # no choice flips under a 1e-6 step
            break
    experts = [tuple(r.standard_normal(s) / math.sqrt(s[0]) for s in ((d, F), (d, F), (F, d)))
               for _ in range(E)]
    sh = tuple(r.standard_normal(s) / math.sqrt(s[0]) for s in ((d, F), (d, F), (F, d)))
    dy = r.standard_normal((T, d))
    return x, wr, experts, sh, dy, idx, k


def _loss(x, wr, experts, sh, dy, idx, k):
    w = moe.weights_for(x, wr, idx)
    return float(np.sum(dy * moe.moe_forward(x, wr, experts, k, shared=sh, routing=(idx, w))))


def _fd(fun, a, entries, e=1e-6):
    out = []
    for ij in entries:
        keep = a[ij]
        a[ij] = keep + e
        up = fun()
        a[ij] = keep - e
        dn = fun()
        a[ij] = keep
        out.append((up - dn) / (2 * e))
    return np.array(out)


def test_backward_matches_finite_differences():
    x, wr, experts, sh, dy, idx, k = _fd_case()
    g = moe.moe_backward(x, wr, experts, k, dy, shared=sh)
    f = lambda: _loss(x, wr, experts, sh, dy, idx, k)
    ent = [(t, c) for t in range(x.shape[0]) for c in range(x.shape[1])]
    np.testing.assert_allclose(g["dx"][tuple(np.array(ent).T)], _fd(f, x, ent), rtol=1e-6, atol=1e-7)
    ent = [(c, e) for c in range(wr.shape[0]) for e in range(wr.shape[1])]
    np.testing.assert_allclose(g["dwr"][tuple(np.array(ent).T)], _fd(f, wr, ent), rtol=1e-6, atol=1e-7)
    used = sorted(set(int(e) for e in idx.ravel()))
    for e in used[:2]:
        for name, a in zip(("dwg", "dwu", "dw2"), experts[e]):
            ent = [(i, j) for i in range(a.shape[0]) for j in range(a.shape[1])][:7]
            np.testing.assert_allclose(g["experts"][e][name][tuple(np.array(ent).T)], _fd(f, a, ent),
                                       rtol=1e-6, atol=1e-7)
    for name, a in zip(("dwg", "dwu", "dw2"), sh):
        ent = [(i, j) for i in range(a.shape[0]) for j in range(a.shape[1])][:7]
        np.testing.assert_allclose(g["shared"][name][tuple(np.array(ent).T)], _fd(f, a, ent),
                                   rtol=1e-6, atol=1e-7)
    # an expert no token chose gets no gradient
    for e in set(range(len(experts))) - set(used):
        assert all(not g["experts"][e][n].any() for n in ("dwg", "dwu", "dw2"))


def test_backward_one_expert_is_the_dense_mlp_backward():
    # k = E = 1: the weight is 1 whatever the logit, so the router gets no gradient and the
    # block's gradients are the dense MLP oracle's
    x, wr, experts, _ = _case(E=1, shared=False)
    dy = np.random.default_rng(7).standard_normal(x.shape)
    g = moe.moe_backward(x, wr, experts, 1, dy)
    wg, wu, w2 = experts[0]
    b = mlp.mlp_backward(x, wg, w2, dy, "swiglu", wu)
    np.testing.assert_allclose(g["dx"], b["dx"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["experts"][0]["dwg"], b["dw1"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["experts"][0]["dw2"], b["dw2"], rtol=1e-12, atol=1e-12)
    assert not g["dwr"].any()
