"""Tensor-parallel MoE block on the GPU through the C ABI, against the float64 oracle.

Routing is a discrete decision taken from fp32 logits, so near ties may break either way.  It is
checked for every token: the GPU's chosen set must be a top-k set of the exact (float64) logits
within the router's rounding bound, listed in descending logit order within that bound, and where
the choice is unique (a clear gap between the k-th and (k+1)-th logit) it must be the oracle's.  Only the GPU's expert indices
go to the oracle: the oracle computes their weights from its own float64 logits, the GPU's
weights are compared with those, and the block's output is compared with the oracle's output on
those experts, rel-L2 <= 2e-2 (bf16) for the whole tensor and for every row.
"""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from tensor_transformer_matmul_b200 import inputs
from tests.helpers import TOL, dev, f64, rel_l2, rel_l2_rows

pytestmark = pytest.mark.gpu


def _setup(lib, T, d, E, k, F, Fs, p, seed, with_bias=True, with_res=True):
    g = dev()
    rnd = lambda shape, std, salt: inputs.normal(shape, std, seed, salt, "bf16", "cpu")
    x = rnd((T, d), 1.0, 1)
    wr = rnd((d, E), 1.0 / np.sqrt(d), 2)
    ex = [(rnd((d, F), 0.05, 10 + 3 * e), rnd((d, F), 0.05, 11 + 3 * e), rnd((F, d), 0.05, 12 + 3 * e))
          for e in range(E)]
    sh = (rnd((d, Fs), 0.05, 5), rnd((d, Fs), 0.05, 6), rnd((Fs, d), 0.05, 7)) if Fs else None
    bias = rnd((d,), 0.5, 8) if with_bias else None
    res = rnd((T, d), 1.0, 9) if with_res else None
    desc = lib.moe_desc(T, d, F, Fs, E, k, p)
    w1p = torch.empty(E * lib.tp_moe_expert_w1_bytes(desc) // 2, dtype=torch.bfloat16, device=g)
    w2p = torch.empty(E * lib.tp_moe_expert_w2_bytes(desc) // 2, dtype=torch.bfloat16, device=g)
    w1s = w2s = None
    if Fs:
        w1s = torch.empty(lib.tp_moe_shared_w1_bytes(desc) // 2, dtype=torch.bfloat16, device=g)
        w2s = torch.empty(lib.tp_moe_shared_w2_bytes(desc) // 2, dtype=torch.bfloat16, device=g)
    dex = [tuple(t.to(g) for t in e) for e in ex]
    lib.tp_moe_pack(desc, [e[0] for e in dex], [e[1] for e in dex], [e[2] for e in dex], w1p, w2p,
                    shared=None if sh is None else tuple(t.to(g) for t in sh), w1p_s=w1s, w2p_s=w2s)
    ws = torch.empty(lib.tp_moe_fwd_workspace(desc), dtype=torch.uint8, device=g)
    st = dict(desc=desc, x=x, wr=wr, ex=ex, sh=sh, bias=bias, res=res, w1p=w1p, w2p=w2p, w1s=w1s,
              w2s=w2s, ws=ws, T=T, d=d, k=k)
    return st


def _run(lib, st):
    g = dev()
    T, d, k = st["T"], st["d"], st["k"]
    y = torch.empty(T, d, dtype=torch.bfloat16, device=g)
    idx = torch.empty(T, k, dtype=torch.int32, device=g)
    w = torch.empty(T, k, dtype=torch.float32, device=g)
    lib.tp_moe_fwd(st["desc"], st["x"].to(g), st["wr"].to(g), st["w1p"], st["w2p"], y,
                   w1p_s=st["w1s"], w2p_s=st["w2s"],
                   bias=None if st["bias"] is None else st["bias"].to(g),
                   residual=None if st["res"] is None else st["res"].to(g),
                   route_idx=idx, route_w=w, workspace=st["ws"])
    return y, idx, w


def router_eps(x, wr):
    """Per-token bound on how far apart the GPU's and the exact logits of two experts can be.

    The router forms each logit as a sum of d products of bf16 values, each exact in fp32, added
    in fp32 in some order; the error of such a sum is at most d * u * sum_k |x_k w_ke|
    (u = 2^-23 also covers an accumulator that truncates).  Two logits: twice that, with 1%
    slack for the bound's higher-order term."""
    d = x.shape[1]
    return 2.0 * 1.01 * d * 2.0 ** -23 * (np.abs(x) @ np.abs(wr)).max(axis=1)


def _check(st, y, idx, w):
    x, wr = f64(st["x"]), f64(st["wr"])
    k, E = st["k"], wr.shape[1]
    gi, gw = idx.cpu().numpy().astype(np.int64), w.cpu().numpy().astype(np.float64)
    assert ((gi >= 0) & (gi < E)).all()
    # every token: a valid top-k set of the exact logits, within the router's rounding
    assert (omoe.topk_margin(x, wr, gi) >= -router_eps(x, wr)).all()
    # where the choice is unique it is the oracle's set; the order is descending in the exact
    # logits, within the same rounding bound
    eps = router_eps(x, wr)
    logits = x @ wr
    ref_idx, _ = omoe.route(x, wr, k)
    srt = -np.sort(-logits, axis=1)
    gap = srt[:, k - 1] - srt[:, k] if k < E else np.full(len(srt), np.inf)
    clear = gap > eps
    assert clear.mean() > 0.8
    assert np.array_equal(np.sort(gi[clear], axis=1), np.sort(ref_idx[clear], axis=1))
    chosen = np.take_along_axis(logits, gi, axis=1)
    assert (chosen[:, :-1] >= chosen[:, 1:] - eps[:, None]).all()
    # the weights of the chosen experts come from the oracle's own logits
    ow = omoe.weights_for(x, wr, gi)
    assert np.abs(gw - ow).max() <= 1e-4
    experts = [tuple(f64(t) for t in e) for e in st["ex"]]
    sh = None if st["sh"] is None else tuple(f64(t) for t in st["sh"])
    ref = omoe.moe_forward(x, wr, experts, k, shared=sh,
                           bias=None if st["bias"] is None else f64(st["bias"]),
                           routing=(gi, ow))
    if st["res"] is not None:
        ref = ref + f64(st["res"])
    assert rel_l2(f64(y), ref) <= TOL["bf16"]
    assert rel_l2_rows(f64(y), ref) <= TOL["bf16"]


@pytest.mark.parametrize("T,d,E,k,F,Fs,p", [
    (200, 256, 16, 2, 512, 256, 2),    # few experts (SIMT router), shared expert, bias, residual
    (150, 512, 64, 4, 256, 0, 4),      # tensor-core router, no shared expert
    (1, 256, 64, 8, 256, 256, 2),      # one token (decode), eight experts
    (300, 264, 128, 2, 384, 128, 1),   # ragged d, 128 experts, p = 1
    (400, 256, 8, 2, 256, 128, 2),     # ~100 rows per expert, some with two row blocks
    (600, 256, 8, 4, 512, 0, 4),       # ~300 rows per expert: three 128-row blocks
])
def test_moe_forward_parity(lib, T, d, E, k, F, Fs, p):
    st = _setup(lib, T, d, E, k, F, Fs, p, seed=50 + T)
    lib.tp_reset_reduction_count()
    y, idx, w = _run(lib, st)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    _check(st, y, idx, w)


def test_moe_skewed_routing(lib):
    # a router column pair that dominates every token: experts 0 and 1 each receive all 300
    # tokens (three 128-row blocks apiece) and the other 62 experts none
    st = _setup(lib, 300, 256, 64, 2, 256, 128, 2, seed=61)
    wr = st["wr"].float()
    wr[:, 0] += 0.5 * torch.sign(st["x"].float().sum(0))
    wr[:, 1] += 0.45 * torch.sign(st["x"].float().sum(0))
    st["wr"] = wr.to(torch.bfloat16)
    st["x"] = (st["x"].float() + torch.sign(st["x"].float().sum(0))).to(torch.bfloat16)
    y, idx, w = _run(lib, st)
    torch.cuda.synchronize()
    counts = torch.bincount(idx.flatten().long().cpu(), minlength=64)
    assert counts[0] == 300 and counts[1] == 300 and counts[2:].sum() == 0
    _check(st, y, idx, w)


def test_moe_skewed_routing_many_blocks(lib):
    # as above with few experts: experts 0 and 1 each receive all 600 tokens (five 128-row
    # blocks apiece, the last part-filled)
    st = _setup(lib, 600, 256, 8, 2, 256, 128, 2, seed=62)
    wr = st["wr"].float()
    wr[:, 0] += 0.5 * torch.sign(st["x"].float().sum(0))
    wr[:, 1] += 0.45 * torch.sign(st["x"].float().sum(0))
    st["wr"] = wr.to(torch.bfloat16)
    st["x"] = (st["x"].float() + torch.sign(st["x"].float().sum(0))).to(torch.bfloat16)
    y, idx, w = _run(lib, st)
    torch.cuda.synchronize()
    counts = torch.bincount(idx.flatten().long().cpu(), minlength=8)
    assert counts[0] == 600 and counts[1] == 600 and counts[2:].sum() == 0
    _check(st, y, idx, w)


def test_moe_deterministic(lib):
    st = _setup(lib, 180, 256, 64, 2, 256, 128, 2, seed=60)
    a = [t.clone() for t in _run(lib, st)]
    b = _run(lib, st)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_moe_rejects(lib):
    assert lib.tp_moe_fwd_workspace(lib.moe_desc(8, 256, 512, 0, 12, 2, 2)) == 0   # E % 8
    assert lib.tp_moe_fwd_workspace(lib.moe_desc(8, 256, 512, 0, 16, 9, 2)) == 0   # top_k > 8
    assert lib.tp_moe_fwd_workspace(lib.moe_desc(8, 256, 510, 0, 16, 2, 4)) == 0   # p | d_ff


@pytest.mark.parametrize("T,d,E,k,F,Fs,p", [
    (200, 256, 16, 2, 512, 256, 2),    # few experts, shared expert
    (150, 512, 64, 4, 256, 0, 4),      # no shared expert, four shards
    (1, 256, 64, 8, 256, 256, 2),      # one token: eight experts of one row each
    (300, 264, 128, 2, 384, 128, 1),   # ragged d, 128 experts (some chosen by no token), p = 1
    (600, 256, 8, 4, 256, 128, 2),     # ~300 rows per expert: several row blocks each
])
def test_moe_backward_parity(lib, T, d, E, k, F, Fs, p):
    # the backward recomputes the routing; the forward's routing of the same x gives the GPU's
    # choice, and the oracle differentiates the block on that choice with its own weights
    st = _setup(lib, T, d, E, k, F, Fs, p, seed=70 + T, with_bias=False, with_res=False)
    _, idx, _ = _run(lib, st)
    g = dev()
    dy = inputs.normal((T, d), 1.0, 70 + T, 13, "bf16", "cpu")
    desc = st["desc"]
    dx = torch.empty(T, d, dtype=torch.bfloat16, device=g)
    dwr = torch.empty(d, E, dtype=torch.float32, device=g)
    dw1p = torch.full((st["w1p"].numel(),), float("nan"), dtype=torch.float32, device=g)
    dw2p = torch.full((st["w2p"].numel(),), float("nan"), dtype=torch.float32, device=g)
    dw1s = dw2s = None
    if Fs:
        dw1s = torch.empty(st["w1s"].numel(), dtype=torch.float32, device=g)
        dw2s = torch.empty(st["w2s"].numel(), dtype=torch.float32, device=g)
    ws = torch.empty(lib.tp_moe_bwd_workspace(desc), dtype=torch.uint8, device=g)
    lib.tp_moe_bwd(desc, st["x"].to(g), st["wr"].to(g), st["w1p"], st["w2p"], dy.to(g), dx, dwr,
                   dw1p, dw2p, w1p_s=st["w1s"], w2p_s=st["w2s"], dw1p_s=dw1s, dw2p_s=dw2s,
                   workspace=ws)
    torch.cuda.synchronize()
    x, wr = f64(st["x"]), f64(st["wr"])
    gi = idx.cpu().numpy().astype(np.int64)
    experts = [tuple(f64(t) for t in e) for e in st["ex"]]
    sh = None if st["sh"] is None else tuple(f64(t) for t in st["sh"])
    ref = omoe.moe_backward(x, wr, experts, k, f64(dy), shared=sh,
                            routing=(gi, omoe.weights_for(x, wr, gi)))
    assert rel_l2(f64(dx), ref["dx"]) <= TOL["bf16"] and rel_l2_rows(f64(dx), ref["dx"]) <= TOL["bf16"]
    assert rel_l2(f64(dwr), ref["dwr"]) <= TOL["bf16"]
    # each expert's gradient, unpacked from its slice of the packed gradients
    md = lib.mlp_desc(T, d, F, p, "swiglu", "bf16")
    n1, n2 = st["w1p"].numel() // E, st["w2p"].numel() // E
    used = set(gi.ravel().tolist())
    for e in range(E):
        a = (torch.empty(d, F, dtype=torch.float32, device=g), torch.empty(d, F, dtype=torch.float32, device=g),
             torch.empty(F, d, dtype=torch.float32, device=g))
        lib.tp_mlp_unpack_grads(md, dw1p[e * n1:(e + 1) * n1], dw2p[e * n2:(e + 1) * n2], *a)
        torch.cuda.synchronize()
        r = ref["experts"][e]
        if e not in used:
            assert all(not t.any() for t in a), e   # zeros, not left over
            continue
        for t, name in zip(a, ("dwg", "dwu", "dw2")):
            assert rel_l2(f64(t), r[name]) <= TOL["bf16"], (e, name)
    if Fs:
        ms = lib.mlp_desc(T, d, Fs, p, "swiglu", "bf16")
        a = (torch.empty(d, Fs, dtype=torch.float32, device=g), torch.empty(d, Fs, dtype=torch.float32, device=g),
             torch.empty(Fs, d, dtype=torch.float32, device=g))
        lib.tp_mlp_unpack_grads(ms, dw1s, dw2s, *a)
        torch.cuda.synchronize()
        for t, name in zip(a, ("dwg", "dwu", "dw2")):
            assert rel_l2(f64(t), ref["shared"][name]) <= TOL["bf16"], name
