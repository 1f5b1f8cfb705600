"""One shard per rank (tp_dist) on CPU: world-size-2 gloo process groups.

The rank driver's own logic is checked here without a GPU: rank r packs and computes shard r,
the group's all-reduce adds the partials (one collective per block forward and one backward),
the residual is added once after the sum, and each rank keeps its own weight gradients.  The
library's shard calls are replaced by a float64 stand-in that computes a shard's partial with the
oracle's per-shard formulas; the result must equal the UNSHARDED oracle block ("How does tensor
parallelism split a transformer feed-forward block's two matmuls", "One collective" and "The
backward pass"; "Tensor Parallelism" (klaylearn), Notes: heads split across ranks, Wo by rows).
The GPU tests check the library's shard calls themselves.
"""

import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import attention as oattn
from oracle import mlp as omlp


class OracleShardLib:
    """Stand-in for the library's shard calls: float64 CPU tensors, oracle arithmetic.

    The 'packed' buffers hold the shard's slices of the user matrices in float64."""

    def mlp_desc(self, T, d, d_ff, p, act, dtype):
        return types.SimpleNamespace(T=T, d=d, F=d_ff, p=p, act=act)

    def attn_desc(self, b, s, h, n_q, n_kv, hd, p, causal, dtype, kv_len, kv_cap=0):
        return types.SimpleNamespace(b=b, s=s, h=h, n_q=n_q, n_kv=n_kv, hd=hd, p=p,
                                     causal=causal)

    # ---- MLP
    def tp_mlp_shard_sizes(self, desc, partial_dtype):
        fs = desc.F // desc.p
        k = 2 if desc.act == "swiglu" else 1
        return types.SimpleNamespace(col_weight_bytes=8 * k * desc.d * fs,
                                     row_weight_bytes=8 * fs * desc.d, saved_bytes=8,
                                     fwd_workspace=8, bwd_workspace=8,
                                     partial_bytes=8 * desc.T * desc.d)

    def _mlp_views(self, desc, w1p, w2p):
        fs = desc.F // desc.p
        k = 2 if desc.act == "swiglu" else 1
        a = w1p.view(torch.float64).view(k, desc.d, fs)
        return a[0], (a[1] if k == 2 else None), w2p.view(torch.float64).view(fs, desc.d)

    def tp_mlp_pack_shard(self, desc, shard, w1, w_up, w2, w1p, w2p):
        fs = desc.F // desc.p
        c = slice(shard * fs, (shard + 1) * fs)
        g, u, o = self._mlp_views(desc, w1p, w2p)
        g.copy_(w1[:, c])
        if u is not None:
            u.copy_(w_up[:, c])
        o.copy_(w2[c, :])

    def tp_mlp_fwd_shard(self, desc, shard, x, w1p, w2p, partial, saved=None, workspace=None):
        g, u, o = self._mlp_views(desc, w1p, w2p)
        y = omlp.mlp_forward(x.numpy(), g.numpy(), o.numpy(), desc.act,
                             None if u is None else u.numpy())
        partial.copy_(torch.from_numpy(y))

    def tp_mlp_bwd_shard(self, desc, shard, dy, x, saved, w1p, w2p, dxp, dw1p, dw2p,
                         workspace=None):
        g, u, o = self._mlp_views(desc, w1p, w2p)
        r = omlp.mlp_backward(x.numpy(), g.numpy(), o.numpy(), dy.numpy(), desc.act,
                              None if u is None else u.numpy())
        dxp.copy_(torch.from_numpy(r["dx"]))
        dg, du, do = self._mlp_views(desc, dw1p, dw2p)
        dg.copy_(torch.from_numpy(r["dw1"]))
        if du is not None:
            du.copy_(torch.from_numpy(r["dw_up"]))
        do.copy_(torch.from_numpy(r["dw2"]))

    # ---- attention
    def tp_attn_shard_sizes(self, desc, partial_dtype):
        qc, kc = desc.n_q // desc.p * desc.hd, desc.n_kv // desc.p * desc.hd
        return types.SimpleNamespace(col_weight_bytes=8 * desc.h * (qc + 2 * kc),
                                     row_weight_bytes=8 * qc * desc.h, saved_bytes=0,
                                     fwd_workspace=8, bwd_workspace=8,
                                     partial_bytes=8 * desc.b * desc.s * desc.h)

    def _attn_views(self, desc, wqkv, wo):
        qc, kc = desc.n_q // desc.p * desc.hd, desc.n_kv // desc.p * desc.hd
        a = wqkv.view(torch.float64).view(desc.h, qc + 2 * kc)
        return a[:, :qc], a[:, qc:qc + kc], a[:, qc + kc:], wo.view(torch.float64).view(qc, desc.h)

    def tp_attn_pack_shard(self, desc, shard, wq, wk, wv, wo, wqkv_s, wo_s):
        qc, kc = desc.n_q // desc.p * desc.hd, desc.n_kv // desc.p * desc.hd
        q, k, v, o = self._attn_views(desc, wqkv_s, wo_s)
        q.copy_(wq[:, shard * qc:(shard + 1) * qc])
        k.copy_(wk[:, shard * kc:(shard + 1) * kc])
        v.copy_(wv[:, shard * kc:(shard + 1) * kc])
        o.copy_(wo[shard * qc:(shard + 1) * qc, :])

    def tp_attn_fwd_shard(self, desc, shard, x, wqkv_s, wo_s, partial, k_cache=None,
                          v_cache=None, workspace=None):
        q, k, v, o = self._attn_views(desc, wqkv_s, wo_s)
        y = oattn.attention_forward(x.numpy(), q.numpy(), k.numpy(), v.numpy(), o.numpy(),
                                    desc.n_q // desc.p, desc.n_kv // desc.p, desc.hd,
                                    causal=desc.causal)
        partial.copy_(torch.from_numpy(y))

    # ---- the residual add after the sum
    def tp_reduce_partials(self, partials, p, n, out, residual=None):
        assert p == 1
        out.copy_(partials + (0 if residual is None else residual))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _mlp_case(act):
    r = np.random.default_rng(7)
    T, d, F = 5, 6, 8
    w = {k: torch.from_numpy(r.standard_normal(s) / np.sqrt(s[0])) for k, s in
         (("x", (T, d)), ("w1", (d, F)), ("wu", (d, F)), ("w2", (F, d)), ("dy", (T, d)),
          ("res", (T, d)))}
    if act != "swiglu":
        w["wu"] = None
    return T, d, F, w


def _worker(rank, world, port, which, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from tensor_transformer_matmul_b200 import tp_dist
        lib = OracleShardLib()
        g = tp_dist.TPGroup()
        out = {}
        if which in ("swiglu", "gelu"):
            T, d, F, w = _mlp_case(which)
            m = tp_dist.ShardedMLP(g, T, d, F, act=which, dtype="f64",
                                   partial_dtype=torch.float64, device="cpu", lib=lib)
            m.pack(w["w1"], w["wu"], w["w2"])
            y = m.forward(w["x"], residual=w["res"])
            after_fwd = g.count
            dx = m.backward(w["dy"], w["x"])
            fs = F // world
            out = {"y": y.numpy().copy(), "dx": dx.numpy().copy(), "count_fwd": after_fwd,
                   "count": g.count,
                   "dw1": m.dw1p.view(torch.float64)[:d * fs].view(d, fs).numpy().copy(),
                   "dw2": m.dw2p.view(torch.float64).view(fs, d).numpy().copy()}
        else:
            r = np.random.default_rng(8)
            b, s, h, n_q, n_kv, hd = 2, 5, 8, 4, 2, 3
            a = {k: torch.from_numpy(r.standard_normal(sh) * 0.5) for k, sh in
                 (("x", (b, s, h)), ("wq", (h, n_q * hd)), ("wk", (h, n_kv * hd)),
                  ("wv", (h, n_kv * hd)), ("wo", (n_q * hd, h)), ("res", (b, s, h)))}
            at = tp_dist.ShardedAttention(g, b, s, h, n_q, n_kv, hd, causal=True, dtype="f64",
                                          partial_dtype=torch.float64, device="cpu", lib=lib)
            at.pack(a["wq"], a["wk"], a["wv"], a["wo"])
            y = at.forward(a["x"], residual=a["res"])
            out = {"y": y.numpy().copy(), "count": g.count}
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def _run(which, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, which, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_sharded_mlp_over_two_ranks_equals_unsharded(act):
    res = _run(act)
    T, d, F, w = _mlp_case(act)
    f = lambda k: None if w[k] is None else w[k].numpy()
    y_ref = omlp.mlp_forward(f("x"), f("w1"), f("w2"), act, f("wu")) + f("res")
    g_ref = omlp.mlp_backward(f("x"), f("w1"), f("w2"), f("dy"), act, f("wu"))
    fs = F // 2
    for rank in (0, 1):
        r = res[rank]
        # every rank holds the replicated result of the one collective
        np.testing.assert_allclose(r["y"], y_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(r["dx"], g_ref["dx"], rtol=1e-12, atol=1e-12)
        # one all-reduce forward, one backward
        assert r["count_fwd"] == 1 and r["count"] == 2
        # rank r owns columns r*F/p .. of W1 and rows of W2: its weight gradients are exactly
        # that slice of the unsharded ones, with no exchange
        c = slice(rank * fs, (rank + 1) * fs)
        np.testing.assert_allclose(r["dw1"], g_ref["dw1"][:, c], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(r["dw2"], g_ref["dw2"][c, :], rtol=1e-12, atol=1e-12)


def test_sharded_attention_over_two_ranks_equals_unsharded():
    res = _run("attention")
    r = np.random.default_rng(8)
    b, s, h, n_q, n_kv, hd = 2, 5, 8, 4, 2, 3
    a = {k: r.standard_normal(sh) * 0.5 for k, sh in
         (("x", (b, s, h)), ("wq", (h, n_q * hd)), ("wk", (h, n_kv * hd)),
          ("wv", (h, n_kv * hd)), ("wo", (n_q * hd, h)), ("res", (b, s, h)))}
    y_ref = oattn.attention_forward(a["x"], a["wq"], a["wk"], a["wv"], a["wo"], n_q, n_kv, hd,
                                    causal=True) + a["res"]
    for rank in (0, 1):
        np.testing.assert_allclose(res[rank]["y"], y_ref, rtol=1e-12, atol=1e-12)
        assert res[rank]["count"] == 1
