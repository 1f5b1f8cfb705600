"""The one-shard-per-device calls on one GPU: run the p shards one after another, add their
partials in shard order with tp_reduce_partials (what the devices' all-reduce does across GPUs),
and compare with the float64 oracle of the UNSHARDED block ("How does tensor parallelism split a
transformer feed-forward block's two matmuls", "One collective", "The backward pass"; "Tensor
Parallelism" (klaylearn), Notes: heads split across devices, Wo by rows).

Also checked: a shard packed on its own (tp_*_pack_shard) is bit for bit the shard's slice of the
p-shard packing, the shard calls add nothing to the reduction counter, and each shard's weight
gradients are its slice of the one-call backward's.  Tolerance: rel-L2 <= 2e-2 (bf16), whole
tensor and row by row.
"""

import numpy as np
import pytest
import torch

from oracle import attention as oattn
from oracle import mlp as omlp
from tensor_transformer_matmul_b200 import inputs
from tests.helpers import TOL, Attn, Mlp, dev, f64, rel_l2, rel_l2_rows

pytestmark = pytest.mark.gpu


def _mlp_shards(lib, inp, p, act, pdt):
    """Pack every shard on its own and run its forward; returns (desc, sizes, shards, partials)."""
    T, d = inp["x"].shape
    F = inp["w1"].shape[1]
    desc = lib.mlp_desc(T, d, F, p, act, "bf16")
    sz = lib.tp_mlp_shard_sizes(desc, pdt)
    g = dev()
    shards, parts = [], []
    for i in range(p):
        w1p = torch.empty(sz.col_weight_bytes // 2, dtype=torch.bfloat16, device=g)
        w2p = torch.empty(sz.row_weight_bytes // 2, dtype=torch.bfloat16, device=g)
        lib.tp_mlp_pack_shard(desc, i, inp["w1"].to(g), None if inp["w_up"] is None else inp["w_up"].to(g),
                              inp["w2"].to(g), w1p, w2p)
        saved = torch.empty(sz.saved_bytes, dtype=torch.uint8, device=g)
        ws = torch.empty(sz.fwd_workspace, dtype=torch.uint8, device=g)
        part = torch.empty(T, d, dtype=pdt, device=g)
        lib.tp_mlp_fwd_shard(desc, i, inp["x"].to(g), w1p, w2p, part, saved=saved, workspace=ws)
        shards.append(dict(w1p=w1p, w2p=w2p, saved=saved))
        parts.append(part)
    return desc, sz, shards, parts


def _sum(lib, parts, out_dtype=torch.bfloat16):
    stack = torch.stack(parts)
    out = torch.empty(parts[0].shape, dtype=out_dtype, device=dev())
    lib.tp_reduce_partials(stack, len(parts), parts[0].numel(), out)
    return out


@pytest.mark.parametrize("act,T,d,F,p,pdt", [
    ("swiglu", 17, 328, 408, 3, torch.float32),   # decode tiles, ragged everything, p = 3
    ("swiglu", 300, 256, 1024, 4, torch.bfloat16),  # prefill pair tiles, bf16 partials
    ("gelu", 64, 256, 768, 2, torch.float32),
])
def test_mlp_shards_sum_to_the_block(lib, act, T, d, F, p, pdt):
    inp = inputs.mlp_inputs(T, d, F, act, "bf16", seed=20, w_std=0.05, backward=True)
    lib.tp_reset_reduction_count()
    desc, sz, shards, parts = _mlp_shards(lib, inp, p, act, pdt)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 0
    y = _sum(lib, parts)
    torch.cuda.synchronize()
    wu = None if inp["w_up"] is None else f64(inp["w_up"])
    ref = omlp.mlp_forward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), act, wu)
    assert rel_l2(f64(y), ref) <= TOL["bf16"] and rel_l2_rows(f64(y), ref) <= TOL["bf16"]
    # each shard alone against the oracle's per-shard partial
    _, ref_parts = omlp.mlp_forward_sharded(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), act, p, wu)
    for i in range(p):
        assert rel_l2(f64(parts[i]), ref_parts[i]) <= TOL["bf16"], i
    # a shard packed alone is its slice of the p-shard packing
    m = Mlp(lib, inp, p, act, "bf16")
    n1, n2 = sz.col_weight_bytes // 2, sz.row_weight_bytes // 2
    for i in range(p):
        assert torch.equal(shards[i]["w1p"], m.w1p[i * n1:(i + 1) * n1])
        assert torch.equal(shards[i]["w2p"], m.w2p[i * n2:(i + 1) * n2])
    # backward: dx partials summed, weight gradients per shard
    g = dev()
    dxs = []
    for i in range(p):
        dxp = torch.empty(T, d, dtype=pdt, device=g)
        dw1 = torch.empty(sz.col_weight_bytes // 2, dtype=torch.float32, device=g)
        dw2 = torch.empty(sz.row_weight_bytes // 2, dtype=torch.float32, device=g)
        ws = torch.empty(sz.bwd_workspace, dtype=torch.uint8, device=g)
        lib.tp_mlp_bwd_shard(desc, i, inp["dy"].to(g), inp["x"].to(g), shards[i]["saved"],
                             shards[i]["w1p"], shards[i]["w2p"], dxp, dw1, dw2, workspace=ws)
        shards[i]["dw1"], shards[i]["dw2"] = dw1, dw2
        dxs.append(dxp)
    dx = _sum(lib, dxs)
    m.forward(inp["x"])
    _, _, _, _, dw1p_all, dw2p_all = m.backward(inp["dy"], inp["x"])
    torch.cuda.synchronize()
    rb = omlp.mlp_backward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), f64(inp["dy"]), act, wu)
    assert rel_l2(f64(dx), rb["dx"]) <= TOL["bf16"] and rel_l2_rows(f64(dx), rb["dx"]) <= TOL["bf16"]
    for i in range(p):
        assert rel_l2(f64(shards[i]["dw1"]), f64(dw1p_all[i * n1:(i + 1) * n1])) <= TOL["bf16"], i
        assert rel_l2(f64(shards[i]["dw2"]), f64(dw2p_all[i * n2:(i + 1) * n2])) <= TOL["bf16"], i


def test_full_size_decode_mlp_eight_shards(lib):
    # T=64, d=8192, d_ff=28672: the 8 shards one after another, bf16 partials (the 1 MiB
    # all-reduce payload of a decode step), every row against the oracle
    T, d, F, p = 64, 8192, 28672, 8
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=0, device="cuda", w_std=0.02)
    _, _, _, parts = _mlp_shards(lib, inp, p, "swiglu", torch.bfloat16)
    y = _sum(lib, parts)
    torch.cuda.synchronize()
    ref = omlp.mlp_forward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), "swiglu", f64(inp["w_up"]))
    assert rel_l2(f64(y), ref) <= TOL["bf16"] and rel_l2_rows(f64(y), ref) <= TOL["bf16"]


@pytest.mark.parametrize("b,s,kv_len,h,n_q,n_kv,hd,p,pdt", [
    (1, 200, 0, 256, 8, 2, 64, 2, torch.float32),      # prefill (tcgen05 flash per shard)
    (2, 37, 0, 256, 4, 4, 128, 4, torch.bfloat16),     # MHA, one head per shard
    (2, 1, 300, 256, 8, 2, 64, 2, torch.float32),      # decode, each shard its own KV cache
])
def test_attention_shards_sum_to_the_block(lib, b, s, kv_len, h, n_q, n_kv, hd, p, pdt):
    inp = inputs.attn_inputs(b, s, h, n_q, n_kv, hd, "bf16", seed=21, w_std=0.05, kv_len=kv_len)
    g = dev()
    desc = lib.attn_desc(b, s, h, n_q, n_kv, hd, p, True, "bf16", kv_len)
    sz = lib.tp_attn_shard_sizes(desc, pdt)
    kh = n_kv // p
    parts, caches = [], []
    lib.tp_reset_reduction_count()
    for i in range(p):
        wqkv = torch.empty(sz.col_weight_bytes // 2, dtype=torch.bfloat16, device=g)
        wo = torch.empty(sz.row_weight_bytes // 2, dtype=torch.bfloat16, device=g)
        lib.tp_attn_pack_shard(desc, i, inp["wq"].to(g), inp["wk"].to(g), inp["wv"].to(g),
                               inp["wo"].to(g), wqkv, wo)
        kc = vc = None
        if kv_len:
            kc = inp["k_cache"][:, i * kh:(i + 1) * kh].contiguous().to(g)
            vc = inp["v_cache"][:, i * kh:(i + 1) * kh].contiguous().to(g)
            caches.append((kc, vc))
        ws = torch.empty(sz.fwd_workspace, dtype=torch.uint8, device=g)
        part = torch.empty(b, s, h, dtype=pdt, device=g)
        lib.tp_attn_fwd_shard(desc, i, inp["x"].to(g), wqkv, wo, part, k_cache=kc, v_cache=vc,
                              workspace=ws)
        parts.append(part)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 0     # the shard calls reduce nothing
    y = _sum(lib, parts)
    torch.cuda.synchronize()
    args = [f64(inp[k]) for k in ("wq", "wk", "wv", "wo")]
    if kv_len:
        ref, kn, vn = oattn.attention_decode(f64(inp["x"])[:, 0], *args,
                                             f64(inp["k_cache"])[:, :, :kv_len],
                                             f64(inp["v_cache"])[:, :, :kv_len], n_q, n_kv, hd)
        ref = ref[:, None]
        for i, (kc, vc) in enumerate(caches):   # the new key/value landed in the shard's cache
            assert rel_l2(f64(kc)[:, :, kv_len], kn[:, i * kh:(i + 1) * kh]) <= TOL["bf16"]
            assert rel_l2(f64(vc)[:, :, kv_len], vn[:, i * kh:(i + 1) * kh]) <= TOL["bf16"]
    else:
        ref = oattn.attention_forward(f64(inp["x"]), *args, n_q, n_kv, hd, causal=True)
    assert rel_l2(f64(y), ref) <= TOL["bf16"] and rel_l2_rows(f64(y), ref) <= TOL["bf16"]


def test_attention_backward_shards(lib):
    b, s, h, n_q, n_kv, hd, p = 1, 160, 256, 8, 2, 64, 2
    inp = inputs.attn_inputs(b, s, h, n_q, n_kv, hd, "bf16", seed=22, w_std=0.05)
    dy = inputs.normal((b, s, h), 1.0, 22, 97, "bf16", "cpu")
    g = dev()
    desc = lib.attn_desc(b, s, h, n_q, n_kv, hd, p)
    sz = lib.tp_attn_shard_sizes(desc, torch.bfloat16)
    assert sz.bwd_workspace > 0
    dxs, dws = [], []
    for i in range(p):
        wqkv = torch.empty(sz.col_weight_bytes // 2, dtype=torch.bfloat16, device=g)
        wo = torch.empty(sz.row_weight_bytes // 2, dtype=torch.bfloat16, device=g)
        lib.tp_attn_pack_shard(desc, i, inp["wq"].to(g), inp["wk"].to(g), inp["wv"].to(g),
                               inp["wo"].to(g), wqkv, wo)
        dxp = torch.empty(b, s, h, dtype=torch.bfloat16, device=g)
        dwqkv = torch.empty(wqkv.numel(), dtype=torch.float32, device=g)
        dwo = torch.empty(wo.numel(), dtype=torch.float32, device=g)
        ws = torch.empty(sz.bwd_workspace, dtype=torch.uint8, device=g)
        lib.tp_attn_bwd_shard(desc, i, inp["x"].to(g), wqkv, wo, dy.to(g), dxp, dwqkv, dwo,
                              workspace=ws)
        dxs.append(dxp)
        dws.append((dwqkv, dwo))
    dx = _sum(lib, dxs)
    a = Attn(lib, inp, p, "bf16", True, n_q=n_q, n_kv=n_kv, hd=hd)
    dwqkv_all = torch.empty(a.wqkv.numel(), dtype=torch.float32, device=g)
    dwo_all = torch.empty(a.wo.numel(), dtype=torch.float32, device=g)
    dx_all = torch.empty(b, s, h, dtype=torch.bfloat16, device=g)
    ws = torch.empty(lib.tp_attn_bwd_workspace(a.desc), dtype=torch.uint8, device=g)
    lib.tp_attn_bwd(a.desc, inp["x"].to(g), a.wqkv, a.wo, dy.to(g), dx_all, dwqkv_all, dwo_all,
                    workspace=ws)
    torch.cuda.synchronize()
    ref = oattn.attention_backward(*(f64(inp[k]) for k in ("x", "wq", "wk", "wv", "wo")), f64(dy),
                                   n_q, n_kv, hd, causal=True)
    assert rel_l2(f64(dx), ref[0]) <= TOL["bf16"] and rel_l2_rows(f64(dx[0]), ref[0][0]) <= TOL["bf16"]
    n1, n2 = sz.col_weight_bytes // 2, sz.row_weight_bytes // 2
    for i in range(p):
        assert rel_l2(f64(dws[i][0]), f64(dwqkv_all[i * n1:(i + 1) * n1])) <= TOL["bf16"], i
        assert rel_l2(f64(dws[i][1]), f64(dwo_all[i * n2:(i + 1) * n2])) <= TOL["bf16"], i


def test_shard_calls_reject_bad_arguments(lib):
    desc = lib.mlp_desc(8, 64, 256, 4, "swiglu", "bf16")
    for shard in (-1, 4):
        with pytest.raises(lib.TpError) as e:
            lib.tp_mlp_pack_shard(desc, shard, torch.zeros(1, device=dev()), torch.zeros(1, device=dev()),
                                  torch.zeros(1, device=dev()), torch.zeros(1, device=dev()),
                                  torch.zeros(1, device=dev()))
        assert e.value.status == lib.TP_ERR_INVALID_ARG
    with pytest.raises(lib.TpError):
        lib.tp_mlp_shard_sizes(lib.mlp_desc(8, 64, 256, 4, "swiglu", "f32"), torch.bfloat16)
