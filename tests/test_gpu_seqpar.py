"""Sequence-parallel collectives and blocks on the GPU through the C ABI, against the oracle.

Tolerance: rel-L2 <= 2e-2 per slice for bf16 outputs, 1e-5 for fp32.  The all-gather moves bytes,
so it is compared bit for bit.  Where the sequence-parallel call does the same arithmetic as the
plain call (the same shard-order sum and residual add), its slices must equal the plain call's
rows bit for bit too.
"""
import numpy as np
import pytest
import torch

from oracle import attention as oattn
from oracle import decode as odec
from oracle import mlp as omlp
from oracle import seqpar as osp
from tensor_transformer_matmul_b200 import inputs
from tests.helpers import TOL, Attn, Mlp, dev, f64, rel_l2

pytestmark = pytest.mark.gpu


def _split(t, p):
    """p contiguous copies of t's token slices (separate allocations)."""
    r = t.shape[0] // p
    return [t[i * r:(i + 1) * r].clone().contiguous() for i in range(p)]


@pytest.mark.parametrize("p,T,d,out_dtype,with_res,with_norm", [
    (3, 9, 40, "bf16", True, True),      # vectorised rows, residual and norm
    (3, 9, 42, "bf16", True, True),      # d not a multiple of 8: the element path
    (8, 64, 8192, "bf16", False, True),  # decode-sized rows of the workload
    (4, 12, 64, "f32", True, False),     # fp32 output
    (1, 5, 16, "bf16", False, False),    # one shard
])
def test_reduce_scatter(lib, p, T, d, out_dtype, with_res, with_norm):
    part = inputs.normal((p, T, d), 1.0, 40, 1, "f32", "cpu")
    res = inputs.normal((T, d), 1.0, 40, 2, out_dtype, "cpu") if with_res else None
    odt = inputs.TORCH_DTYPE[out_dtype]
    outs = [torch.empty(T // p, d, dtype=odt, device=dev()) for _ in range(p)]
    norms = [torch.empty(T // p, d, dtype=torch.bfloat16, device=dev()) for _ in range(p)] if with_norm else None
    res_sl = _split(res.to(dev()), p) if with_res else None
    lib.tp_reset_reduction_count()
    lib.tp_reduce_scatter_partials(part.to(dev()), p, outs, residual=res_sl, norm=norms)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    ref = osp.reduce_scatter(f64(part), None if res is None else [f64(r) for r in _split(res, p)])
    tol = TOL[out_dtype]
    for i in range(p):
        assert rel_l2(f64(outs[i]), ref[i]) <= tol, i
        if with_norm:
            # the norm is taken of the stored output rows
            assert rel_l2(f64(norms[i]), odec.rmsnorm(f64(outs[i]))) <= TOL["bf16"], i


@pytest.mark.parametrize("eps", [0.0, 1e-5])
def test_reduce_scatter_eps_is_used_as_given(lib, eps):
    # rows of size ~1e-3 (mean square ~1e-6), so eps = 1e-5 changes the norm by a factor ~3 and
    # eps = 0 must give x / sqrt(mean(x^2)) exactly as tp_rmsnorm does with the same eps
    p, T, d = 2, 4, 64
    part = inputs.normal((p, T, d), 1e-3, 42, 1, "f32", "cpu")
    outs = [torch.empty(T // p, d, device=dev()) for _ in range(p)]
    norms = [torch.empty(T // p, d, device=dev()) for _ in range(p)]
    lib.tp_reduce_scatter_partials(part.to(dev()), p, outs, norm=norms, eps=eps)
    torch.cuda.synchronize()
    for i in range(p):
        assert rel_l2(f64(norms[i]), odec.rmsnorm(f64(outs[i]), eps=eps)) <= TOL["f32"], i
        other = 1e-5 if eps == 0.0 else 0.0
        assert rel_l2(f64(norms[i]), odec.rmsnorm(f64(outs[i]), eps=other)) > 0.1, i


@pytest.mark.parametrize("p,R,d,dtype", [(4, 3, 8192, "bf16"), (3, 5, 7, "bf16"), (2, 4, 6, "f32"),
                                         (8, 8, 8192, "f32")])
def test_all_gather_exact(lib, p, R, d, dtype):
    full = inputs.normal((p * R, d), 1.0, 41, 1, dtype, "cpu").to(dev())
    slices = _split(full, p)
    out = torch.empty_like(full)
    lib.tp_all_gather_slices(slices, out)
    torch.cuda.synchronize()
    assert torch.equal(out, full)
    assert np.array_equal(f64(out), osp.all_gather([f64(s) for s in slices]))


def test_reduce_scatter_rejects_ragged_tokens(lib):
    part = torch.zeros(2, 5, 8, device=dev())
    outs = [torch.empty(2, 8, dtype=torch.bfloat16, device=dev()) for _ in range(2)]
    with pytest.raises(lib.TpError):
        lib.tp_reduce_scatter_partials(part, 2, outs)


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_mlp_forward_backward_sp(lib, act):
    # T = 520 tokens over p = 4 slices of 130 rows; the GEMMs are the pair-tile prefill path
    T, d, F, p = 520, 776, 1536, 4
    inp = inputs.mlp_inputs(T, d, F, act, "bf16", seed=42, w_std=0.05, backward=True)
    m = Mlp(lib, inp, p, act, "bf16")
    res = inputs.normal((T, d), 1.0, 42, 99, "bf16", "cpu").to(dev())
    x = inp["x"].to(dev())
    # plain block: y = residual + sum of partials, y_norm = RMSNorm(y)
    y = torch.empty(T, d, dtype=torch.bfloat16, device=dev())
    yn = torch.empty_like(y)
    lib.tp_mlp_fwd(m.desc, x, m.w1p, m.w2p, y, residual=res, saved=m.saved, workspace=m.ws_f,
                   y_norm=yn)
    # sequence-parallel block on the slices
    ys = [torch.empty(T // p, d, dtype=torch.bfloat16, device=dev()) for _ in range(p)]
    yns = [torch.empty_like(ys[0]) for _ in range(p)]
    ws = torch.empty(lib.tp_mlp_fwd_sp_workspace(m.desc), dtype=torch.uint8, device=dev())
    saved_sp = torch.empty_like(m.saved)
    lib.tp_reset_reduction_count()
    lib.tp_mlp_fwd_sp(m.desc, _split(x, p), m.w1p, m.w2p, ys, residual_slices=_split(res, p),
                      y_norm_slices=yns, saved=saved_sp, workspace=ws)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    assert torch.equal(torch.cat(ys), y) and torch.equal(torch.cat(yns), yn)
    wu = None if inp["w_up"] is None else f64(inp["w_up"])
    ref = osp.reduce_scatter(omlp.mlp_forward_sharded(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]),
                                                      act, p, wu)[1],
                             [f64(r) for r in _split(res.cpu(), p)])
    for i in range(p):
        assert rel_l2(f64(ys[i]), ref[i]) <= TOL["bf16"], i
    # backward: dy and x arrive as slices, dx leaves as slices
    dy = inp["dy"].to(dev())
    dxs = [torch.empty(T // p, d, dtype=torch.bfloat16, device=dev()) for _ in range(p)]
    dw1p = torch.empty(m.w1p.numel(), dtype=torch.float32, device=dev())
    dw2p = torch.empty(m.w2p.numel(), dtype=torch.float32, device=dev())
    wsb = torch.empty(lib.tp_mlp_bwd_sp_workspace(m.desc), dtype=torch.uint8, device=dev())
    lib.tp_reset_reduction_count()
    lib.tp_mlp_bwd_sp(m.desc, _split(dy, p), _split(x, p), saved_sp, m.w1p, m.w2p, dxs, dw1p, dw2p,
                      workspace=wsb)
    dx, _, _, _, dw1p_ref, dw2p_ref = m.backward(inp["dy"], inp["x"])
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 2   # the SP backward and the plain one
    assert torch.equal(torch.cat(dxs), dx)
    assert torch.equal(dw1p, dw1p_ref) and torch.equal(dw2p, dw2p_ref)
    g = omlp.mlp_backward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), f64(inp["dy"]), act, wu)
    ref_dx = osp.token_slices(T, p)
    for i, rows in enumerate(ref_dx):
        assert rel_l2(f64(dxs[i]), g["dx"][rows]) <= TOL["bf16"], i


def test_mlp_sp_rejects(lib):
    inp = inputs.mlp_inputs(10, 64, 256, "swiglu", "bf16", seed=43, w_std=0.05)
    fused = lib.mlp_desc(10, 64, 256, 2, "swiglu", "bf16", lib.TP_REDUCE_FUSED)
    assert lib.tp_mlp_fwd_sp_workspace(fused) == 0
    ragged = lib.mlp_desc(10, 64, 256, 4, "swiglu", "bf16")
    assert lib.tp_mlp_fwd_sp_workspace(ragged) == 0   # 4 does not divide 10 tokens


def test_attention_forward_sp(lib):
    # b=2, s=150: 300 token rows over p = 2 slices; tcgen05 flash forward (head_dim 128)
    b, s, h, n_q, n_kv, hd, p = 2, 150, 256, 4, 2, 128, 2
    inp = inputs.attn_inputs(b, s, h, n_q, n_kv, hd, "bf16", seed=44, w_std=0.05)
    a = Attn(lib, inp, p, "bf16", True, n_q=n_q, n_kv=n_kv, hd=hd)
    res = inputs.normal((b, s, h), 1.0, 44, 99, "bf16", "cpu").to(dev())
    y = torch.empty(b, s, h, dtype=torch.bfloat16, device=dev())
    yn = torch.empty_like(y)
    lib.tp_attn_fwd(a.desc, inp["x"].to(dev()), a.wqkv, a.wo, y, residual=res, workspace=a.ws,
                    y_norm=yn)
    T = b * s
    xs = _split(inp["x"].to(dev()).reshape(T, h), p)
    ys = [torch.empty(T // p, h, dtype=torch.bfloat16, device=dev()) for _ in range(p)]
    yns = [torch.empty_like(ys[0]) for _ in range(p)]
    ws = torch.empty(lib.tp_attn_fwd_sp_workspace(a.desc), dtype=torch.uint8, device=dev())
    lib.tp_reset_reduction_count()
    lib.tp_attn_fwd_sp(a.desc, xs, a.wqkv, a.wo, ys, residual_slices=_split(res.reshape(T, h), p),
                       y_norm_slices=yns, workspace=ws)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    assert torch.equal(torch.cat(ys), y.reshape(T, h))
    assert torch.equal(torch.cat(yns), yn.reshape(T, h))
    ref = oattn.attention_forward(*(f64(inp[k]) for k in ("x", "wq", "wk", "wv", "wo")),
                                  n_q, n_kv, hd, causal=True).reshape(T, h) + f64(res.cpu()).reshape(T, h)
    for i, rows in enumerate(osp.token_slices(T, p)):
        assert rel_l2(f64(ys[i]), ref[rows]) <= TOL["bf16"], i


def test_attention_backward_sp(lib):
    # x and dy as 2 slices of 150 token rows, dx out as slices: equal to tp_attn_bwd's rows bit for
    # bit (the same shard-order fp32 sum and rounding), and to the oracle; the weight gradients
    # equal tp_attn_bwd's
    b, s, h, n_q, n_kv, hd, p = 2, 150, 256, 4, 2, 128, 2
    inp = inputs.attn_inputs(b, s, h, n_q, n_kv, hd, "bf16", seed=45, w_std=0.05)
    a = Attn(lib, inp, p, "bf16", True, n_q=n_q, n_kv=n_kv, hd=hd)
    dy = inputs.normal((b, s, h), 1.0, 45, 97, "bf16", "cpu").to(dev())
    g = dev()
    dx = torch.empty(b, s, h, dtype=torch.bfloat16, device=g)
    dwqkv = torch.empty(a.wqkv.numel(), dtype=torch.float32, device=g)
    dwo = torch.empty(a.wo.numel(), dtype=torch.float32, device=g)
    ws = torch.empty(lib.tp_attn_bwd_workspace(a.desc), dtype=torch.uint8, device=g)
    lib.tp_attn_bwd(a.desc, inp["x"].to(g), a.wqkv, a.wo, dy, dx, dwqkv, dwo, workspace=ws)
    T = b * s
    xs = _split(inp["x"].to(g).reshape(T, h), p)
    dys = _split(dy.reshape(T, h), p)
    dxs = [torch.empty(T // p, h, dtype=torch.bfloat16, device=g) for _ in range(p)]
    dwqkv_sp = torch.empty_like(dwqkv)
    dwo_sp = torch.empty_like(dwo)
    ws_sp = torch.empty(lib.tp_attn_bwd_sp_workspace(a.desc), dtype=torch.uint8, device=g)
    lib.tp_reset_reduction_count()
    lib.tp_attn_bwd_sp(a.desc, xs, a.wqkv, a.wo, dys, dxs, dwqkv_sp, dwo_sp, workspace=ws_sp)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    assert torch.equal(torch.cat(dxs), dx.reshape(T, h))
    assert torch.equal(dwqkv_sp, dwqkv) and torch.equal(dwo_sp, dwo)
    ref = oattn.attention_backward(*(f64(inp[k]) for k in ("x", "wq", "wk", "wv", "wo")),
                                   f64(dy.cpu()), n_q, n_kv, hd, causal=True)[0].reshape(T, h)
    for i, rows in enumerate(osp.token_slices(T, p)):
        assert rel_l2(f64(dxs[i]), ref[rows]) <= TOL["bf16"], i
    # fused reduce mode and ragged token counts are refused
    fused = lib.attn_desc(b, s, h, n_q, n_kv, hd, p, reduce_mode=lib.TP_REDUCE_FUSED)
    assert lib.tp_attn_bwd_sp_workspace(fused) == 0
    assert lib.tp_attn_bwd_sp_workspace(lib.attn_desc(1, 5, h, n_q, n_kv, hd, p)) == 0
