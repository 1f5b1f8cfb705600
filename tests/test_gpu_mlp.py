"""MLP block on the GPU through the C ABI, element by element against the float64 oracle.

Tolerance (rel-L2 of each output tensor): 2e-2 for bf16, 1e-5 for fp32.
"""

import numpy as np
import pytest
import torch

from oracle import mlp as omlp
from tensor_transformer_matmul_b200 import inputs
from tests.helpers import TOL, Mlp, dev, f64, rel_l2, rel_l2_rows

pytestmark = pytest.mark.gpu


def _oracle_fwd(inp, act):
    wu = None if inp["w_up"] is None else f64(inp["w_up"])
    return omlp.mlp_forward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), act, wu)


def test_tiny_config_fp32(lib):
    # T=4 tokens, d=8, d_ff=32, p=4 logical shards, GELU, fp32; W ~ N(0, 1/sqrt(fan_in)), seed 0
    inp = inputs.mlp_inputs(4, 8, 32, "gelu", "f32", seed=0)
    m = Mlp(lib, inp, 4, "gelu", "f32")
    lib.tp_reset_reduction_count()
    y = m.forward(inp["x"])
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    ref = _oracle_fwd(inp, "gelu")
    assert rel_l2(f64(y), ref) <= TOL["f32"]
    # the sharded sum equals the unsharded result for every p dividing d_ff
    for p in (1, 2, 8, 16, 32):
        mp = Mlp(lib, inp, p, "gelu", "f32")
        assert rel_l2(f64(mp.forward(inp["x"])), ref) <= TOL["f32"], p


@pytest.mark.parametrize("reduce_mode", [0, 1])
@pytest.mark.parametrize("act", ["swiglu", "gelu", "relu", "identity"])
@pytest.mark.parametrize("T", [1, 17, 64, 100, 200, 300])
def test_bf16_forward_parity(lib, act, T, reduce_mode):
    # several tiles and ragged tails in every dimension: d = 328 (5 K-blocks + 8), F_s = 136
    # (padded to 256 per shard), p = 3 (not a power of two, as in the h=2/d_ff=3 worked example);
    # T <= 128 runs the stream-K decode schedule, reduce_mode 1 fuses the shard reduce into it
    d, F, p = 328, 408, 3
    inp = inputs.mlp_inputs(T, d, F, act, "bf16", seed=1, w_std=0.05)
    m = Mlp(lib, inp, p, act, "bf16", reduce_mode)
    y = m.forward(inp["x"])
    torch.cuda.synchronize()
    assert rel_l2(f64(y), _oracle_fwd(inp, act)) <= TOL["bf16"]


def test_bf16_residual_and_saved(lib):
    T, d, F, p = 150, 256, 1024, 4
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=2, w_std=0.05)
    m = Mlp(lib, inp, p, "swiglu", "bf16")
    res = inputs.normal((T, d), 1.0, 2, 99, "bf16", "cpu").to(dev())
    y = m.forward(inp["x"], residual=res)
    torch.cuda.synchronize()
    ref = _oracle_fwd(inp, "swiglu") + f64(res)
    assert rel_l2(f64(y), ref) <= TOL["bf16"]
    # residual may alias the output
    y2 = res.clone()
    m.lib.tp_mlp_fwd(m.desc, inp["x"].to(dev()), m.w1p, m.w2p, y2, residual=y2, workspace=m.ws_f)
    torch.cuda.synchronize()
    assert rel_l2(f64(y2), ref) <= TOL["bf16"]


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
@pytest.mark.parametrize("dtype,T", [("bf16", 200), ("bf16", 37), ("f32", 9)])
def test_backward_parity(lib, act, dtype, T):
    d, F, p = (328, 408, 3) if dtype == "bf16" else (24, 48, 4)
    inp = inputs.mlp_inputs(T, d, F, act, dtype, seed=3, w_std=0.05, backward=True)
    m = Mlp(lib, inp, p, act, dtype)
    lib.tp_reset_reduction_count()
    m.forward(inp["x"])
    dx, dw1, dwu, dw2, dw1p, _ = m.backward(inp["dy"], inp["x"])
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 2   # one forward, one backward
    wu = None if inp["w_up"] is None else f64(inp["w_up"])
    ref = omlp.mlp_backward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), f64(inp["dy"]), act, wu)
    tol = TOL[dtype]
    assert rel_l2(f64(dx), ref["dx"]) <= tol
    assert rel_l2(f64(dw1), ref["dw1"]) <= tol
    assert rel_l2(f64(dw2), ref["dw2"]) <= tol
    if act == "swiglu":
        assert rel_l2(f64(dwu), ref["dw_up"]) <= tol


@pytest.mark.parametrize("reduce_mode", [0, 1])
@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_pair_tiles_forward_backward(lib, act, reduce_mode):
    # the prefill and backward GEMMs run 256 x 256 tiles on SM pairs: T = 520 gives three token
    # tiles (the last one ragged, its second half empty), d = 776 a ragged K and N, F_s = 512 two
    # feature tiles per shard; every GEMM of forward and backward has several tiles per dimension.
    # reduce_mode 1 sums the shards of the down and dx GEMMs in their accumulators.
    T, d, F, p = 520, 776, 1536, 3
    inp = inputs.mlp_inputs(T, d, F, act, "bf16", seed=11, w_std=0.05, backward=True)
    m = Mlp(lib, inp, p, act, "bf16", reduce_mode)
    lib.tp_reset_reduction_count()
    y = m.forward(inp["x"])
    dx, dw1, dwu, dw2, _, _ = m.backward(inp["dy"], inp["x"])
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 2
    wu = None if inp["w_up"] is None else f64(inp["w_up"])
    assert rel_l2(f64(y), _oracle_fwd(inp, act)) <= TOL["bf16"]
    ref = omlp.mlp_backward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), f64(inp["dy"]), act, wu)
    assert rel_l2(f64(dx), ref["dx"]) <= TOL["bf16"]
    assert rel_l2(f64(dw1), ref["dw1"]) <= TOL["bf16"]
    assert rel_l2(f64(dw2), ref["dw2"]) <= TOL["bf16"]
    if act == "swiglu":
        assert rel_l2(f64(dwu), ref["dw_up"]) <= TOL["bf16"]


def test_backward_padding_gradients_are_zero(lib):
    # F_s = 136 pads to 256 per shard: the padding rows of the packed gradient must be exactly 0
    d, F, p, T = 64, 408, 3, 40
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=4, w_std=0.05, backward=True)
    m = Mlp(lib, inp, p, "swiglu", "bf16")
    m.forward(inp["x"])
    _, _, _, _, dw1p, dw2p = m.backward(inp["dy"], inp["x"])
    torch.cuda.synchronize()
    g1 = dw1p.view(p, 2, 256, d)         # [shard][block][gate|up rows][d]
    g2 = dw2p.view(p, d, 256)
    # block 1 holds features 128..255 (gate rows 0..127, up rows 128..255); 136.. are padding
    pad = np.concatenate([f64(g1[:, 1, 8:128]), f64(g1[:, 1, 136:256])], axis=1)
    assert np.count_nonzero(pad) == 0
    assert np.count_nonzero(np.asarray(f64(g2[:, :, 136:]))) == 0


def test_empty_batch(lib):
    inp = inputs.mlp_inputs(0, 64, 256, "swiglu", "bf16", seed=5, backward=True)
    desc = lib.mlp_desc(0, 64, 256, 2, "swiglu", "bf16")
    w1p = torch.full((lib.tp_mlp_w1_packed_bytes(desc) // 2,), 1.0, dtype=torch.bfloat16, device=dev())
    w2p = torch.full((lib.tp_mlp_w2_packed_bytes(desc) // 2,), 1.0, dtype=torch.bfloat16, device=dev())
    y = torch.empty(0, 64, dtype=torch.bfloat16, device=dev())
    lib.tp_mlp_fwd(desc, inp["x"].to(dev()), w1p, w2p, y)
    dw1p = torch.full((w1p.numel(),), 7.0, device=dev())
    dw2p = torch.full((w2p.numel(),), 7.0, device=dev())
    dx = torch.empty(0, 64, dtype=torch.bfloat16, device=dev())
    lib.tp_mlp_bwd(desc, inp["dy"].to(dev()), inp["x"].to(dev()), None, w1p, w2p, dx, dw1p, dw2p)
    torch.cuda.synchronize()
    assert float(dw1p.abs().sum()) == 0.0 and float(dw2p.abs().sum()) == 0.0


def test_deterministic(lib):
    # fixed-order reduction: two runs give identical bytes
    inp = inputs.mlp_inputs(130, 256, 1024, "swiglu", "bf16", seed=6, w_std=0.05)
    m = Mlp(lib, inp, 8, "swiglu", "bf16")
    a = m.forward(inp["x"]).clone()
    b = m.forward(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_full_size_decode_mlp(lib):
    # T=64 (batch 64, s=1), d=8192, d_ff=28672, p=8, bf16 x ~ N(0,1), W ~ N(0, 0.02): every row
    # against the oracle, whole tensor and row by row
    T, d, F, p = 64, 8192, 28672, 8
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=0, device="cuda", w_std=0.02)
    m = Mlp(lib, inp, p, "swiglu", "bf16")
    y = m.forward(inp["x"], save=False)
    torch.cuda.synchronize()
    ref = omlp.mlp_forward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), "swiglu",
                           f64(inp["w_up"]))
    assert rel_l2(f64(y), ref) <= TOL["bf16"]
    assert rel_l2_rows(f64(y), ref) <= TOL["bf16"]


def _one_per_block(n, block, salt):
    """One index in every ``block``-wide block of range(n), at a different offset in each."""
    return [b * block + (salt * (b + 1) * 37) % min(block, n - b * block)
            for b in range((n + block - 1) // block)]


@pytest.mark.parametrize("mode", [0, 1])
def test_full_size_prefill_mlp_sampled(lib, mode):
    # T=4096 (b=1, s=4096), d=8192, d_ff=28672, p=8: one row of y and dx in every 256-row tile
    # (the SM-pair GEMM's token tile), and one hidden feature of every shard for the dWg / dWu
    # columns and the dW2 row, each computed by the oracle over its full contraction and checked
    # as a whole and row by row (column by column for dW1); mode 1 adds the 8 shard partials of
    # y and of dx inside the GEMM accumulators
    T, d, F, p = 4096, 8192, 28672, 8
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=0, device="cuda", w_std=0.02,
                            backward=True)
    m = Mlp(lib, inp, p, "swiglu", "bf16", mode)
    y = m.forward(inp["x"])
    dx, dw1, dwu, dw2, _, _ = m.backward(inp["dy"], inp["x"])
    torch.cuda.synchronize()
    x, wg, wu, w2, dy = (f64(inp[k]) for k in ("x", "w1", "w_up", "w2", "dy"))
    rows = _one_per_block(T, 256, 3)
    cols = _one_per_block(F, F // p, 5)        # one feature per shard
    w2rows = _one_per_block(F, F // p, 7)
    ref_y = omlp.mlp_forward_rows(x, wg, w2, "swiglu", rows, wu)
    got_y = f64(y)[rows]
    assert rel_l2(got_y, ref_y) <= TOL["bf16"] and rel_l2_rows(got_y, ref_y) <= TOL["bf16"]
    s = omlp.mlp_backward_samples(x, wg, w2, dy, "swiglu", rows, cols, w2rows, wu)
    checks = ((f64(dx)[rows], s["dx"]),
              (f64(dw1)[:, cols].T, s["dw1_cols"].T),
              (f64(dwu)[:, cols].T, s["dw_up_cols"].T),
              (f64(dw2)[w2rows], s["dw2_rows"]))
    for got, ref in checks:
        assert rel_l2(got, ref) <= TOL["bf16"]
        assert rel_l2_rows(got, ref) <= TOL["bf16"]


def test_f32_residual_stream(lib):
    # TP_FLAG_F32_RESIDUAL: bf16 inputs and weights, float32 residual and output
    T, d, F, p = 33, 256, 1024, 4
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=7, w_std=0.05)
    m = Mlp(lib, inp, p, "swiglu", "bf16")
    desc = lib.mlp_desc(T, d, F, p, "swiglu", "bf16", flags=lib.TP_FLAG_F32_RESIDUAL)
    res = torch.randn(T, d, device=dev())
    y = torch.empty(T, d, device=dev())
    lib.tp_mlp_fwd(desc, inp["x"].to(dev()), m.w1p, m.w2p, y, residual=res, workspace=m.ws_f)
    torch.cuda.synchronize()
    assert y.dtype == torch.float32
    assert rel_l2(f64(y), _oracle_fwd(inp, "swiglu") + f64(res)) <= TOL["bf16"]


@pytest.mark.parametrize("T,d,F,p", [(64, 2048, 8192, 8), (16, 4096, 4096, 4), (128, 1024, 16384, 16),
                                     (1, 8192, 3584, 8)])
def test_stream_k_splits_fused_vs_separate(lib, T, d, F, p):
    # decode shapes whose k-blocks split tiles across CTAs at many different points; the fused
    # reduce (shards added inside the GEMM) and the separate reduce both match the oracle
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=8, w_std=0.02)
    ref = _oracle_fwd(inp, "swiglu")
    outs = []
    for mode in (0, 1):
        m = Mlp(lib, inp, p, "swiglu", "bf16", mode)
        lib.tp_reset_reduction_count()
        outs.append(m.forward(inp["x"], save=False))
        torch.cuda.synchronize()
        assert lib.tp_reduction_count() == 1
        assert rel_l2(f64(outs[-1]), ref) <= TOL["bf16"]
    assert rel_l2(f64(outs[0]), f64(outs[1])) <= 1e-2


@pytest.mark.parametrize("T,d,F,p,act", [
    (2, 5568, 14336, 7, "gelu"),     # 87 k-blocks per up tile (two per stage, one left over), a
                                     # ragged last block of 64 output rows, 7 shards
    (3, 2048, 19072, 1, "swiglu"),   # one shard, 149 up tiles of 256 packed rows
    (5, 4096, 22400, 5, "swiglu"),   # 175 up tiles, 160 down tiles
    (40, 1024, 3072, 3, "relu"),     # 64-token tiles, three shards
])
def test_decode_one_launch_shapes(lib, T, d, F, p, act):
    # the one-launch decode MLP (up tiles, then down tiles taken from a device counter once their
    # shard's h is complete): checked against the oracle row by row, and two runs give the same
    # bits
    inp = inputs.mlp_inputs(T, d, F, act, "bf16", seed=11 + T, w_std=0.03)
    m = Mlp(lib, inp, p, act, "bf16", 0)
    a = m.forward(inp["x"], save=False).clone()
    b = m.forward(inp["x"], save=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    ref = _oracle_fwd(inp, act)
    assert rel_l2(f64(a), ref) <= TOL["bf16"] and rel_l2_rows(f64(a), ref) <= TOL["bf16"]


def test_fused_reduce_deterministic(lib):
    inp = inputs.mlp_inputs(64, 1024, 4096, "swiglu", "bf16", seed=9, w_std=0.02)
    m = Mlp(lib, inp, 8, "swiglu", "bf16", 1)
    a = m.forward(inp["x"], save=False).clone()
    b = m.forward(inp["x"], save=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("reduce_mode", [0, 1])
@pytest.mark.parametrize("T", [1, 150])
def test_y_norm_output(lib, reduce_mode, T):
    # the reduction also writes RMSNorm(y): the replicated normalization after the residual add
    from oracle import decode as odec
    d, F, p = 256, 1024, 4
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=10, w_std=0.05)
    m = Mlp(lib, inp, p, "swiglu", "bf16", reduce_mode)
    res = inputs.normal((T, d), 1.0, 10, 99, "bf16", "cpu").to(dev())
    y = torch.empty(T, d, dtype=torch.bfloat16, device=dev())
    yn = torch.empty_like(y)
    lib.tp_mlp_fwd(m.desc, inp["x"].to(dev()), m.w1p, m.w2p, y, residual=res, workspace=m.ws_f,
                   y_norm=yn)
    torch.cuda.synchronize()
    ref = _oracle_fwd(inp, "swiglu") + f64(res)
    assert rel_l2(f64(y), ref) <= TOL["bf16"]
    assert rel_l2(f64(yn), odec.rmsnorm(ref)) <= TOL["bf16"]


@pytest.mark.parametrize("reduce_mode", [0, 1])
@pytest.mark.parametrize("act", ["swiglu", "gelu", "relu", "identity"])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_few_tokens_decode_path(lib, act, T, reduce_mode):
    # 1..4 tokens (the decode stack's batch sizes) on the swapped decode tiles, both reduce modes:
    # d = 512, d_ff = 1536 over p = 3 (512 features per shard), residual and RMSNorm output
    from oracle import decode as odec
    d, F, p = 512, 1536, 3
    inp = inputs.mlp_inputs(T, d, F, act, "bf16", seed=30 + T, w_std=0.05, backward=True)
    m = Mlp(lib, inp, p, act, "bf16", reduce_mode)
    res = inputs.normal((T, d), 1.0, 30, 99, "bf16", "cpu").to(dev())
    y = torch.empty(T, d, dtype=torch.bfloat16, device=dev())
    yn = torch.empty_like(y)
    lib.tp_reset_reduction_count()
    lib.tp_mlp_fwd(m.desc, inp["x"].to(dev()), m.w1p, m.w2p, y, residual=res, saved=m.saved,
                   workspace=m.ws_f, y_norm=yn)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    ref = _oracle_fwd(inp, act) + f64(res)
    assert rel_l2(f64(y), ref) <= TOL["bf16"] and rel_l2_rows(f64(y), ref) <= TOL["bf16"]
    assert rel_l2(f64(yn), odec.rmsnorm(ref)) <= TOL["bf16"]
    # the saved pre-activations feed the backward pass
    dx, dw1, dwu, dw2, _, _ = m.backward(inp["dy"], inp["x"])
    torch.cuda.synchronize()
    wu = None if inp["w_up"] is None else f64(inp["w_up"])
    rb = omlp.mlp_backward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), f64(inp["dy"]), act, wu)
    assert rel_l2(f64(dx), rb["dx"]) <= TOL["bf16"]
    assert rel_l2(f64(dw2), rb["dw2"]) <= TOL["bf16"]
    # deterministic: a second call gives the same bytes
    y2 = torch.empty_like(y)
    lib.tp_mlp_fwd(m.desc, inp["x"].to(dev()), m.w1p, m.w2p, y2, residual=res, workspace=m.ws_f)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


def test_decode_full_size_one_token(lib):
    # the decode stack's MLP shape at b = 1: d=8192, d_ff=28672, p=8, one token
    T, d, F, p = 1, 8192, 28672, 8
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=0, device="cuda", w_std=0.02)
    m = Mlp(lib, inp, p, "swiglu", "bf16")
    y = m.forward(inp["x"], save=False)
    torch.cuda.synchronize()
    ref = omlp.mlp_forward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), "swiglu",
                           f64(inp["w_up"]))
    assert rel_l2(f64(y), ref) <= TOL["bf16"]
