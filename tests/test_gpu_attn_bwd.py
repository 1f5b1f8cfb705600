"""Attention block backward on the GPU through the C ABI, against the float64 oracle.

Tolerance: rel-L2 <= 2e-2 per gradient tensor (bf16 inputs and intermediates, fp32 sums).
"""
import numpy as np
import pytest
import torch

from oracle import attention as oattn
from tensor_transformer_matmul_b200 import inputs
from tests.helpers import TOL, Attn, dev, f64, rel_l2

pytestmark = pytest.mark.gpu


def _grads_ref(inp, dy, n_q, n_kv, hd, causal):
    return oattn.attention_backward(f64(inp["x"]), f64(inp["wq"]), f64(inp["wk"]), f64(inp["wv"]),
                                    f64(inp["wo"]), f64(dy), n_q, n_kv, hd, causal)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("b,s,h,n_q,n_kv,hd,p", [
    (2, 37, 256, 8, 2, 32, 2),      # ragged sequence, 4 query heads per KV head, SIMT forward
    (1, 130, 192, 4, 4, 64, 4),     # MHA, flash forward (head_dim 64), two query tiles
    (1, 200, 512, 8, 2, 128, 1),    # one shard, flash forward (head_dim 128), 200 tokens
    (3, 9, 64, 8, 8, 8, 8),         # tiny head_dim, p = n_kv
    (2, 150, 256, 4, 2, 128, 2),    # tcgen05 backward, two sequences, ragged second block
    (3, 70, 256, 8, 2, 64, 1),      # tcgen05 backward (head_dim 64), three short sequences
])
def test_backward_parity(lib, causal, b, s, h, n_q, n_kv, hd, p):
    inp = inputs.attn_inputs(b, s, h, n_q, n_kv, hd, "bf16", seed=31, w_std=0.05)
    dy = inputs.normal((b, s, h), 1.0, 31, 97, "bf16", "cpu")
    a = Attn(lib, inp, p, "bf16", causal, n_q=n_q, n_kv=n_kv, hd=hd)
    lib.tp_reset_reduction_count()
    got = a.backward(inp["x"], dy)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    ref = _grads_ref(inp, dy, n_q, n_kv, hd, causal)
    names = ("dx", "dwq", "dwk", "dwv", "dwo")
    for name, g, r in zip(names, got, ref):
        err = rel_l2(f64(g), r)
        assert err <= TOL["bf16"], (name, err)


@pytest.mark.parametrize("b,s,h,n_q,n_kv,hd,p", [
    (2, 37, 256, 8, 2, 32, 2),
    (2, 150, 264, 4, 2, 128, 2),    # h = 264: ragged K of the dx GEMM's second shard tile
])
def test_backward_fused_dx(lib, b, s, h, n_q, n_kv, hd, p):
    # TP_REDUCE_FUSED: the dx GEMM adds the shards in its accumulator and writes dx directly
    inp = inputs.attn_inputs(b, s, h, n_q, n_kv, hd, "bf16", seed=35, w_std=0.05)
    dy = inputs.normal((b, s, h), 1.0, 35, 97, "bf16", "cpu")
    a = Attn(lib, inp, p, "bf16", True, n_q=n_q, n_kv=n_kv, hd=hd, reduce_mode=1)
    lib.tp_reset_reduction_count()
    got = a.backward(inp["x"], dy)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    ref = _grads_ref(inp, dy, n_q, n_kv, hd, True)
    for name, g, r in zip(("dx", "dwq", "dwk", "dwv", "dwo"), got, ref):
        err = rel_l2(f64(g), r)
        assert err <= TOL["bf16"], (name, err)


def test_backward_deterministic(lib):
    inp = inputs.attn_inputs(1, 100, 256, 8, 2, 64, "bf16", seed=32, w_std=0.05)
    dy = inputs.normal((1, 100, 256), 1.0, 32, 97, "bf16", "cpu")
    a = Attn(lib, inp, 2, "bf16", True, n_q=8, n_kv=2, hd=64)
    g1 = a.backward(inp["x"], dy)
    g2 = a.backward(inp["x"], dy)
    torch.cuda.synchronize()
    for u, v in zip(g1, g2):
        assert torch.equal(u, v)


def test_backward_rejects_unsupported(lib):
    inp = inputs.attn_inputs(1, 1, 64, 4, 2, 16, "bf16", seed=33, w_std=0.05, kv_len=5)
    a = Attn(lib, inp, 2, "bf16", True, kv_len=5, n_q=4, n_kv=2, hd=16)
    assert lib.tp_attn_bwd_workspace(a.desc) == 0      # decode has no backward
    with pytest.raises(lib.TpError):
        a.backward(inp["x"], torch.zeros(1, 1, 64, dtype=torch.bfloat16))


def test_backward_llama_heads(lib):
    # the full head structure of the attention configuration (h=8192, 64 query / 8 KV heads,
    # head_dim 128, p=8) at 512 tokens: four query tiles of the flash forward, every shard
    inp = inputs.attn_inputs(1, 512, 8192, 64, 8, 128, "bf16", seed=34, w_std=0.02)
    dy = inputs.normal((1, 512, 8192), 1.0, 34, 97, "bf16", "cpu")
    a = Attn(lib, inp, 8, "bf16", True, n_q=64, n_kv=8, hd=128)
    got = a.backward(inp["x"], dy)
    torch.cuda.synchronize()
    ref = _grads_ref(inp, dy, 64, 8, 128, True)
    for name, g, r in zip(("dx", "dwq", "dwk", "dwv", "dwo"), got, ref):
        err = rel_l2(f64(g), r)
        assert err <= TOL["bf16"], (name, err)
