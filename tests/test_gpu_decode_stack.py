"""The decode layer stack (pre-RMSNorm, TP attention + residual, pre-RMSNorm, TP SwiGLU MLP +
residual, per layer) through the C ABI against the float64 oracle decode stack."""

import numpy as np
import pytest
import torch

from oracle import decode as odec
from tensor_transformer_matmul_b200 import inputs
from tensor_transformer_matmul_b200.decode_stack import DecodeStack
from tests.helpers import TOL, dev, f64, rel_l2

pytestmark = pytest.mark.gpu


def _oracle_stack(cfg, x0, caches, device):
    """Run the oracle over the same seeded per-layer weights, drawn again on ``device``."""
    n_q, n_kv, hd = cfg["n_q"], cfg["n_kv"], cfg["hd"]

    def weights(l):
        if l >= cfg["layers"]:
            return None
        a = inputs.attn_inputs(cfg["b"], 1, cfg["h"], n_q, n_kv, hd, "bf16", seed=cfg["seed"],
                               device=device, w_std=0.02, kv_len=cfg["kv_len"], layer=l)
        m = inputs.mlp_inputs(cfg["b"], cfg["h"], cfg["F"], "swiglu", "bf16", seed=cfg["seed"],
                              device=device, w_std=0.02, layer=l)
        return {"wq": f64(a["wq"]), "wk": f64(a["wk"]), "wv": f64(a["wv"]), "wo": f64(a["wo"]),
                "wg": f64(m["w1"]), "wu": f64(m["w_up"]), "w2": f64(m["w2"])}

    return odec.decode_stack(x0, weights, lambda l: caches[l], n_q, n_kv, hd)


def _run(cfg, device, graph=False):
    st = DecodeStack(cfg["layers"], cfg["h"], cfg["F"], cfg["n_q"], cfg["n_kv"], cfg["hd"],
                     cfg["p"], cfg["kv_len"], b=cfg["b"], seed=cfg["seed"], device=dev())
    caches = [(f64(l["k_cache"])[:, :, :cfg["kv_len"]], f64(l["v_cache"])[:, :, :cfg["kv_len"]])
              for l in st.layers]
    x0 = inputs.normal((cfg["b"], 1, cfg["h"]), 1.0, cfg["seed"], 97, "bf16", "cpu")
    x = x0.to(dev()).float()   # float32 residual stream
    return st, caches, x0, x


@pytest.mark.parametrize("graph", [False, True])
def test_small_stack(lib, graph):
    cfg = dict(layers=3, b=2, h=512, F=1536, n_q=8, n_kv=2, hd=64, p=2, kv_len=300, seed=3)
    st, caches, x0, x = _run(cfg, dev())
    lib.tp_reset_reduction_count()
    if graph:
        xg = x.clone()
        st.capture(xg)           # runs one eager warm-up step, then records the next
        x_eager_once = xg.clone()
        xg.copy_(x)
        st.replay()
        torch.cuda.synchronize()
        out = xg
        assert torch.equal(out, x_eager_once) or rel_l2(f64(out), f64(x_eager_once)) <= TOL["bf16"]
    else:
        out = st.step(x)
        torch.cuda.synchronize()
        assert lib.tp_reduction_count() == 2 * cfg["layers"]   # 2 reductions per decoded layer
    ref, _ = _oracle_stack(cfg, f64(x0)[:, 0], caches, dev())
    assert rel_l2(f64(out)[:, 0], ref) <= TOL["bf16"]


def test_full_size_stack(lib):
    # 16 Llama-70B-shaped layers: h=8192, d_ff=28672, 64 Q / 8 KV heads, hd=128, p=8,
    # b=1, s=1, KV length 4096; 2 reductions of 1 x 8192 per layer
    cfg = dict(layers=16, b=1, h=8192, F=28672, n_q=64, n_kv=8, hd=128, p=8, kv_len=4096, seed=0)
    st, caches, x0, x = _run(cfg, dev())
    lib.tp_reset_reduction_count()
    out = st.step(x)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 32
    del st
    torch.cuda.empty_cache()
    ref, _ = _oracle_stack(cfg, f64(x0)[:, 0], caches, dev())
    assert rel_l2(f64(out)[:, 0], ref) <= TOL["bf16"]
