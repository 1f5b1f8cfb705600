"""Shared test plumbing: run the library's calls on seeded inputs and compare with the oracle."""

import numpy as np
import torch

from tensor_transformer_matmul_b200 import inputs

# parity tolerances: rel-L2 <= 2e-2 for bf16, <= 1e-5 for fp32
TOL = {"bf16": 2e-2, "f32": 1e-5}


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def rel_l2_rows(got, ref):
    """The largest rel-L2 over the rows (the last axis) of got against ref: a wrong tile or a
    wrong shard's block shows up in its own rows even when the whole-tensor norm hides it."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    g = got.reshape(-1, got.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    num = np.linalg.norm(g - r, axis=1)
    den = np.maximum(np.linalg.norm(r, axis=1), 1e-300)
    return float((num / den).max()) if len(r) else 0.0


def f64(t):
    return inputs.to_f64(t)


def dev():
    return torch.device("cuda", 0)


class Mlp:
    """Packs one MLP block's weights with the library and runs forward / backward."""

    def __init__(self, lib, inp, p, act, dtype, reduce_mode=0):
        self.lib = lib
        x, w1, wu, w2 = inp["x"], inp["w1"], inp["w_up"], inp["w2"]
        self.T, self.d = x.shape
        self.F = w1.shape[1]
        self.dtype, self.act = dtype, act
        self.desc = lib.mlp_desc(self.T, self.d, self.F, p, act, dtype, reduce_mode)
        tdt = inputs.TORCH_DTYPE[dtype]
        g = dev()
        self.w1p = torch.empty(lib.tp_mlp_w1_packed_bytes(self.desc) // (2 if dtype == "bf16" else 4),
                               dtype=tdt, device=g)
        self.w2p = torch.empty(lib.tp_mlp_w2_packed_bytes(self.desc) // (2 if dtype == "bf16" else 4),
                               dtype=tdt, device=g)
        lib.tp_mlp_pack(self.desc, w1.to(g), None if wu is None else wu.to(g), w2.to(g), self.w1p, self.w2p)
        self.ws_f = torch.empty(lib.tp_mlp_fwd_workspace(self.desc), dtype=torch.uint8, device=g)
        self.ws_b = torch.empty(lib.tp_mlp_bwd_workspace(self.desc), dtype=torch.uint8, device=g)
        self.saved = torch.empty(lib.tp_mlp_saved_bytes(self.desc), dtype=torch.uint8, device=g)

    def forward(self, x, residual=None, save=True):
        y = torch.empty(self.T, self.d, dtype=inputs.TORCH_DTYPE[self.dtype], device=dev())
        self.lib.tp_mlp_fwd(self.desc, x.to(dev()), self.w1p, self.w2p, y, residual=residual,
                            saved=self.saved if save else None, workspace=self.ws_f)
        return y

    def backward(self, dy, x):
        g = dev()
        dx = torch.empty(self.T, self.d, dtype=inputs.TORCH_DTYPE[self.dtype], device=g)
        dw1p = torch.empty(self.lib.tp_mlp_w1_packed_bytes(self.desc) // (2 if self.dtype == "bf16" else 4),
                           dtype=torch.float32, device=g)
        dw2p = torch.empty(self.lib.tp_mlp_w2_packed_bytes(self.desc) // (2 if self.dtype == "bf16" else 4),
                           dtype=torch.float32, device=g)
        self.lib.tp_mlp_bwd(self.desc, dy.to(g), x.to(g), self.saved, self.w1p, self.w2p, dx,
                            dw1p, dw2p, workspace=self.ws_b)
        dw1 = torch.empty(self.d, self.F, dtype=torch.float32, device=g)
        dwu = torch.empty(self.d, self.F, dtype=torch.float32, device=g) if self.act == "swiglu" else None
        dw2 = torch.empty(self.F, self.d, dtype=torch.float32, device=g)
        self.lib.tp_mlp_unpack_grads(self.desc, dw1p, dw2p, dw1, dwu, dw2)
        return dx, dw1, dwu, dw2, dw1p, dw2p


class Attn:
    """Packs one attention block's weights with the library and runs tp_attn_fwd."""

    def __init__(self, lib, inp, p, dtype, causal=True, kv_len=0, n_q=None, n_kv=None, hd=None,
                 reduce_mode=0):
        self.lib = lib
        x = inp["x"]
        self.b, self.s, self.h = x.shape
        self.n_q, self.n_kv, self.hd = n_q, n_kv, hd
        self.dtype = dtype
        self.desc = lib.attn_desc(self.b, self.s, self.h, n_q, n_kv, hd, p, causal, dtype, kv_len,
                                  reduce_mode=reduce_mode)
        tdt = inputs.TORCH_DTYPE[dtype]
        eb = 2 if dtype == "bf16" else 4
        g = dev()
        self.wqkv = torch.empty(lib.tp_attn_wqkv_packed_bytes(self.desc) // eb, dtype=tdt, device=g)
        self.wo = torch.empty(lib.tp_attn_wo_packed_bytes(self.desc) // eb, dtype=tdt, device=g)
        lib.tp_attn_pack(self.desc, inp["wq"].to(g), inp["wk"].to(g), inp["wv"].to(g),
                         inp["wo"].to(g), self.wqkv, self.wo)
        self.ws = torch.empty(lib.tp_attn_fwd_workspace(self.desc), dtype=torch.uint8, device=g)

    def forward(self, x, k_cache=None, v_cache=None, residual=None):
        y = torch.empty(self.b, self.s, self.h, dtype=inputs.TORCH_DTYPE[self.dtype], device=dev())
        self.lib.tp_attn_fwd(self.desc, x.to(dev()), self.wqkv, self.wo, y, k_cache=k_cache,
                             v_cache=v_cache, residual=residual, workspace=self.ws)
        return y

    def backward(self, x, dy):
        """tp_attn_bwd; returns dx and the unpacked fp32 weight gradients dwq, dwk, dwv, dwo."""
        g = dev()
        lib = self.lib
        dx = torch.empty(self.b, self.s, self.h, dtype=inputs.TORCH_DTYPE[self.dtype], device=g)
        dwqkv_p = torch.empty(self.wqkv.numel(), dtype=torch.float32, device=g)
        dwo_p = torch.empty(self.wo.numel(), dtype=torch.float32, device=g)
        ws = torch.empty(lib.tp_attn_bwd_workspace(self.desc), dtype=torch.uint8, device=g)
        lib.tp_attn_bwd(self.desc, x.to(g), self.wqkv, self.wo, dy.to(g), dx, dwqkv_p, dwo_p,
                        workspace=ws)
        dwq = torch.empty(self.h, self.n_q * self.hd, dtype=torch.float32, device=g)
        dwk = torch.empty(self.h, self.n_kv * self.hd, dtype=torch.float32, device=g)
        dwv = torch.empty(self.h, self.n_kv * self.hd, dtype=torch.float32, device=g)
        dwo = torch.empty(self.n_q * self.hd, self.h, dtype=torch.float32, device=g)
        lib.tp_attn_unpack_grads(self.desc, dwqkv_p, dwo_p, dwq, dwk, dwv, dwo)
        return dx, dwq, dwk, dwv, dwo
