"""A stack of pre-norm decode layers built from the library's C-ABI calls.

Each layer, for a batch of b single-token sequences x (b, h):

    x <- x + sum_i Attn_i(RMSNorm(x))        (tp_attn_fwd with residual = x)
    x <- x + sum_i MLP_i(RMSNorm(x))         (tp_mlp_fwd with residual = x)

Each reduction also writes RMSNorm of its result (the y_norm output), which is the next
sublayer's input, so the only separate normalization is the first one of a step.

"How does tensor parallelism split a transformer feed-forward block's two matmuls", "One
collective": after the reduction the full y is "ready for the residual add and the following
normalization layer, both of which stay replicated"; page 1 (llms-explorer) facts: a dense Llama
layer makes 2 reductions (o_proj and down_proj).  Every step of the computation runs in the
library's kernels; this module only owns buffers and sequences the calls (optionally replaying
them as one CUDA graph).

Weights are synthetic (seeded, see ``inputs``), one set per layer; each layer has its own KV
cache of ``kv_len + 1`` slots, and every step writes the new token's key and value into slot
``kv_len`` so the KV length stays fixed from step to step.

The residual stream x is kept in float32 (TP_FLAG_F32_RESIDUAL): the GEMM inputs are the bf16
RMSNorm outputs, while the sums of the partials and the residual adds are rounded to fp32, so
sixteen layers never round the skip path to bf16.
"""

import torch

from . import inputs
from . import tpblock as tp


class DecodeStack:
    def __init__(self, layers, h, d_ff, n_q, n_kv, head_dim, p, kv_len, b=1, seed=0,
                 w_std=0.02, device=None, reduce_mode=tp.TP_REDUCE_SEPARATE):
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.L, self.h, self.b = layers, h, b
        self.adesc = tp.attn_desc(b, 1, h, n_q, n_kv, head_dim, p, True, "bf16", kv_len,
                                  reduce_mode=reduce_mode, flags=tp.TP_FLAG_F32_RESIDUAL)
        self.mdesc = tp.mlp_desc(b, h, d_ff, p, "swiglu", "bf16", reduce_mode,
                                 flags=tp.TP_FLAG_F32_RESIDUAL)
        self.layers = []
        for l in range(layers):
            a = inputs.attn_inputs(b, 1, h, n_q, n_kv, head_dim, "bf16", seed=seed,
                                   device=self.device, w_std=w_std, kv_len=kv_len, layer=l)
            m = inputs.mlp_inputs(b, h, d_ff, "swiglu", "bf16", seed=seed, device=self.device,
                                  w_std=w_std, layer=l)
            lay = {
                "wqkv": torch.empty(tp.tp_attn_wqkv_packed_bytes(self.adesc) // 2,
                                    dtype=torch.bfloat16, device=self.device),
                "wo": torch.empty(tp.tp_attn_wo_packed_bytes(self.adesc) // 2,
                                  dtype=torch.bfloat16, device=self.device),
                "w1p": torch.empty(tp.tp_mlp_w1_packed_bytes(self.mdesc) // 2,
                                   dtype=torch.bfloat16, device=self.device),
                "w2p": torch.empty(tp.tp_mlp_w2_packed_bytes(self.mdesc) // 2,
                                   dtype=torch.bfloat16, device=self.device),
                "k_cache": a["k_cache"], "v_cache": a["v_cache"],
            }
            tp.tp_attn_pack(self.adesc, a["wq"], a["wk"], a["wv"], a["wo"], lay["wqkv"], lay["wo"])
            tp.tp_mlp_pack(self.mdesc, m["w1"], m["w_up"], m["w2"], lay["w1p"], lay["w2p"])
            del a, m
            self.layers.append(lay)
        ws = max(tp.tp_attn_fwd_workspace(self.adesc), tp.tp_mlp_fwd_workspace(self.mdesc))
        self.ws = torch.empty(ws, dtype=torch.uint8, device=self.device)
        self.normed = torch.empty(b, 1, h, dtype=torch.bfloat16, device=self.device)
        self.normed2 = torch.empty(b, 1, h, dtype=torch.bfloat16, device=self.device)
        self.graph = None

    def step(self, x):
        """One decode step over all layers; x (b, 1, h) float32 on the device, updated in place."""
        tp.tp_rmsnorm(x, self.normed)
        for li, lay in enumerate(self.layers):
            tp.tp_attn_fwd(self.adesc, self.normed, lay["wqkv"], lay["wo"], x,
                           k_cache=lay["k_cache"], v_cache=lay["v_cache"], residual=x,
                           workspace=self.ws, y_norm=self.normed2)
            last = li == len(self.layers) - 1
            tp.tp_mlp_fwd(self.mdesc, self.normed2.view(self.b, self.h), lay["w1p"], lay["w2p"],
                          x.view(self.b, self.h), residual=x.view(self.b, self.h),
                          workspace=self.ws,
                          y_norm=None if last else self.normed.view(self.b, self.h))
        return x

    def capture(self, x):
        """Record step(x) into a CUDA graph (x must stay at the same address for replays)."""
        self.step(x)  # warm-up outside capture: tensor maps, kernel attributes
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                self.step(x)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = g
        return g

    def replay(self):
        self.graph.replay()
