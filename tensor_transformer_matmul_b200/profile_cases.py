"""Small, fixed workloads for kernel captures with a profiler.

A capture replays every profiled launch tens of times, so it wants a case that holds a few GB on
the device and runs a handful of launches.  Each case here draws its synthetic inputs, packs the
weights and runs the call ``--reps`` times (the first launches serve as warm-up; pick the launch
to capture with the profiler's skip count).

    python -m tensor_transformer_matmul_b200.profile_cases mlp_fwd --tokens 1024
    python -m tensor_transformer_matmul_b200.profile_cases attn_fwd --tokens 2048 --fused
    python -m tensor_transformer_matmul_b200.profile_cases attn_bwd --tokens 2048
    python -m tensor_transformer_matmul_b200.profile_cases moe_fwd --tokens 1024
    python -m tensor_transformer_matmul_b200.profile_cases decode_layer --tokens 1
"""
import argparse

import torch

from tensor_transformer_matmul_b200 import inputs
from tensor_transformer_matmul_b200 import tpblock as tp


def mlp_fwd(tokens, reps, fused, d=8192, d_ff=28672, p=8):
    """SwiGLU MLP forward with the decode/prefill configuration's weights (d=8192, d_ff=28672,
    p=8, bf16, W ~ N(0, 0.02))."""
    mode = tp.TP_REDUCE_FUSED if fused else tp.TP_REDUCE_SEPARATE
    desc = tp.mlp_desc(tokens, d, d_ff, p, "swiglu", "bf16", mode)
    inp = inputs.mlp_inputs(tokens, d, d_ff, "swiglu", "bf16", device="cuda", w_std=0.02)
    w1p = torch.empty(tp.tp_mlp_w1_packed_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    w2p = torch.empty(tp.tp_mlp_w2_packed_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    tp.tp_mlp_pack(desc, inp["w1"], inp["w_up"], inp["w2"], w1p, w2p)
    del inp["w1"], inp["w_up"], inp["w2"]
    ws = torch.empty(tp.tp_mlp_fwd_workspace(desc), dtype=torch.uint8, device="cuda")
    y = torch.empty(tokens, d, dtype=torch.bfloat16, device="cuda")
    for _ in range(reps):
        tp.tp_mlp_fwd(desc, inp["x"], w1p, w2p, y, workspace=ws)
    torch.cuda.synchronize()
    return y


def attn_fwd(tokens, reps, fused, h=8192, n_q=64, n_kv=8, hd=128, p=8):
    """GQA attention block forward (b=1, causal) with the attention configuration's heads."""
    mode = tp.TP_REDUCE_FUSED if fused else tp.TP_REDUCE_SEPARATE
    desc = tp.attn_desc(1, tokens, h, n_q, n_kv, hd, p, reduce_mode=mode)
    ai = inputs.attn_inputs(1, tokens, h, n_q, n_kv, hd, "bf16", seed=0, device="cuda")
    wqkv = torch.empty(tp.tp_attn_wqkv_packed_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    wo = torch.empty(tp.tp_attn_wo_packed_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    tp.tp_attn_pack(desc, ai["wq"], ai["wk"], ai["wv"], ai["wo"], wqkv, wo)
    ws = torch.empty(tp.tp_attn_fwd_workspace(desc), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(ai["x"])
    for _ in range(reps):
        tp.tp_attn_fwd(desc, ai["x"], wqkv, wo, y, workspace=ws)
    torch.cuda.synchronize()
    return y


def attn_bwd(tokens, reps, fused, h=8192, n_q=64, n_kv=8, hd=128, p=8):
    """GQA attention block backward (b=1, causal) with the attention configuration's heads."""
    mode = tp.TP_REDUCE_FUSED if fused else tp.TP_REDUCE_SEPARATE
    desc = tp.attn_desc(1, tokens, h, n_q, n_kv, hd, p, reduce_mode=mode)
    ai = inputs.attn_inputs(1, tokens, h, n_q, n_kv, hd, "bf16", seed=0, device="cuda")
    wqkv = torch.empty(tp.tp_attn_wqkv_packed_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    wo = torch.empty(tp.tp_attn_wo_packed_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    tp.tp_attn_pack(desc, ai["wq"], ai["wk"], ai["wv"], ai["wo"], wqkv, wo)
    dy = inputs.normal((1, tokens, h), 1.0, 0, 97, "bf16", "cuda")
    dx = torch.empty_like(ai["x"])
    dwqkv = torch.empty(wqkv.numel(), dtype=torch.float32, device="cuda")
    dwo = torch.empty(wo.numel(), dtype=torch.float32, device="cuda")
    ws = torch.empty(tp.tp_attn_bwd_workspace(desc), dtype=torch.uint8, device="cuda")
    for _ in range(reps):
        tp.tp_attn_bwd(desc, ai["x"], wqkv, wo, dy, dx, dwqkv, dwo, workspace=ws)
    torch.cuda.synchronize()
    return dx


def moe_fwd(tokens, reps, fused, d=7168, n_experts=32, top_k=8, d_ff=2048, p=8):
    """MoE block forward with DeepSeek-V3-shaped experts (d=7168, width 2048, top-8, a shared
    expert of width 2048, p=8) but 32 experts, so that the weights take about 3 GB."""
    desc = tp.moe_desc(tokens, d, d_ff, d_ff, n_experts, top_k, p)
    e1, e2 = tp.tp_moe_expert_w1_bytes(desc) // 2, tp.tp_moe_expert_w2_bytes(desc) // 2
    w1p = torch.empty(n_experts * e1, dtype=torch.bfloat16, device="cuda")
    w2p = torch.empty(n_experts * e2, dtype=torch.bfloat16, device="cuda")
    ed = tp.mlp_desc(1, d, d_ff, p, "swiglu", "bf16")
    for e in range(n_experts):
        g, u, o = (inputs.normal(s, 0.02, 0, 1000 + 3 * e + j, "bf16", "cuda")
                   for j, s in enumerate(((d, d_ff), (d, d_ff), (d_ff, d))))
        tp.tp_mlp_pack(ed, g, u, o, w1p[e * e1:(e + 1) * e1], w2p[e * e2:(e + 1) * e2])
    w1s = torch.empty(tp.tp_moe_shared_w1_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    w2s = torch.empty(tp.tp_moe_shared_w2_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    g, u, o = (inputs.normal(s, 0.02, 0, 900 + j, "bf16", "cuda")
               for j, s in enumerate(((d, d_ff), (d, d_ff), (d_ff, d))))
    tp.tp_mlp_pack(ed, g, u, o, w1s, w2s)
    wr = inputs.normal((d, n_experts), d ** -0.5, 0, 901, "bf16", "cuda")
    x = inputs.normal((tokens, d), 1.0, 0, 902, "bf16", "cuda")
    y = torch.empty_like(x)
    ws = torch.empty(tp.tp_moe_fwd_workspace(desc), dtype=torch.uint8, device="cuda")
    for _ in range(reps):
        tp.tp_moe_fwd(desc, x, wr, w1p, w2p, y, w1p_s=w1s, w2p_s=w2s, workspace=ws)
    torch.cuda.synchronize()
    return y


def decode_layer(tokens, reps, fused, h=8192, d_ff=28672, n_q=64, n_kv=8, hd=128, p=8,
                 kv_len=4096):
    """One layer of the decode stack (b = ``tokens`` single-token sequences, KV length 4096):
    the attention block (QKV GEMM, split-KV decode attention with the KV append, O projection,
    reduce + RMSNorm) then the SwiGLU MLP block, fp32 residual stream."""
    from tensor_transformer_matmul_b200.decode_stack import DecodeStack
    mode = tp.TP_REDUCE_FUSED if fused else tp.TP_REDUCE_SEPARATE
    st = DecodeStack(1, h, d_ff, n_q, n_kv, hd, p, kv_len, b=tokens, reduce_mode=mode)
    x = torch.randn(tokens, 1, h, device="cuda")
    for _ in range(reps):
        st.step(x)
    torch.cuda.synchronize()
    return x


CASES = {"mlp_fwd": mlp_fwd, "attn_fwd": attn_fwd, "attn_bwd": attn_bwd, "moe_fwd": moe_fwd,
         "decode_layer": decode_layer}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("case", choices=sorted(CASES))
    ap.add_argument("--tokens", type=int, default=1024)
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--fused", action="store_true", help="TP_REDUCE_FUSED instead of SEPARATE")
    a = ap.parse_args(argv)
    y = CASES[a.case](a.tokens, a.reps, a.fused)
    print(f"{a.case} tokens={a.tokens} reps={a.reps} fused={a.fused} ok, mean|y|="
          f"{float(y.float().abs().mean()):.4f}")


if __name__ == "__main__":
    main()
