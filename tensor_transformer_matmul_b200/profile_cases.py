"""Small, fixed workloads for kernel captures with a profiler.

A capture replays every profiled launch tens of times, so it wants a case that holds a few GB on
the device and runs a handful of launches.  Each case here draws its synthetic inputs, packs the
weights and runs the call ``--reps`` times (the first launches serve as warm-up; pick the launch
to capture with the profiler's skip count).

    python -m tensor_transformer_matmul_b200.profile_cases mlp_fwd --tokens 1024
    python -m tensor_transformer_matmul_b200.profile_cases attn_fwd --tokens 2048 --fused
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


CASES = {"mlp_fwd": mlp_fwd, "attn_fwd": attn_fwd}


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
