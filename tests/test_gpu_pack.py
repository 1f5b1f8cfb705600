"""The shard packer's layouts, bit for bit, against the formulas the C header states.

"How does tensor parallelism split a transformer feed-forward block's two matmuls", "Column
split, then row split": shard i owns the columns i*F_s .. (i+1)*F_s - 1 of W1 (and of Wu for the
gated form) and exactly the matching rows of W2; "Tensor Parallelism" (klaylearn), Notes: shard i
owns whole query heads and whole KV heads, Wo by the matching rows.  The packed layouts are part
of the ABI (the weight gradients come back in them), so they are checked here directly: each
expected buffer is built on the host from the header's index formulas and compared with the
packer's output with torch.equal.  Random bf16 / fp32 values make any permutation of rows,
columns or shards visible (a feature permutation inside a shard leaves the block's results
unchanged, so the parity tests cannot see it).
"""

import pytest
import torch

from tensor_transformer_matmul_b200 import inputs
from tests.helpers import dev

pytestmark = pytest.mark.gpu


def _expected_mlp(w1, wu, w2, p, dtype):
    """w1p [p][R][d] and w2p [p][d][F_sp] from the header's formulas."""
    d, F = w1.shape
    Fs = F // p
    Fsp = (Fs + 127) // 128 * 128
    gated = wu is not None
    R = 2 * Fsp if gated else Fsp
    w1p = torch.zeros(p, R, d, dtype=dtype)
    w2p = torch.zeros(p, d, Fsp, dtype=dtype)
    for i in range(p):
        for f in range(Fs):
            col = i * Fs + f
            if gated:
                blk, r = divmod(f, 128)
                w1p[i, blk * 256 + r] = w1[:, col]
                w1p[i, blk * 256 + 128 + r] = wu[:, col]
            else:
                w1p[i, f] = w1[:, col]
            w2p[i, :, f] = w2[col, :]
    return w1p, w2p


@pytest.mark.parametrize("act,dtype,d,F,p", [
    ("swiglu", "bf16", 40, 408, 3),     # F_s = 136: two 128-feature blocks per shard, padded
    ("swiglu", "bf16", 24, 1024, 4),    # F_s = 256: exactly two blocks
    ("gelu", "bf16", 16, 96, 2),        # single W1, F_s = 48 padded to 128
    ("swiglu", "f32", 8, 300, 2),       # fp32 path
])
def test_mlp_packed_layout(lib, act, dtype, d, F, p):
    tdt = inputs.TORCH_DTYPE[dtype]
    w1 = inputs.normal((d, F), 1.0, 70, 1, dtype, "cpu")
    wu = inputs.normal((d, F), 1.0, 70, 2, dtype, "cpu") if act == "swiglu" else None
    w2 = inputs.normal((F, d), 1.0, 70, 3, dtype, "cpu")
    desc = lib.mlp_desc(1, d, F, p, act, dtype)
    eb = 2 if dtype == "bf16" else 4
    # the packer must write the padding too: start from a non-zero fill
    w1p = torch.full((lib.tp_mlp_w1_packed_bytes(desc) // eb,), 9.0, dtype=tdt, device=dev())
    w2p = torch.full((lib.tp_mlp_w2_packed_bytes(desc) // eb,), 9.0, dtype=tdt, device=dev())
    lib.tp_mlp_pack(desc, w1.to(dev()), None if wu is None else wu.to(dev()), w2.to(dev()),
                    w1p, w2p)
    torch.cuda.synchronize()
    e1, e2 = _expected_mlp(w1, wu, w2, p, tdt)
    assert w1p.numel() == e1.numel() and w2p.numel() == e2.numel()
    assert torch.equal(w1p.cpu().view(e1.shape), e1)
    assert torch.equal(w2p.cpu().view(e2.shape), e2)


@pytest.mark.parametrize("h,n_q,n_kv,hd,p", [(64, 8, 2, 16, 2), (48, 6, 3, 8, 3), (32, 4, 4, 8, 1)])
def test_attention_packed_layout(lib, h, n_q, n_kv, hd, p):
    wq = inputs.normal((h, n_q * hd), 1.0, 71, 1, "bf16", "cpu")
    wk = inputs.normal((h, n_kv * hd), 1.0, 71, 2, "bf16", "cpu")
    wv = inputs.normal((h, n_kv * hd), 1.0, 71, 3, "bf16", "cpu")
    wo = inputs.normal((n_q * hd, h), 1.0, 71, 4, "bf16", "cpu")
    desc = lib.attn_desc(1, 1, h, n_q, n_kv, hd, p)
    wqkv = torch.full((lib.tp_attn_wqkv_packed_bytes(desc) // 2,), 9.0, dtype=torch.bfloat16,
                      device=dev())
    wop = torch.full((lib.tp_attn_wo_packed_bytes(desc) // 2,), 9.0, dtype=torch.bfloat16,
                     device=dev())
    lib.tp_attn_pack(desc, wq.to(dev()), wk.to(dev()), wv.to(dev()), wo.to(dev()), wqkv, wop)
    torch.cuda.synchronize()
    qh, kh = n_q // p, n_kv // p
    Ra = (qh + 2 * kh) * hd
    e_qkv = torch.empty(p, Ra, h, dtype=torch.bfloat16)
    e_o = torch.empty(p, h, qh * hd, dtype=torch.bfloat16)
    for i in range(p):
        for r in range(qh * hd):
            e_qkv[i, r] = wq[:, i * qh * hd + r]
        for r in range(kh * hd):
            e_qkv[i, qh * hd + r] = wk[:, i * kh * hd + r]
            e_qkv[i, qh * hd + kh * hd + r] = wv[:, i * kh * hd + r]
        for c in range(qh * hd):
            e_o[i, :, c] = wo[i * qh * hd + c, :]
    assert torch.equal(wqkv.cpu().view(e_qkv.shape), e_qkv)
    assert torch.equal(wop.cpu().view(e_o.shape), e_o)
