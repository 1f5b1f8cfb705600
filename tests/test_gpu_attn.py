"""GQA attention block on the GPU through the C ABI against the float64 oracle.

Tolerance (rel-L2 of each output tensor): 2e-2 for bf16, 1e-5 for fp32.
"""

import numpy as np
import pytest
import torch

from oracle import attention as oattn
from tensor_transformer_matmul_b200 import inputs
from tests.helpers import rel_l2_rows
from tests.helpers import TOL, Attn, dev, f64, rel_l2

pytestmark = pytest.mark.gpu


def _ref(inp, n_q, n_kv, hd, causal):
    return oattn.attention_forward(*(f64(inp[k]) for k in ("x", "wq", "wk", "wv", "wo")),
                                   n_q, n_kv, hd, causal=causal)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("b,s,h,n_q,n_kv,hd,p", [
    (2, 37, 256, 8, 2, 32, 2),      # ragged sequence, two shards, 4 Q heads per KV head
    (1, 130, 192, 4, 4, 64, 4),     # MHA (n_kv = n_q), one head per shard
    (1, 200, 512, 16, 2, 128, 1),   # one shard owns everything (p = 1)
    (3, 9, 64, 8, 8, 8, 8),         # tiny head_dim, p = n_kv
])
def test_prefill_bf16(lib, causal, b, s, h, n_q, n_kv, hd, p):
    inp = inputs.attn_inputs(b, s, h, n_q, n_kv, hd, "bf16", seed=1, w_std=0.05)
    a = Attn(lib, inp, p, "bf16", causal, n_q=n_q, n_kv=n_kv, hd=hd, reduce_mode=int(causal))
    lib.tp_reset_reduction_count()
    y = a.forward(inp["x"])
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    assert rel_l2(f64(y), _ref(inp, n_q, n_kv, hd, causal)) <= TOL["bf16"]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("b,s,hd", [(2, 300, 128), (1, 257, 64), (3, 128, 128), (1, 1, 128)])
def test_prefill_tensor_core_kernel(lib, causal, b, s, hd):
    # head_dim 64/128 runs the tcgen05 flash kernel: several 128-row query tiles, ragged last
    # tile, sequences packed back to back, a single-token sequence
    h, n_q, n_kv, p = 256, 8, 2, 2
    inp = inputs.attn_inputs(b, s, h, n_q, n_kv, hd, "bf16", seed=9, w_std=0.05)
    a = Attn(lib, inp, p, "bf16", causal, n_q=n_q, n_kv=n_kv, hd=hd)
    y = a.forward(inp["x"])
    torch.cuda.synchronize()
    assert rel_l2(f64(y), _ref(inp, n_q, n_kv, hd, causal)) <= TOL["bf16"]


def test_prefill_fp32(lib):
    inp = inputs.attn_inputs(2, 21, 48, 6, 2, 8, "f32", seed=2, w_std=0.1)
    a = Attn(lib, inp, 2, "f32", True, n_q=6, n_kv=2, hd=8)
    y = a.forward(inp["x"])
    torch.cuda.synchronize()
    assert rel_l2(f64(y), _ref(inp, 6, 2, 8, True)) <= TOL["f32"]


def test_residual(lib):
    inp = inputs.attn_inputs(1, 50, 256, 8, 2, 32, "bf16", seed=3, w_std=0.05)
    a = Attn(lib, inp, 2, "bf16", True, n_q=8, n_kv=2, hd=32)
    res = inputs.normal((1, 50, 256), 1.0, 3, 77, "bf16", "cpu").to(dev())
    y = a.forward(inp["x"], residual=res)
    torch.cuda.synchronize()
    assert rel_l2(f64(y), _ref(inp, 8, 2, 32, True) + f64(res)) <= TOL["bf16"]


@pytest.mark.parametrize("dtype,b,kv_len,h,n_q,n_kv,hd,p,mode", [
    ("bf16", 3, 300, 256, 8, 2, 64, 2, 0),     # three key chunks
    ("bf16", 3, 300, 256, 8, 2, 64, 2, 1),     # same, shard reduce fused into the O projection
    ("bf16", 1, 4096, 512, 16, 2, 128, 2, 1),  # 33 chunks, group of 8 query heads per KV head
    ("bf16", 2, 1, 128, 4, 4, 32, 4, 0),       # a single cached key
    ("f32", 2, 37, 64, 4, 2, 32, 2, 0),
    # output projection of 4 x 40 = 160 tiles of 32 k-blocks: the 12 past a wave are split,
    # then every CTA runs whole tiles
    ("bf16", 2, 64, 5120, 64, 8, 128, 4, 0),
])
def test_decode(lib, dtype, b, kv_len, h, n_q, n_kv, hd, p, mode):
    inp = inputs.attn_inputs(b, 1, h, n_q, n_kv, hd, dtype, seed=4, w_std=0.05, kv_len=kv_len)
    a = Attn(lib, inp, p, dtype, True, kv_len=kv_len, n_q=n_q, n_kv=n_kv, hd=hd, reduce_mode=mode)
    kc, vc = inp["k_cache"].to(dev()), inp["v_cache"].to(dev())
    y = a.forward(inp["x"], k_cache=kc, v_cache=vc)
    torch.cuda.synchronize()
    kc0, vc0 = f64(inp["k_cache"])[:, :, :kv_len], f64(inp["v_cache"])[:, :, :kv_len]
    ref, kn, vn = oattn.attention_decode(f64(inp["x"])[:, 0], *(f64(inp[k]) for k in ("wq", "wk", "wv", "wo")),
                                         kc0, vc0, n_q, n_kv, hd)
    tol = TOL[dtype]
    assert rel_l2(f64(y)[:, 0], ref) <= tol
    # the new token's key and value landed in slot kv_len; the cached slots are untouched
    assert rel_l2(f64(kc)[:, :, kv_len], kn) <= tol
    assert rel_l2(f64(vc)[:, :, kv_len], vn) <= tol
    assert np.array_equal(f64(kc)[:, :, :kv_len], kc0)


@pytest.mark.parametrize("b,kv_len,n_q,n_kv,hd,spare", [
    (1, 64, 4, 4, 128, 0),     # one query head per KV head; the new token opens a 32-key tile
    (2, 31, 8, 4, 128, 7),     # two per KV head; the new token closes a tile; spare slots
    (1, 4111, 16, 2, 128, 0),  # eight per KV head, a last split of a few keys
    (2, 700, 8, 2, 64, 33),    # head_dim 64, four per KV head, spare slots past the new token
    (3, 17, 16, 2, 64, 0),     # one split holding 18 keys
    (1, 6000, 16, 2, 128, 0),  # 19 splits, more than a cluster takes: merged through memory
])
def test_decode_edges(lib, b, kv_len, n_q, n_kv, hd, spare):
    # slots past the new token (kv_cap > kv_len + 1) hold NaN: they must never be read
    h, p = 256, 2
    inp = inputs.attn_inputs(b, 1, h, n_q, n_kv, hd, "bf16", seed=5, w_std=0.05, kv_len=kv_len)
    cap = kv_len + 1 + spare
    kc = torch.full((b, n_kv, cap, hd), float("nan"), dtype=torch.bfloat16, device=dev())
    vc = torch.full_like(kc, float("nan"))
    kc[:, :, :kv_len] = inp["k_cache"][:, :, :kv_len].to(dev())
    vc[:, :, :kv_len] = inp["v_cache"][:, :, :kv_len].to(dev())
    a = Attn(lib, inp, p, "bf16", True, kv_len=kv_len, n_q=n_q, n_kv=n_kv, hd=hd)
    desc = lib.attn_desc(b, 1, h, n_q, n_kv, hd, p, True, "bf16", kv_len, kv_cap=cap)
    ws = torch.empty(lib.tp_attn_fwd_workspace(desc), dtype=torch.uint8, device=dev())
    y = torch.empty(b, 1, h, dtype=torch.bfloat16, device=dev())
    lib.tp_attn_fwd(desc, inp["x"].to(dev()), a.wqkv, a.wo, y, k_cache=kc, v_cache=vc, workspace=ws)
    torch.cuda.synchronize()
    kc0, vc0 = f64(inp["k_cache"])[:, :, :kv_len], f64(inp["v_cache"])[:, :, :kv_len]
    ref, kn, vn = oattn.attention_decode(f64(inp["x"])[:, 0], *(f64(inp[k]) for k in ("wq", "wk", "wv", "wo")),
                                         kc0, vc0, n_q, n_kv, hd)
    assert rel_l2(f64(y)[:, 0], ref) <= TOL["bf16"]
    assert rel_l2_rows(f64(y)[:, 0], ref) <= TOL["bf16"]
    assert rel_l2(f64(kc)[:, :, kv_len], kn) <= TOL["bf16"]
    assert rel_l2(f64(vc)[:, :, kv_len], vn) <= TOL["bf16"]
    assert np.array_equal(f64(kc)[:, :, :kv_len], kc0)
    assert torch.isnan(kc[:, :, kv_len + 1:].float()).all()


def test_decode_matches_prefill_last_row(lib):
    # decoding position L over a cache holding the keys/values of positions 0..L-1 equals the
    # last row of causal prefill over L+1 tokens (both through the library)
    b, L, h, n_q, n_kv, hd, p = 1, 64, 256, 8, 2, 64, 2
    inp = inputs.attn_inputs(b, L + 1, h, n_q, n_kv, hd, "bf16", seed=5, w_std=0.05)
    pre = Attn(lib, inp, p, "bf16", True, n_q=n_q, n_kv=n_kv, hd=hd)
    y_pre = pre.forward(inp["x"])
    x = f64(inp["x"])[0]
    kc = (x[:L] @ f64(inp["wk"])).reshape(L, n_kv, hd).transpose(1, 0, 2)[None]
    vc = (x[:L] @ f64(inp["wv"])).reshape(L, n_kv, hd).transpose(1, 0, 2)[None]
    kcache = torch.zeros(1, n_kv, L + 1, hd, dtype=torch.bfloat16)
    vcache = torch.zeros_like(kcache)
    kcache[:, :, :L] = torch.tensor(kc, dtype=torch.float64).to(torch.bfloat16)
    vcache[:, :, :L] = torch.tensor(vc, dtype=torch.float64).to(torch.bfloat16)
    dinp = dict(inp)
    dinp["x"] = inp["x"][:, L:L + 1].contiguous()
    dec = Attn(lib, dinp, p, "bf16", True, kv_len=L, n_q=n_q, n_kv=n_kv, hd=hd)
    kd, vd = kcache.to(dev()), vcache.to(dev())
    y_dec = dec.forward(dinp["x"], k_cache=kd, v_cache=vd)
    torch.cuda.synchronize()
    assert rel_l2(f64(y_dec)[0, 0], f64(y_pre)[0, L]) <= TOL["bf16"]


@pytest.mark.parametrize("mode", [0, 1])
def test_full_size_attention_sampled(lib, mode):
    # b=1, s=2048, h=8192, 64 Q / 8 KV heads, head_dim 128, p=8, causal, W ~ N(0, 0.02);
    # mode 1 adds the 8 shard partials inside the output projection's accumulator
    cfg = dict(b=1, s=2048, h=8192, n_q=64, n_kv=8, hd=128)
    inp = inputs.attn_inputs(*cfg.values(), "bf16", seed=0, device="cuda", w_std=0.02)
    a = Attn(lib, inp, 8, "bf16", True, n_q=64, n_kv=8, hd=128, reduce_mode=mode)
    y = a.forward(inp["x"])
    torch.cuda.synchronize()
    # one row in every 256-row block of the sequence (two 128-query flash tiles), plus the first
    # and last rows; whole block and row by row
    rows = sorted({0, 1, 2047} | {b * 256 + (37 * (b + 1) * 3) % 256 for b in range(8)})
    ref = oattn.attention_forward_rows(*(f64(inp[k]) for k in ("x", "wq", "wk", "wv", "wo")),
                                       64, 8, 128, rows, causal=True)
    assert rel_l2(f64(y)[0][rows], ref) <= TOL["bf16"]
    assert rel_l2_rows(f64(y)[0][rows], ref) <= TOL["bf16"]


def test_full_size_decode_layer_attention(lib):
    # one decode step of the attention block: b=1, KV length 4096 + the new token
    inp = inputs.attn_inputs(1, 1, 8192, 64, 8, 128, "bf16", seed=0, device="cuda", w_std=0.02,
                             kv_len=4096)
    a = Attn(lib, inp, 8, "bf16", True, kv_len=4096, n_q=64, n_kv=8, hd=128)
    kc, vc = inp["k_cache"].clone(), inp["v_cache"].clone()
    y = a.forward(inp["x"], k_cache=kc, v_cache=vc)
    torch.cuda.synchronize()
    ref, _, _ = oattn.attention_decode(f64(inp["x"])[:, 0], *(f64(inp[k]) for k in ("wq", "wk", "wv", "wo")),
                                       f64(inp["k_cache"])[:, :, :4096], f64(inp["v_cache"])[:, :, :4096],
                                       64, 8, 128)
    assert rel_l2(f64(y)[:, 0], ref) <= TOL["bf16"]


def test_f32_residual_stream(lib):
    inp = inputs.attn_inputs(1, 40, 256, 8, 2, 32, "bf16", seed=8, w_std=0.05)
    a = Attn(lib, inp, 2, "bf16", True, n_q=8, n_kv=2, hd=32)
    desc = lib.attn_desc(1, 40, 256, 8, 2, 32, 2, True, "bf16", flags=lib.TP_FLAG_F32_RESIDUAL)
    res = torch.randn(1, 40, 256, device=dev())
    y = torch.empty(1, 40, 256, device=dev())
    lib.tp_attn_fwd(desc, inp["x"].to(dev()), a.wqkv, a.wo, y, residual=res, workspace=a.ws)
    torch.cuda.synchronize()
    assert rel_l2(f64(y), _ref(inp, 8, 2, 32, True) + f64(res)) <= TOL["bf16"]


@pytest.mark.parametrize("rows,d", [
    (5, 300),      # d not a multiple of 8: one block per row
    (1, 8192),     # few rows: each row spread over 16 blocks of 512 columns
    (3, 1000),     # few rows, ragged last 512-column block
    (200, 64),     # more rows than SMs: one block per row
])
@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
def test_rmsnorm_dtypes(lib, rows, d, in_dtype):
    from oracle import decode as odec
    x = torch.randn(rows, d, device=dev()).to(in_dtype)
    for out_dtype, tol in ((torch.bfloat16, TOL["bf16"]), (torch.float32, TOL["f32"])):
        out = torch.empty(rows, d, dtype=out_dtype, device=dev())
        lib.tp_rmsnorm(x, out)
        torch.cuda.synchronize()
        assert rel_l2(f64(out), odec.rmsnorm(f64(x))) <= tol


@pytest.mark.parametrize("kv_len", [0, 200])
def test_y_norm_output(lib, kv_len):
    from oracle import decode as odec
    s_len = 1 if kv_len else 40
    inp = inputs.attn_inputs(2, s_len, 256, 8, 2, 64, "bf16", seed=11, w_std=0.05, kv_len=kv_len)
    a = Attn(lib, inp, 2, "bf16", True, kv_len=kv_len, n_q=8, n_kv=2, hd=64)
    res = torch.randn(2, s_len, 256, device=dev())
    desc = lib.attn_desc(2, s_len, 256, 8, 2, 64, 2, True, "bf16", kv_len,
                         flags=lib.TP_FLAG_F32_RESIDUAL)
    y = torch.empty(2, s_len, 256, device=dev())
    yn = torch.empty(2, s_len, 256, dtype=torch.bfloat16, device=dev())
    kc = inp["k_cache"].to(dev()) if kv_len else None
    vc = inp["v_cache"].to(dev()) if kv_len else None
    lib.tp_attn_fwd(desc, inp["x"].to(dev()), a.wqkv, a.wo, y, k_cache=kc, v_cache=vc,
                    residual=res, workspace=a.ws, y_norm=yn)
    torch.cuda.synchronize()
    if kv_len:
        ref, _, _ = oattn.attention_decode(f64(inp["x"])[:, 0], *(f64(inp[k]) for k in ("wq", "wk", "wv", "wo")),
                                           f64(inp["k_cache"])[:, :, :kv_len], f64(inp["v_cache"])[:, :, :kv_len],
                                           8, 2, 64)
        ref = ref[:, None] + f64(res)
    else:
        ref = _ref(inp, 8, 2, 64, True) + f64(res)
    assert rel_l2(f64(y), ref) <= TOL["bf16"]
    assert rel_l2(f64(yn), odec.rmsnorm(ref)) <= TOL["bf16"]
