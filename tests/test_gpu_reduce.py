"""tp_reduce_partials through the C ABI: the all-reduce's arithmetic on one GPU.

"One collective" (katajob, "How does tensor parallelism split ..."): y = sum_i y_i.  The library
adds the p partials in the fixed order 0..p-1 in fp32, adds the residual last, and rounds once:
the result must equal, bit for bit, that sequence of fp32 additions done on the host, and must
be within rounding of the float64 sum.
"""

import numpy as np
import pytest
import torch

from tests.helpers import TOL, dev, f64, rel_l2

pytestmark = pytest.mark.gpu


def _host_in_order(parts, res):
    acc = parts[0].astype(np.float32).copy()
    for s in range(1, parts.shape[0]):
        acc = (acc + parts[s].astype(np.float32)).astype(np.float32)
    if res is not None:
        acc = (res.astype(np.float32) + acc).astype(np.float32)
    return acc


@pytest.mark.parametrize("p", [1, 3, 8, 16])
@pytest.mark.parametrize("n", [8192, 8192 * 64 + 8, 1001])   # vector path, tail, scalar path
@pytest.mark.parametrize("residual", [False, True])
def test_fp32_partials_bit_exact_in_order(lib, p, n, residual):
    g = torch.Generator().manual_seed(p * 7 + n)
    parts = torch.randn(p, n, generator=g)
    res = torch.randn(n, generator=g) if residual else None
    out = torch.empty(n, device=dev())
    lib.tp_reset_reduction_count()
    lib.tp_reduce_partials(parts.to(dev()), p, n, out, residual=None if res is None else res.to(dev()))
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    want = _host_in_order(parts.numpy(), None if res is None else res.numpy())
    assert np.array_equal(out.cpu().numpy(), want)
    ref = f64(parts).sum(axis=0) + (0 if res is None else f64(res))
    assert rel_l2(f64(out), ref) <= 1e-6


@pytest.mark.parametrize("in_dt,out_dt", [(torch.float32, torch.bfloat16), (torch.bfloat16, torch.bfloat16),
                                          (torch.bfloat16, torch.float32)])
def test_dtype_combinations(lib, in_dt, out_dt):
    p, n = 8, 64 * 8192
    g = torch.Generator().manual_seed(3)
    parts = torch.randn(p, n, generator=g).to(in_dt)
    res = torch.randn(n, generator=g).to(out_dt)
    out = torch.empty(n, dtype=out_dt, device=dev())
    lib.tp_reduce_partials(parts.to(dev()), p, n, out, residual=res.to(dev()))
    torch.cuda.synchronize()
    want = torch.tensor(_host_in_order(parts.float().numpy(), res.float().numpy())).to(out_dt)
    assert torch.equal(out.cpu(), want)   # one RNE rounding of the in-order fp32 sum
    ref = f64(parts).sum(axis=0) + f64(res)
    assert rel_l2(f64(out), ref) <= TOL["bf16"]


def test_empty(lib):
    out = torch.empty(0, device=dev())
    lib.tp_reduce_partials(torch.empty(0, device=dev()), 4, 0, out)
    torch.cuda.synchronize()


@pytest.mark.parametrize("T,d,p", [
    (1, 8192, 8),      # a decode row of the workload: one cluster, one vector per thread
    (3, 776, 12),      # ragged column split, 12 partials (two groups of loads)
    (147, 512, 2),     # the most rows that still take the few-rows path (fewer than the SMs)
    (2, 16384, 4),     # two vectors per thread: the widest row of the cluster kernel
    (2, 16392, 4),     # one vector too wide: the two-kernel path
    (1, 8, 1),         # one shard, one vector: seven of the eight CTAs hold no columns
])
def test_reduce_norm_few_rows(lib, T, d, p):
    # reduce + RMSNorm of fewer rows than SMs (the decode reductions): y must equal, bit for bit,
    # the plain reduce of the same partials (the same in-order sum and rounding), and y_norm must
    # be the RMSNorm of the stored y rows
    from oracle import decode as odec
    from oracle import mlp as omlp
    from tensor_transformer_matmul_b200 import inputs
    from tests.helpers import Mlp, rel_l2_rows
    F = 128 * p
    inp = inputs.mlp_inputs(T, d, F, "gelu", "bf16", seed=60 + T, w_std=0.05)
    m = Mlp(lib, inp, p, "gelu", "bf16", 0)
    res = inputs.normal((T, d), 1.0, 60, 99, "bf16", "cpu").to(dev())
    x = inp["x"].to(dev())
    y_plain = torch.empty(T, d, dtype=torch.bfloat16, device=dev())
    lib.tp_mlp_fwd(m.desc, x, m.w1p, m.w2p, y_plain, residual=res, workspace=m.ws_f)
    y = torch.empty_like(y_plain)
    yn = torch.empty_like(y_plain)
    lib.tp_reset_reduction_count()
    lib.tp_mlp_fwd(m.desc, x, m.w1p, m.w2p, y, residual=res, workspace=m.ws_f, y_norm=yn)
    torch.cuda.synchronize()
    assert lib.tp_reduction_count() == 1
    assert torch.equal(y, y_plain)
    ref_norm = odec.rmsnorm(f64(y))
    assert rel_l2(f64(yn), ref_norm) <= 4e-3 and rel_l2_rows(f64(yn), ref_norm) <= 4e-3
    ref = omlp.mlp_forward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), "gelu") + f64(res)
    assert rel_l2(f64(y), ref) <= TOL["bf16"]
