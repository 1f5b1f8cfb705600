"""The allocation-free MLP forward (tp_mlp_fwd_static_ws) against the regular tp_mlp_fwd.

Some callers cannot call cudaMalloc (for example a plug-in whose host application owns all device
memory, or a loop where an allocation that may synchronize the device is not allowed).  For them
the library keeps its own fixed scratch array and tp_mlp_fwd_static_ws takes only inputs and
outputs.  It runs the same kernels as tp_mlp_fwd on the same descriptor, and every reduction in
them has a fixed order, so its output must equal the regular entry point's bit for bit.  This file
checks, through the C ABI, two calls in a row (of different shapes, so the second reads scratch
last written by another shape) for bit equality with tp_mlp_fwd, one of them also against the
float64 oracle, the residual path, and that a shape too large for the array is refused with
nothing written.  It runs last (file name) and works both alone in a fresh process and after the
other tests.
"""

import pytest
import torch

from oracle import mlp as omlp
from tensor_transformer_matmul_b200 import inputs
from tests.helpers import TOL, Mlp, dev, f64, rel_l2

pytestmark = pytest.mark.gpu


def _regular_and_static(lib, T, d, F, p, seed):
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=seed, w_std=0.05)
    m = Mlp(lib, inp, p, "swiglu", "bf16")
    x = inp["x"].to(dev())
    y_ref = m.forward(x, save=False)
    y_static = torch.full_like(y_ref, float("nan"))
    lib.tp_mlp_fwd_static_ws(m.desc, x, m.w1p, m.w2p, y_static)
    torch.cuda.synchronize()
    return inp, y_ref, y_static


def test_two_calls_in_a_row_match_regular_entry_point(lib):
    # first call: decode-shaped batch; second call: a different, ragged shape, so the scratch it
    # reads was last written by a call of another shape
    for i, (T, d, F, p, seed) in enumerate(((64, 1024, 4096, 8, 11), (37, 512, 3 * 1024, 3, 12))):
        inp, y_ref, y_static = _regular_and_static(lib, T, d, F, p, seed)
        assert torch.equal(y_static, y_ref), (T, d, F, p)
        if i == 0:
            ref = omlp.mlp_forward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), "swiglu",
                                   f64(inp["w_up"]))
            assert rel_l2(f64(y_static), ref) <= TOL["bf16"]


def test_residual_through_static_scratch(lib):
    T, d, F, p = 16, 256, 1024, 4
    inp = inputs.mlp_inputs(T, d, F, "swiglu", "bf16", seed=13, w_std=0.05)
    m = Mlp(lib, inp, p, "swiglu", "bf16")
    x = inp["x"].to(dev())
    res = inputs.normal((T, d), 1.0, 13, 99, "bf16", "cpu").to(dev())
    y_ref = m.forward(x, residual=res, save=False)
    y_static = torch.empty_like(y_ref)
    lib.tp_mlp_fwd_static_ws(m.desc, x, m.w1p, m.w2p, y_static, residual=res)
    torch.cuda.synchronize()
    assert torch.equal(y_static, y_ref)


def test_too_large_for_static_scratch_is_rejected(lib):
    # T = 4096 at d = 8192, d_ff = 28672, p = 8 needs ~1.7 GB of scratch: refused before anything
    # is enqueued, so the output keeps its sentinel
    desc = lib.mlp_desc(4096, 8192, 28672, 8, "swiglu", "bf16")
    assert lib.tp_mlp_fwd_workspace(desc) > (32 << 20)
    x = torch.zeros(8, dtype=torch.bfloat16, device=dev())  # never read: the call is refused first
    y = torch.full((8,), 3.0, dtype=torch.bfloat16, device=dev())
    with pytest.raises(lib.TpError) as e:
        lib.tp_mlp_fwd_static_ws(desc, x, x, x, y)
    assert e.value.status == lib.TP_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(y, torch.full_like(y, 3.0))
