"""Failure detection on the GPU without a fault.

A bounded device wait that runs out must reach the host as TP_ERR_TIMEOUT through
tp_check_device_error and leave the context usable.  The library's self-test kernel waits,
through the same bounded mbarrier wait the tensor-core kernels use, on a barrier that nothing
completes, with a short limit; no kernel here traps, faults or hangs.
"""
import pytest
import torch

from oracle import mlp as omlp
from tensor_transformer_matmul_b200 import inputs
from tests.helpers import TOL, Mlp, f64, rel_l2

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared(lib):
    lib.tp_check_device_error()              # start from a clean error word
    lib.tp_selftest_wait_timeout(20000)      # 20 ms limit
    with pytest.raises(lib.TpError) as e:
        lib.tp_check_device_error()
    assert e.value.status == lib.TP_ERR_TIMEOUT
    # both waits ran out: the pipeline's mbarrier wait (bit 1) and the cross-CTA counter wait of
    # the one-launch decode MLP (bit 32)
    assert "site bits 33" in str(e.value)
    lib.tp_check_device_error()              # the report cleared the word


def test_context_usable_after_timeout(lib):
    lib.tp_selftest_wait_timeout(5000)
    with pytest.raises(lib.TpError):
        lib.tp_check_device_error()
    inp = inputs.mlp_inputs(17, 64, 256, "swiglu", "bf16", seed=3, w_std=0.05)
    m = Mlp(lib, inp, 4, "swiglu", "bf16")
    y = m.forward(inp["x"])
    torch.cuda.synchronize()
    lib.tp_check_device_error()
    ref = omlp.mlp_forward(f64(inp["x"]), f64(inp["w1"]), f64(inp["w2"]), "swiglu",
                           f64(inp["w_up"]))
    assert rel_l2(f64(y), ref) <= TOL["bf16"]
