"""The cost-model arithmetic against the figures the pages print (tests/golden/costmodel_figures.txt).

Where a page mixes MiB and GB the figure is accepted within 6 percent.
"""

import os

from oracle import costmodel as cm

MiB = 1 << 20
KiB = 1 << 10


def _golden():
    vals = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "costmodel_figures.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("=", 1))
                vals[k] = float(v)
    return vals


def _close(a, b, rel):
    return abs(a - b) <= rel * abs(b)


def test_reduction_counts():
    g = _golden()
    assert cm.reductions_per_microbatch(80, training=True) == g["reduces_80_layers_training"]
    assert cm.reductions_per_token(80) == g["reduces_80_layers_decode"]
    assert cm.reductions_per_token(61) == g["reduces_61_layers_decode"]


def test_prefill_message_and_ring_traffic():
    g = _golden()
    n = cm.message_bytes(1, 4096, 8192, 2)
    assert n == g["message_b1_s4096_h8192_bf16_MiB"] * MiB
    ring = cm.ring_bytes_per_rank(n, 8)
    assert ring == g["ring_per_gpu_tp8_MiB"] * MiB
    total = 320 * ring
    assert _close(total / 1e9, g["traffic_320_calls_GB"], 0.01)
    assert _close(total / 450e9, g["nvlink_time_s"], 0.06)
    assert _close(total / 50e9, g["nic_time_s"], 0.01)


def test_decode_payloads():
    g = _golden()
    n = cm.message_bytes(64, 1, 8192, 2)
    assert n == g["decode_b64_h8192_fp16_bytes"]
    assert cm.ring_bytes_per_rank(n, 8) == g["ring_per_rank_p8_MiB"] * MiB
    per_token = 2 * 80 * cm.ring_bytes_per_rank(n, 8)
    assert per_token == g["per_token_80_layers_MiB"] * MiB
    assert _close(per_token / 25e9 * 1e3, g["ethernet_200g_ms"], 0.06)
    p4 = 2 * 80 * cm.ring_bytes_per_rank(n, 4)
    assert p4 == g["p4_per_token_MiB"] * MiB
    assert _close(p4 / 450e9 * 1e3, g["p4_nvlink_450_ms"], 0.06)
    assert cm.message_bytes(1, 1, 8192, 2) == g["decode_b1_h8192_bf16_KiB"] * KiB
    assert cm.message_bytes(1, 1, 7168, 2) == g["decode_b1_h7168_bf16_KB"] * 1024
    assert _close(cm.reductions_per_token(80) * 20e-6 * 1e3, g["latency_160_x_20us_ms"], 1e-9)


def test_weight_streaming():
    g = _golden()
    t1 = cm.weight_stream_time_s(g["weights_70b_fp16_GB"] * 1e9, g["h100_hbm_TBps"] * 1e12)
    assert _close(t1 * 1e3, g["stream_1gpu_ms"], 0.005)
    t4 = cm.weight_stream_time_s(g["weights_70b_fp16_GB"] / 4 * 1e9, g["h100_hbm_TBps"] * 1e12)
    assert _close(t4 * 1e3, g["stream_p4_ms"], 0.005)
