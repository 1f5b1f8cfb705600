"""Pins for the sequence-parallel oracle ("Why tensor parallelism has to stay in scale-up",
"Where the 320 comes from": each all-reduce becomes a reduce-scatter plus an all-gather, the call
count doubles and the bytes stay the same).

None of these re-types the oracle's formula: they use the all-reduce as a library sum, brute-force
loops, the page's worked example and printed figures, and the MLP oracle's sharding invariant.
"""

import os

import numpy as np
import pytest

from oracle import costmodel as cm
from oracle import mlp
from oracle import seqpar as sp

MiB = 1 << 20


def _golden(name):
    vals = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("=", 1))
                vals[k] = [float(t) for t in v.split()]
    return vals


def test_reduce_scatter_then_all_gather_is_the_all_reduce():
    r = np.random.default_rng(0)
    parts = [r.standard_normal((12, 5)) for _ in range(4)]
    full = sp.all_gather(sp.reduce_scatter(parts))
    np.testing.assert_allclose(full, np.stack(parts).sum(axis=0), rtol=1e-14, atol=1e-14)


def test_reduce_scatter_brute_force_with_residual():
    # p = 2 shards, T = 4 tokens, d = 3, small integers: every value is exact
    parts = [np.arange(12).reshape(4, 3), 10 * np.arange(12).reshape(4, 3)]
    res = [np.full((2, 3), 100), np.full((2, 3), 200)]
    out = sp.reduce_scatter(parts, res)
    assert len(out) == 2
    for i in range(2):
        assert out[i].shape == (2, 3)
        for rr in range(2):
            for c in range(3):
                t = 2 * i + rr
                want = parts[0][t][c] + parts[1][t][c] + res[i][rr][c]
                assert out[i][rr][c] == want


def test_slices_follow_token_order():
    # shard i holds rows i*T/p .. (i+1)*T/p - 1: tag each row with its index
    T, p = 12, 3
    tagged = np.repeat(np.arange(T, dtype=np.float64)[:, None], 2, axis=1)
    out = sp.reduce_scatter([tagged, np.zeros_like(tagged)])
    # two partials -> two slices of 6 rows
    assert [s[:, 0].tolist() for s in out] == [list(range(6)), list(range(6, 12))]
    out3 = sp.reduce_scatter([tagged / 3] * 3)
    assert [s[:, 0].tolist() for s in out3] == [[0.0, 1, 2, 3], [4.0, 5, 6, 7], [8.0, 9, 10, 11]]


def test_p_must_divide_tokens():
    with pytest.raises(ValueError):
        sp.reduce_scatter([np.zeros((5, 2))] * 2)
    with pytest.raises(ValueError):
        sp.token_slices(7, 3)


def test_worked_example_under_sequence_parallelism():
    # "What is Tensor Parallel": x = [1, 2] -> y = [1, 2, 3] -> z = [4, 5] with TP = 3.  Three
    # tokens k x (k = 1, 2, 3) give k z (the block is linear); with SP over 3 shards, shard k-1's
    # slice is token k's output.
    g = _golden("worked_example_h2_dff3.txt")
    A = np.array([g["A_row0"], g["A_row1"]])
    B = np.array([g["B_row0"], g["B_row1"], g["B_row2"]])
    x = np.array([[k * v for v in g["x"]] for k in (1, 2, 3)])
    _, partials = mlp.mlp_forward_sharded(x, A, B, "identity", int(g["tp"][0]))
    slices = sp.reduce_scatter(partials)
    for k in (1, 2, 3):
        assert np.array_equal(slices[k - 1], np.array([[k * v for v in g["z"]]]))


def test_sequence_parallel_block_equals_unsharded_block():
    r = np.random.default_rng(1)
    T, d, F, p = 8, 6, 12, 4
    x, w1, wu, w2 = (r.standard_normal((T, d)), r.standard_normal((d, F)),
                     r.standard_normal((d, F)), r.standard_normal((F, d)))
    x_slices = [x[i * 2:(i + 1) * 2] for i in range(p)]
    _, partials = mlp.mlp_forward_sharded(sp.all_gather(x_slices), w1, w2, "swiglu", p, wu)
    got = sp.all_gather(sp.reduce_scatter(partials))
    np.testing.assert_allclose(got, mlp.mlp_forward(x, w1, w2, "swiglu", wu), rtol=1e-12)


def test_call_count_doubles_and_bytes_stay():
    g = _golden("costmodel_figures.txt")
    # 80 layers, training: 320 all-reduces (printed) -> 640 collectives with SP
    assert 80 * sp.collective_calls_per_layer(True, False) == g["reduces_80_layers_training"][0]
    assert 80 * sp.collective_calls_per_layer(True, True) == 2 * g["reduces_80_layers_training"][0]
    assert sp.collective_calls_per_layer(False, True) == 4
    # the same bytes: b=1, s=4096, h=8192 bf16 message (64 MiB printed), TP=8 ring: 112 MiB
    n = cm.message_bytes(1, 4096, 8192, 2)
    assert sp.ring_bytes_per_rank(n, 8, True) == sp.ring_bytes_per_rank(n, 8, False)
    assert sp.ring_bytes_per_rank(n, 8, True) == g["ring_per_gpu_tp8_MiB"][0] * MiB
    assert sp.ring_bytes_per_rank(n, 8, True) == cm.ring_bytes_per_rank(n, 8)
