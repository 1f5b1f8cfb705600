"""Oracle for the sequence-parallel form of the block's collective (float64, CPU).

Test infrastructure only (see the package docstring).

Source (page title, section): "Why tensor parallelism has to stay in scale-up" (keysight),
"Where the 320 comes from": with sequence parallelism each all-reduce becomes a reduce-scatter
plus an all-gather; the number of collective calls roughly doubles while the bytes moved stay the
same; each message is one b x s x h activation.

Readings where the page leaves a step open (the Megatron pairing it names):

* The scattered dimension is the token dimension: shard i keeps token rows
  [i T/p, (i+1) T/p) of the [T, d] sum, and p divides T.
* The residual add and the normalisation between blocks act on those slices; the all-gather
  restores the full [T, d] input in token order before the next column-parallel matmul.
* In the backward pass the all-gather's gradient is a reduce-scatter and the reduce-scatter's an
  all-gather, so the input gradient ends up token-sliced as well.
"""

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def token_slices(T, p):
    """The row range of every shard's slice."""
    if p < 1 or T % p:
        raise ValueError("p must divide the token count")
    r = T // p
    return [slice(i * r, (i + 1) * r) for i in range(p)]


def reduce_scatter(partials, residual_slices=None):
    """partials: sequence of p arrays [T, d].  Shard i's slice of sum_s partials[s] (summed in the
    order s = 0 .. p-1), plus residual_slices[i] when given."""
    p = len(partials)
    total = np.zeros_like(_f64(partials[0]))
    for part in partials:
        total = total + _f64(part)
    out = []
    for i, rows in enumerate(token_slices(total.shape[0], p)):
        y = total[rows]
        if residual_slices is not None:
            y = _f64(residual_slices[i]) + y
        out.append(y)
    return out


def all_gather(slices):
    """Concatenate the p slices in shard (token) order."""
    return np.concatenate([_f64(s) for s in slices], axis=0)


def collective_calls_per_layer(training=True, sequence_parallel=False):
    """Collectives of one layer: 2 all-reduces forward (attention, MLP) and 2 backward; with
    sequence parallelism each becomes a reduce-scatter and an all-gather."""
    all_reduces = 4 if training else 2
    return 2 * all_reduces if sequence_parallel else all_reduces


def ring_bytes_per_rank(n_bytes, p, sequence_parallel=False):
    """Bytes a rank sends for one block's collective on a ring of p ranks: an all-reduce sends
    2 (p-1)/p n; a reduce-scatter and an all-gather send (p-1)/p n each."""
    if sequence_parallel:
        return (p - 1) / p * n_bytes + (p - 1) / p * n_bytes
    return 2.0 * (p - 1) / p * n_bytes
