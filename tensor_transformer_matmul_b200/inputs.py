"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws numbers: it holds none of the block's arithmetic.  Every tensor is
``N(0, std)`` drawn in float32 by a ``torch.Generator`` seeded from (seed, stream id), scaled,
then rounded to the storage dtype (round-to-nearest-even for bf16).  Small cases are drawn on the
CPU; full-size cases are drawn on the GPU (``device="cuda"``) because tens of GB of weights cannot
be drawn on the host in reasonable time.  The draws are a function of (seed, stream, shape,
device), so both sides of a parity check always receive identical bytes: the oracle gets a host
copy of the very tensors the GPU path reads.

Stream ids fix the draw order of each workload: x, W1 (or Wg), Wu, W2, dY for the MLP;
x, Wq, Wk, Wv, Wo, K cache, V cache for attention.
"""

import torch

# stream ids (one independent generator per tensor role)
S_X, S_W1, S_WU, S_W2, S_DY = 1, 2, 3, 4, 5
S_WQ, S_WK, S_WV, S_WO, S_KC, S_VC = 11, 12, 13, 14, 15, 16

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def normal(shape, std, seed, stream, dtype="bf16", device="cpu"):
    """N(0, std) tensor of ``shape``; ``dtype`` in {"f32", "bf16"}."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(TORCH_DTYPE[dtype])


def mlp_inputs(T, d, F, act, dtype="bf16", seed=0, device="cpu", w_std=None, backward=False,
               layer=0):
    """Inputs of one MLP block.  ``w_std=None`` means N(0, 1/sqrt(fan_in)) (fan_in = d for
    W1/Wu, F for W2); otherwise every weight is N(0, w_std).  x and dY are N(0, 1)."""
    base = seed + 7919 * layer
    s1 = (1.0 / d ** 0.5) if w_std is None else w_std
    s2 = (1.0 / F ** 0.5) if w_std is None else w_std
    out = {
        "x": normal((T, d), 1.0, base, S_X, dtype, device),
        "w1": normal((d, F), s1, base, S_W1, dtype, device),
        "w_up": normal((d, F), s1, base, S_WU, dtype, device) if act == "swiglu" else None,
        "w2": normal((F, d), s2, base, S_W2, dtype, device),
    }
    if backward:
        out["dy"] = normal((T, d), 1.0, base, S_DY, dtype, device)
    return out


def attn_inputs(b, s, h, n_q, n_kv, head_dim, dtype="bf16", seed=0, device="cpu", w_std=0.02,
                kv_len=0, layer=0):
    """Inputs of one attention block.  With ``kv_len > 0`` the K/V caches are
    (b, n_kv, kv_len + 1, head_dim) N(0, 1) tensors whose last slot is overwritten by the call."""
    base = seed + 7919 * layer
    out = {
        "x": normal((b, s, h), 1.0, base, S_X, dtype, device),
        "wq": normal((h, n_q * head_dim), w_std, base, S_WQ, dtype, device),
        "wk": normal((h, n_kv * head_dim), w_std, base, S_WK, dtype, device),
        "wv": normal((h, n_kv * head_dim), w_std, base, S_WV, dtype, device),
        "wo": normal((n_q * head_dim, h), w_std, base, S_WO, dtype, device),
    }
    if kv_len > 0:
        out["k_cache"] = normal((b, n_kv, kv_len + 1, head_dim), 1.0, base, S_KC, dtype, device)
        out["v_cache"] = normal((b, n_kv, kv_len + 1, head_dim), 1.0, base, S_VC, dtype, device)
    return out


def to_f64(t):
    """Host float64 numpy copy of a tensor (exact for bf16 and f32)."""
    return t.detach().to("cpu", torch.float64).numpy()
