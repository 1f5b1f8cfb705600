"""The pages' reduction-count and message-size arithmetic (test infrastructure only).

Sources (page title, section):

* "Why tensor parallelism has to stay in scale-up" (keysight), "Where the 320 comes from":
  attention 1 forward + 1 backward reduction, MLP 1 forward + 1 backward, 4 x layers per
  micro-batch, independent of head count and hidden size; each message is one b x s x h
  activation; ring all-reduce moves 2(n-1)/n of the message per GPU; decode has no backward.
* "Tensor Parallelism" (klaylearn), Notes: ring all-reduce of n bytes over p ranks moves
  2 (p-1)/p n bytes per rank; T_ar ~ 2 (p-1)/p n / B + alpha 2 (p-1); decode payloads.
* Page 1 (llms-explorer), facts: 2 reductions per decoded layer for dense Llama / DeepSeek V3
  in mlx-lm, and the 61-layer count.
"""

FWD_REDUCES_PER_LAYER = 2   # attention output projection + MLP down projection
BWD_REDUCES_PER_LAYER = 2   # input gradient of the attention block + of the MLP block


def reductions_per_microbatch(layers, training=True):
    per_layer = FWD_REDUCES_PER_LAYER + (BWD_REDUCES_PER_LAYER if training else 0)
    return per_layer * layers


def reductions_per_token(layers):
    """Decode: forward only."""
    return reductions_per_microbatch(layers, training=False)


def message_bytes(b, s, h, dtype_bytes):
    """One reduction carries one b x s x h activation."""
    return b * s * h * dtype_bytes


def ring_bytes_per_rank(n_bytes, p):
    return 2.0 * (p - 1) / p * n_bytes


def ring_time_s(n_bytes, p, link_bytes_per_s, alpha_s=0.0):
    return ring_bytes_per_rank(n_bytes, p) / link_bytes_per_s + alpha_s * 2 * (p - 1)


def weight_stream_time_s(weight_bytes, hbm_bytes_per_s):
    """Decode with no batch reuse reads every weight once per token."""
    return weight_bytes / hbm_bytes_per_s
