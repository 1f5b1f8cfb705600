"""Tensor parallelism with one shard per GPU.

"Tensor Parallelism" (klaylearn), Notes: shard i of the column-parallel weights (and the matching
rows of the row-parallel ones) lives on device i, each device computes a full-shape partial, and
an all-reduce adds the partials; "How does tensor parallelism split a transformer feed-forward
block's two matmuls", "One collective" and "The backward pass": one all-reduce per block forward
(on y) and one backward (on dx), weight gradients stay on their device.  "Why tensor parallelism
has to stay in scale-up", "Where the 320 comes from": two reductions per layer forward and two
backward.

Rank r of the process group holds shard r (p = the group's size).  Each block here

* packs only its own shard from the full user weights (``tp_*_pack_shard``),
* computes its partial with the library's shard call (``tp_*_fwd_shard`` / ``tp_*_bwd_shard``;
  every step of the block runs in the library's kernels),
* sums the partials with the group's all-reduce (NCCL over NVLink on GPUs), then
* adds the residual once to the sum (``tp_reduce_partials`` with p = 1, one rounding).

The collective is torch.distributed's; ``TPGroup`` counts the all-reduces and, when asked,
times each one with CUDA events on the current stream (the per-collective latency).  The shard
arithmetic never leaves the library: ``lib`` defaults to the C-ABI binding, which raises if the
library is missing.  Tests on CPU pass a stand-in ``lib`` so that the orchestration (shard
ownership, the collective, the counts) can run on gloo ranks without a GPU.
"""

import torch
import torch.distributed as dist


class TPGroup:
    """The process group of one tensor-parallel block: rank r holds shard r."""

    def __init__(self, group=None, timing=False):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.count = 0
        self.timing = timing
        self._events = []

    def all_reduce(self, t):
        """Sum ``t`` over the group in place (the block's one collective)."""
        self.count += 1
        if self.timing and t.is_cuda:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
            b.record()
            self._events.append((a, b))
        else:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
        return t

    def latencies_ms(self):
        """Durations of the timed all-reduces so far (synchronizes), then forgets them."""
        if not self._events:
            return []
        torch.cuda.synchronize()
        out = [a.elapsed_time(b) for a, b in self._events]
        self._events = []
        return out


def _lib(lib):
    if lib is not None:
        return lib
    from . import tpblock
    tpblock.load()
    return tpblock


def _bytes(n, device):
    return torch.empty(max(int(n), 1), dtype=torch.uint8, device=device)


class ShardedMLP:
    """The MLP block with this rank's shard: y = residual + all_reduce(act(x W1_r) W2_r)."""

    def __init__(self, group, T, d, d_ff, act="swiglu", dtype="bf16", partial_dtype=torch.float32,
                 device=None, lib=None):
        self.g = group
        self.lib = _lib(lib)
        self.shard = group.rank
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.T, self.d = T, d
        self.dtype = dtype
        self.desc = self.lib.mlp_desc(T, d, d_ff, group.world, act, dtype)
        self.partial_dtype = partial_dtype
        sz = self.lib.tp_mlp_shard_sizes(self.desc, partial_dtype)
        self.sizes = sz
        self.w1p = _bytes(sz.col_weight_bytes, self.device)
        self.w2p = _bytes(sz.row_weight_bytes, self.device)
        self.saved = _bytes(sz.saved_bytes, self.device)
        self.ws_f = _bytes(sz.fwd_workspace, self.device)
        self.ws_b = _bytes(sz.bwd_workspace, self.device)
        self.partial = torch.empty(T, d, dtype=partial_dtype, device=self.device)
        self.dx_partial = torch.empty(T, d, dtype=partial_dtype, device=self.device)
        self.dw1p = _bytes(sz.col_weight_bytes * 4 // _elem(dtype), self.device)
        self.dw2p = _bytes(sz.row_weight_bytes * 4 // _elem(dtype), self.device)

    def pack(self, w1, w_up, w2):
        """Pack this rank's shard from the full user weights W1 (Wg), Wu [d][d_ff], W2 [d_ff][d]."""
        self.lib.tp_mlp_pack_shard(self.desc, self.shard, w1, w_up, w2, self.w1p, self.w2p)

    def forward(self, x, residual=None, out=None):
        self.lib.tp_mlp_fwd_shard(self.desc, self.shard, x, self.w1p, self.w2p, self.partial,
                                  saved=self.saved, workspace=self.ws_f)
        self.g.all_reduce(self.partial)
        return _finish(self.lib, self.partial, residual, out, self.dtype)

    def backward(self, dy, x, out=None):
        """dx = all_reduce(dx_r); this rank's fp32 weight gradients land in dw1p / dw2p."""
        self.lib.tp_mlp_bwd_shard(self.desc, self.shard, dy, x, self.saved, self.w1p, self.w2p,
                                  self.dx_partial, self.dw1p, self.dw2p, workspace=self.ws_b)
        self.g.all_reduce(self.dx_partial)
        return _finish(self.lib, self.dx_partial, None, out, self.dtype)


class ShardedAttention:
    """The GQA attention block with this rank's n_q/p query heads and n_kv/p KV heads (and, for
    decode, its own KV cache [b][n_kv/p][kv_cap][hd]): y = residual + all_reduce(Attn_r(x) Wo_r)."""

    def __init__(self, group, b, s, h, n_q, n_kv, head_dim, causal=True, dtype="bf16", kv_len=0,
                 kv_cap=0, partial_dtype=torch.float32, device=None, lib=None):
        self.g = group
        self.lib = _lib(lib)
        self.shard = group.rank
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.shape = (b, s, h)
        self.dtype = dtype
        self.desc = self.lib.attn_desc(b, s, h, n_q, n_kv, head_dim, group.world, causal, dtype,
                                       kv_len, kv_cap=kv_cap)
        sz = self.lib.tp_attn_shard_sizes(self.desc, partial_dtype)
        self.sizes = sz
        self.wqkv = _bytes(sz.col_weight_bytes, self.device)
        self.wo = _bytes(sz.row_weight_bytes, self.device)
        self.ws_f = _bytes(sz.fwd_workspace, self.device)
        self.ws_b = _bytes(sz.bwd_workspace, self.device)
        self.partial = torch.empty(b, s, h, dtype=partial_dtype, device=self.device)
        self.dx_partial = None
        self.dwqkv = self.dwo = None

    def pack(self, wq, wk, wv, wo):
        self.lib.tp_attn_pack_shard(self.desc, self.shard, wq, wk, wv, wo, self.wqkv, self.wo)

    def forward(self, x, k_cache=None, v_cache=None, residual=None, out=None):
        self.lib.tp_attn_fwd_shard(self.desc, self.shard, x, self.wqkv, self.wo, self.partial,
                                   k_cache=k_cache, v_cache=v_cache, workspace=self.ws_f)
        self.g.all_reduce(self.partial)
        return _finish(self.lib, self.partial, residual, out, self.dtype)

    def backward(self, x, dy, out=None):
        """Self-attention backward: dx = all_reduce(dx_r) (bf16 partials); this rank's fp32
        weight gradients land in dwqkv / dwo."""
        if self.dx_partial is None:
            self.dx_partial = torch.empty(*self.shape, dtype=torch.bfloat16, device=self.device)
            self.dwqkv = _bytes(self.sizes.col_weight_bytes * 2, self.device)
            self.dwo = _bytes(self.sizes.row_weight_bytes * 2, self.device)
        self.lib.tp_attn_bwd_shard(self.desc, self.shard, x, self.wqkv, self.wo, dy,
                                   self.dx_partial, self.dwqkv, self.dwo, workspace=self.ws_b)
        self.g.all_reduce(self.dx_partial)
        return _finish(self.lib, self.dx_partial, None, out, self.dtype)


def _elem(dtype):
    return 2 if dtype == "bf16" else 4


_TORCH = {"bf16": torch.bfloat16, "f32": torch.float32}


def _finish(lib, summed, residual, out, dtype):
    """out = residual + summed, one rounding to the block's dtype (or the residual's)."""
    if residual is None and out is None and summed.dtype == _TORCH.get(dtype, summed.dtype):
        return summed
    if out is None:
        out_dtype = residual.dtype if residual is not None else _TORCH.get(dtype, summed.dtype)
        out = torch.empty(summed.shape, dtype=out_dtype, device=summed.device)
    lib.tp_reduce_partials(summed, 1, summed.numel(), out, residual=residual)
    return out
