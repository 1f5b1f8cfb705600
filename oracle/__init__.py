"""Oracle: a plain, slow, CPU float64 reference of the UNSHARDED tensor-parallel block.

This package is test infrastructure. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The product path
(the CUDA library and its Python binding) never imports, calls or links anything here, and
nothing here imports the product path.

What it computes, and where the method is stated:

* ``mlp``       -- y = act(x W1) W2 and its chain-rule backward, unsharded
                   ("How does tensor parallelism split a transformer feed-forward block's two
                   matmuls", sections "The shape of the block" and "The backward pass";
                   "Tensor Parallelism", Notes, the column/row split paragraph).
* ``attention`` -- grouped-query scaled-dot-product attention with Q/K/V/O projections
                   ("Tensor Parallelism", Notes, the grouped-query attention paragraph).
* ``decode``    -- one Llama-shaped decode layer (pre-RMSNorm, attention, residual, pre-RMSNorm,
                   SwiGLU MLP, residual) with a KV cache ("How does tensor parallelism split ...",
                   "One collective": the residual add and the following normalization stay
                   replicated).
* ``costmodel`` -- the pages' reduction-count and message-byte arithmetic.
* ``moe``       -- the tensor-parallel mixture-of-experts block: replicated top-k router, SwiGLU
                   experts and shared expert sharded in place, one block-level sum, bias once
                   ("Tensor-parallel all-reduce count per transformer layer in MLX shard_linear",
                   facts on MoE layers).
* ``seqpar``    -- the sequence-parallel form of the collective: reduce-scatter of the partials
                   into token slices and all-gather of the slices ("Why tensor parallelism has to
                   stay in scale-up", "Where the 320 comes from").

Each function also has a *sharded reference mode* (loop over the p shards and add the partial
results in order) used only by the invariant tests that check "the sharded sum equals the
unsharded result".

Everything is float64 numpy; matrix products use numpy's matmul as a library primitive, and the
error function comes from scipy.  No blocking, fusion or reordering beyond the stated formulas.
"""

from . import mlp, attention, decode, costmodel, seqpar, moe  # noqa: F401
