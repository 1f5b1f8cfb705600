/*
 * tp_block.h -- C ABI of the tensor-parallel transformer block library (libtpblock.so).
 *
 * The library computes the Megatron-style tensor-parallel block on ONE GPU, with p as a logical
 * partition of the weights:
 *
 *   MLP  ("How does tensor parallelism split a transformer feed-forward block's two matmuls
 *         across devices?", sections "Column split, then row split", "The nonlinearity is free",
 *         "Second matmul, row-parallel", "One collective"; "Tensor Parallelism" (klaylearn), Notes,
 *         the column/row split paragraph):
 *     shard i owns the column slice W1_i (and Wu_i for the gated form) and the matching row slice
 *     W2_i;  h_i = act(x W1_i)  (column-parallel, activation local to the shard);
 *     y_i = h_i W2_i  (row-parallel: a full-shape partial sum);  y = sum_i y_i  (the all-reduce's
 *     arithmetic, done on the device in the fixed order i = 0 .. p-1 in fp32).
 *   Backward ("The backward pass"): dY is replicated (the exit's backward is the identity); every
 *     shard computes its own dW1_i, dW2_i with no exchange and a partial dx_i; dx = sum_i dx_i.
 *   Attention ("Tensor Parallelism", Notes, grouped-query paragraph): Q/K/V column-parallel so a
 *     shard owns n_q/p whole query heads and n_kv/p whole KV heads, attention runs locally over
 *     them, the output projection is row-parallel and the p partials are summed.
 *
 * Conventions for every call:
 *   - Every buffer is caller-owned device memory unless stated otherwise; the library allocates
 *     nothing.  Matrices are row-major and densely packed.  "stream" is a cudaStream_t (NULL = the
 *     legacy default stream); every call only enqueues work on it and returns without waiting.
 *   - bf16 data (TP_BF16) is accumulated in fp32; results are rounded once to bf16 (round to
 *     nearest even).  TP_F32 data is computed in fp32 throughout.
 *   - Arguments are validated before anything is enqueued; on any error nothing is written and
 *     the call returns a non-zero tp_status; tp_last_error() gives a message (per host thread).
 *   - No call traps or aborts.  Device-side waits are bounded; a wait that runs out records an
 *     error word that tp_check_device_error() reports as TP_ERR_TIMEOUT.
 *   - Weights are taken in the pages' orientation Y = X W, i.e. W[in][out] row-major, and packed
 *     once into a per-shard device layout (below) by the *_pack calls.
 */
#ifndef TP_BLOCK_H
#define TP_BLOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TP_OK = 0,
  TP_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative size, bad enum value          */
  TP_ERR_SHAPE = 2,         /* p does not divide d_ff, or n_q / n_kv; n_kv does not divide n_q  */
  TP_ERR_UNSUPPORTED = 3,   /* valid but not implemented combination                            */
  TP_ERR_WORKSPACE = 4,     /* workspace smaller than the *_workspace() query says              */
  TP_ERR_CUDA = 5,          /* a CUDA runtime call failed (message in tp_last_error)            */
  TP_ERR_TIMEOUT = 6        /* a bounded device-side wait ran out (tp_check_device_error)       */
} tp_status;

typedef enum { TP_F32 = 0, TP_BF16 = 1 } tp_dtype;

/* The elementwise nonlinearity between the two MLP matmuls ("The nonlinearity is free":
 * GELU, ReLU, or a gated variant computed from the same slice).  GELU is the exact erf form;
 * SWIGLU is h = silu(x Wg) * (x Wu) with silu(z) = z / (1 + exp(-z)). */
typedef enum { TP_ACT_IDENTITY = 0, TP_ACT_RELU = 1, TP_ACT_GELU = 2, TP_ACT_SWIGLU = 3 } tp_act;

/* How the p partial sums are added ("One collective").
 *   TP_REDUCE_SEPARATE: each shard's partial goes to fp32 workspace, then one vectorised
 *                       reduce kernel adds them (order 0..p-1) and rounds once.
 *   TP_REDUCE_FUSED:    the row-parallel GEMM adds the p shard partials of its output tile
 *                       in the same order without writing them to memory: for up to 128
 *                       tokens by a stream-K split over the shards' k-blocks, for more tokens
 *                       by running shard 0, 1, ..., p-1's k-blocks into one fp32 accumulator.
 *                       It applies to the forward's down / output projection and to the
 *                       backward's dx GEMM (tp_mlp_bwd, tp_attn_bwd).                          */
typedef enum { TP_REDUCE_SEPARATE = 0, TP_REDUCE_FUSED = 1 } tp_reduce_mode;

/* Descriptor flags.
 *   TP_FLAG_F32_RESIDUAL: y and residual are float32 (a float32 residual stream) while x and the
 *   weights stay in dtype.  The residual plus the sum of the partials is then rounded to fp32
 *   instead of bf16, so a deep stack of bf16 layers never rounds its skip path to bf16. */
#define TP_FLAG_F32_RESIDUAL 1

/* ------------------------------------------------------------------------------------------ */
/* MLP block                                                                                   */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  int64_t T;            /* tokens (rows of x); 0 is allowed (empty batch)                     */
  int64_t d;            /* hidden size                                                        */
  int64_t d_ff;         /* intermediate size F; must be a multiple of p                       */
  int32_t p;            /* logical shards, >= 1                                               */
  int32_t act;          /* tp_act                                                             */
  int32_t dtype;        /* tp_dtype of x, weights, y, dy, dx                                  */
  int32_t reduce_mode;  /* tp_reduce_mode                                                     */
  int32_t flags;        /* TP_FLAG_* (0 = none)                                               */
  float norm_eps;       /* eps of the RMSNorm written to y_norm (0 means 1e-5)                */
} tp_mlp_desc;

/* Packed layouts.  F_s = d_ff / p; F_sp = F_s rounded up to a multiple of 128 (padding rows and
 * columns are zero).  R = 2*F_sp for SWIGLU, else F_sp.  Element type = desc.dtype.
 *   w1p  [p][R][d]   SWIGLU: rows of shard i come in blocks of 256; rows 0..127 of block j hold
 *                    gate features f = j*128 + r (column i*F_s + f of Wg), rows 128..255 the same
 *                    features of Wu.  Other activations: row c of shard i is column i*F_s + c of
 *                    W1.  (Each row is one column of the user's matrix: K-major for x W1.)
 *   w2p  [p][d][F_sp] w2p[i][n][c] = W2[i*F_s + c][n]  (shard i's row slice, transposed).       */
size_t tp_mlp_w1_packed_bytes(const tp_mlp_desc* desc);
size_t tp_mlp_w2_packed_bytes(const tp_mlp_desc* desc);

/* Pack user weights into the per-shard layout.  w1 = W1 (or Wg) [d][d_ff]; w_up = Wu [d][d_ff]
 * for SWIGLU, NULL otherwise; w2 = W2 [d_ff][d].  All device pointers, element type desc.dtype.
 * One-time setup; not part of the steady-state step. */
tp_status tp_mlp_pack(const tp_mlp_desc* desc, const void* w1, const void* w_up, const void* w2,
                      void* w1p, void* w2p, void* stream);

/* Activations saved by the forward pass for the backward pass: z [T][p*R] (the pre-activations
 * in w1p's row order) followed by h [T][p*F_sp] (the activated values), element type dtype. */
size_t tp_mlp_saved_bytes(const tp_mlp_desc* desc);

/* Workspace of tp_mlp_fwd in bytes (its contents need not survive between calls). */
size_t tp_mlp_fwd_workspace(const tp_mlp_desc* desc);

/* Forward: y = residual + sum_{i=0}^{p-1} act(x W1_i) W2_i.
 *   x [T][d], y [T][d] (dtype; float32 with TP_FLAG_F32_RESIDUAL).  residual: NULL, or like y,
 *   added once after the sum (the residual add that follows the reduction and stays
 *   replicated).  residual may equal y.
 *   y_norm: NULL, or [T][d] dtype that receives RMSNorm(y) (unit weight, eps desc.norm_eps):
 *   the replicated normalization that follows the residual add, fused into the reduction.
 *   saved: NULL, or tp_mlp_saved_bytes() of device memory that receives z and h for
 *   tp_mlp_bwd.  Adds 1 to the reduction counter.
 *   Errors: TP_ERR_INVALID_ARG (null x/w1p/w2p/y/workspace with T>0, bad enum),
 *   TP_ERR_SHAPE (p < 1, d < 1, d_ff % p), TP_ERR_WORKSPACE (ws_bytes too small). */
tp_status tp_mlp_fwd(const tp_mlp_desc* desc, const void* x, const void* w1p, const void* w2p,
                     const void* residual, void* y, void* y_norm, void* saved, void* workspace,
                     size_t ws_bytes, void* stream);

/* Workspace of tp_mlp_bwd in bytes. */
size_t tp_mlp_bwd_workspace(const tp_mlp_desc* desc);

/* Backward from the replicated output gradient dy [T][d] (dtype), the forward's x and saved.
 *   dx  [T][d] dtype = sum_i dx_i (summed in order 0..p-1 in fp32, rounded once).
 *   dw1p, dw2p: fp32 gradients in the packed layouts of w1p / w2p, one slice per shard with no
 *   exchange between shards (padding entries are zero).  Adds 1 to the reduction counter. */
tp_status tp_mlp_bwd(const tp_mlp_desc* desc, const void* dy, const void* x, const void* saved,
                     const void* w1p, const void* w2p, void* dx, void* dw1p, void* dw2p,
                     void* workspace, size_t ws_bytes, void* stream);

/* tp_mlp_fwd for callers that cannot allocate device memory (the pages have no counterpart:
 * this is a deployment convenience, not part of the method).  Some callers cannot call
 * cudaMalloc -- a plug-in inside a host application that owns all device memory and gives its
 * plug-ins no allocator, or a latency-critical loop where an allocation, which may synchronize
 * the device, is not allowed.  This variant takes only inputs and outputs (same meaning as in
 * tp_mlp_fwd, no `saved`) and runs in scratch held in a fixed array of TP_MLP_STATIC_WS_BYTES
 * (32 MiB) of the library's own device memory, which every GPU that loads the library keeps
 * until exit.  It allocates nothing.
 *   - A shape whose tp_mlp_fwd_workspace() exceeds TP_MLP_STATIC_WS_BYTES returns
 *     TP_ERR_WORKSPACE before anything is enqueued (e.g. T <= 64 fits for d = 8192,
 *     d_ff = 28672, p = 8).
 *   - The first call on a device looks up the array's device address once for that device; make
 *     it before any stream capture.
 *   - All calls share the array: calls that overlap on the GPU race and must be serialised by
 *     the caller.  The array keeps the last call's contents; nothing in it needs to start at
 *     zero, since every scratch byte a call reads is written by that call first.
 * Same errors, results and reduction count as tp_mlp_fwd otherwise. */
#define TP_MLP_STATIC_WS_BYTES ((size_t)32 << 20)
tp_status tp_mlp_fwd_static_ws(const tp_mlp_desc* desc, const void* x, const void* w1p,
                               const void* w2p, const void* residual, void* y, void* stream);

/* Scatter packed fp32 gradients back to the user layout (fp32): dw1 [d][d_ff] (dWg for SWIGLU),
 * dw_up [d][d_ff] (SWIGLU only, else NULL), dw2 [d_ff][d]. */
tp_status tp_mlp_unpack_grads(const tp_mlp_desc* desc, const void* dw1p, const void* dw2p,
                              void* dw1, void* dw_up, void* dw2, void* stream);

/* ------------------------------------------------------------------------------------------ */
/* Attention block                                                                             */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  int64_t b;            /* sequences                                                          */
  int64_t s;            /* tokens per sequence in this call (1 for decode)                    */
  int64_t h;            /* hidden size                                                        */
  int32_t n_q;          /* query heads                                                        */
  int32_t n_kv;         /* key/value heads; must divide n_q                                   */
  int32_t head_dim;     /* multiple of 8, <= 256                                              */
  int32_t p;            /* logical shards; must divide n_q and n_kv (heads are never split)  */
  int32_t causal;       /* 1: query t sees keys <= t                                          */
  int32_t dtype;        /* tp_dtype                                                           */
  int64_t kv_len;       /* 0: self-attention over the s tokens.  > 0: decode (s must be 1) over
                           kv_len cached positions plus the new token                         */
  int64_t kv_cap;       /* slots per head in the caches (>= kv_len + 1); 0 means kv_len + 1  */
  int32_t reduce_mode;  /* tp_reduce_mode                                                     */
  int32_t flags;        /* TP_FLAG_* (0 = none)                                               */
  float norm_eps;       /* eps of the RMSNorm written to y_norm (0 means 1e-5)                */
  int32_t reserved;
} tp_attn_desc;

/* Packed layouts (element type dtype): qh = n_q/p, kh = n_kv/p, hd = head_dim,
 * R_a = (qh + 2*kh) * hd.
 *   wqkv_p [p][R_a][h]: shard i's rows are Wq columns i*qh*hd .. (qh*hd rows), then Wk columns
 *                       i*kh*hd .. (kh*hd rows), then Wv columns likewise.
 *   wo_p   [p][h][qh*hd]: wo_p[i][n][c] = Wo[i*qh*hd + c][n].                                 */
size_t tp_attn_wqkv_packed_bytes(const tp_attn_desc* desc);
size_t tp_attn_wo_packed_bytes(const tp_attn_desc* desc);

/* wq [h][n_q*hd], wk and wv [h][n_kv*hd], wo [n_q*hd][h]; device pointers, dtype. */
tp_status tp_attn_pack(const tp_attn_desc* desc, const void* wq, const void* wk, const void* wv,
                       const void* wo, void* wqkv_p, void* wo_p, void* stream);

size_t tp_attn_fwd_workspace(const tp_attn_desc* desc);

/* y = residual + sum_i Attn_i(x) Wo_i.  x [b][s][h] dtype; y and residual as in tp_mlp_fwd
 * (residual NULL or like y); y_norm NULL or [b][s][h] dtype receiving RMSNorm(y).
 * Query head j of shard i attends over KV head floor(j / (n_q/n_kv)); scale 1/sqrt(head_dim).
 * Decode (kv_len > 0, s == 1): k_cache and v_cache are [b][n_kv][kv_cap][hd] dtype; the new
 * token's key and value are written to slot kv_len and it attends to slots 0..kv_len.
 * Self-attention (kv_len == 0): caches may be NULL.  Adds 1 to the reduction counter. */
tp_status tp_attn_fwd(const tp_attn_desc* desc, const void* x, const void* wqkv_p,
                      const void* wo_p, void* k_cache, void* v_cache, const void* residual,
                      void* y, void* y_norm, void* workspace, size_t ws_bytes, void* stream);

/* Backward of the self-attention block (kv_len == 0; bf16 with h a multiple of 8; no flags).
 * ("Tensor Parallelism" (klaylearn), Notes: Q/K/V column-parallel, local attention, row-parallel
 * output projection; "How does tensor parallelism split a transformer feed-forward block's two
 * matmuls", "The backward pass": dY replicated, per-shard weight gradients with no exchange,
 * the input gradient summed from per-shard partials.)
 *   dy [b][s][h] bf16 = dL/dy (the output of tp_attn_fwd without residual);
 *   dx [b][s][h] bf16 = sum_i dx_i, summed in shard order in fp32 (adds 1 to the reduction
 *      counter);
 *   dwqkv_p, dwo_p: fp32 gradients of wqkv_p and wo_p in their packed per-shard layouts
 *      (tp_attn_wqkv_packed_bytes / tp_attn_wo_packed_bytes * 2 bytes; tp_attn_unpack_grads
 *      scatters them back), summed over the batch.
 * The forward's q, k, v, o and row log-sum-exp are recomputed from x inside the call (the
 * forward keeps no activations).  workspace: tp_attn_bwd_workspace(desc) bytes (0 for an
 * unsupported descriptor).  Returns TP_ERR_UNSUPPORTED for decode, fp32, flags or head_dim > 256. */
size_t tp_attn_bwd_workspace(const tp_attn_desc* desc);
tp_status tp_attn_bwd(const tp_attn_desc* desc, const void* x, const void* wqkv_p,
                      const void* wo_p, const void* dy, void* dx, void* dwqkv_p, void* dwo_p,
                      void* workspace, size_t ws_bytes, void* stream);

/* Scatter packed fp32 attention gradients back to the user layout (fp32): dwq [h][n_q*hd],
 * dwk and dwv [h][n_kv*hd], dwo [n_q*hd][h]. */
tp_status tp_attn_unpack_grads(const tp_attn_desc* desc, const void* dwqkv_p, const void* dwo_p,
                               void* dwq, void* dwk, void* dwv, void* dwo, void* stream);

/* ------------------------------------------------------------------------------------------ */
/* Reduction and glue                                                                          */
/* ------------------------------------------------------------------------------------------ */

/* out[j] = residual[j] + sum_{i=0}^{p-1} partials[i*n + j]: the all-reduce's arithmetic
 * ("One collective"; "Tensor Parallelism", Notes: Y = sum_i Z_i).  Summed in fp32 in the order
 * i = 0 .. p-1, residual (optional, out_dtype) added last, rounded once to out_dtype.
 * partials: [p][n] of in_dtype.  Adds 1 to the reduction counter. */
tp_status tp_reduce_partials(const void* partials, int32_t p, int64_t n, int32_t in_dtype,
                             const void* residual, void* out, int32_t out_dtype, void* stream);

/* Row-wise RMSNorm with unit weight: out = x / sqrt(mean(x^2) + eps), fp32 math, the
 * normalization that follows the residual add and stays replicated ("One collective").
 * x [rows][d] of x_dtype, out [rows][d] of out_dtype (out may equal x when the dtypes match). */
tp_status tp_rmsnorm(const void* x, int32_t x_dtype, int64_t rows, int64_t d, float eps,
                     void* out, int32_t out_dtype, void* stream);

/* ------------------------------------------------------------------------------------------ */
/* Mixture of experts                                                                          */
/* ------------------------------------------------------------------------------------------ */
/* "Tensor-parallel all-reduce count per transformer layer in MLX shard_linear" (llms-explorer),
 * facts on MoE layers: the router is replicated; the routed experts and the shared expert are
 * sharded in place; the block makes ONE sum of the shards' outputs (the shared expert's slice
 * folded in); the bias is added once, after the sum.  Readings: every expert is a SwiGLU block,
 * sharded over p like the dense MLP; a token takes the top_k experts with the largest router
 * logits (ties: lower index) weighted by the softmax of those k logits.
 *   y = residual + bias + sum_{i<p} [ shared_i(x) + sum_{j<k} w_j expert_{e_j,i}(x) ]
 * bf16 only; d and n_experts multiples of 8; top_k <= 8; p divides d_ff and d_ff_shared. */
typedef struct {
  int64_t T;            /* tokens                                                             */
  int64_t d;            /* hidden size                                                        */
  int64_t d_ff;         /* each routed expert's intermediate size                             */
  int64_t d_ff_shared;  /* the shared expert's intermediate size (0: no shared expert)        */
  int32_t n_experts;    /* E                                                                  */
  int32_t top_k;        /* experts per token                                                  */
  int32_t p;            /* logical shards                                                     */
  int32_t dtype;        /* TP_BF16                                                            */
  int32_t flags;        /* 0                                                                  */
  int32_t reserved;
} tp_moe_desc;

/* Packed bytes of ONE routed expert (the dense MLP's packed layout for d, d_ff, p, SWIGLU; the E
 * experts' packings lie back to back: w1p [E][...], w2p [E][...]) and of the shared expert. */
size_t tp_moe_expert_w1_bytes(const tp_moe_desc* desc);
size_t tp_moe_expert_w2_bytes(const tp_moe_desc* desc);
size_t tp_moe_shared_w1_bytes(const tp_moe_desc* desc);
size_t tp_moe_shared_w2_bytes(const tp_moe_desc* desc);

/* Pack the experts.  wg, wu, w2: HOST arrays of E device pointers to expert e's Wg, Wu [d][d_ff]
 * and W2 [d_ff][d] (bf16, input-major); wg_s, wu_s, w2_s: the shared expert (ignored when
 * d_ff_shared == 0).  w1p, w2p: E * tp_moe_expert_w{1,2}_bytes; w1p_s, w2p_s: the shared sizes.
 * The experts are packed in order; a null pointer inside the arrays is found when its expert
 * is reached (TP_ERR_INVALID_ARG), after the experts before it were enqueued. */
tp_status tp_moe_pack(const tp_moe_desc* desc, const void* const* wg, const void* const* wu,
                      const void* const* w2, const void* wg_s, const void* wu_s, const void* w2_s,
                      void* w1p, void* w2p, void* w1p_s, void* w2p_s, void* stream);

/* Forward of the MoE block.  x [T][d]; wr [d][E] router weights (bf16, replicated, not packed);
 * bias [d] and residual [T][d] optional; y [T][d] bf16.  route_idx (int32 [T][top_k]) and route_w
 * (fp32 [T][top_k]) receive the routing when non-null (descending logit order).  Routing,
 * dispatch, the grouped expert GEMMs, the shared expert and the one reduction all run on the
 * device; nothing is read back to the host.  workspace: tp_moe_fwd_workspace(desc) bytes.  Adds 1
 * to the reduction counter. */
size_t tp_moe_fwd_workspace(const tp_moe_desc* desc);
tp_status tp_moe_fwd(const tp_moe_desc* desc, const void* x, const void* wr, const void* w1p,
                     const void* w2p, const void* w1p_s, const void* w2p_s, const void* bias,
                     const void* residual, void* y, void* route_idx, void* route_w,
                     void* workspace, size_t ws_bytes, void* stream);

/* Backward of the MoE block: the chain rule through the forward above with the routing held
 * fixed (the top-k choice is constant wherever the k-th and (k+1)-th logits differ).
 *   routed row (t, j): d o = w_tj dy_t through expert e_tj; dw_tj = <dy_t, o_tj>;
 *   router: dl_t[e_tj] = w_tj (dw_tj - sum_i w_ti dw_ti), dWr = x^T dl, dx += dl Wr^T;
 *   shared expert: its MLP backward with dy.
 * dy [T][d] bf16, the gradient of y.  dx [T][d] bf16 receives the gradient through the routed
 * experts, the shared expert and the router, summed in that order in fp32 with one rounding (the
 * residual passes dy straight through and is not added; the bias gradient, the column sum of dy,
 * is not computed).  dwr [d][E] fp32.  dw1p, dw2p: fp32 gradients of the packed expert weights,
 * E * 2 * tp_moe_expert_w{1,2}_bytes bytes, expert e's at element offset e * w{1,2}p elements in
 * the packed layout of its weights (tp_mlp_unpack_grads with the dense desc {d, d_ff, p, SWIGLU}
 * unpacks it); an expert no token chose gets zeros.  dw1p_s, dw2p_s: the shared expert's, the
 * same way (ignored when d_ff_shared == 0).  The routing and the expert activations are
 * recomputed from x.  The routed experts' GEMMs run expert by expert, so the call reads the E
 * per-expert row counts back to the host once (it synchronises the stream and cannot be
 * captured in a CUDA graph).  workspace: tp_moe_bwd_workspace(desc) bytes. */
size_t tp_moe_bwd_workspace(const tp_moe_desc* desc);
tp_status tp_moe_bwd(const tp_moe_desc* desc, const void* x, const void* wr, const void* w1p,
                     const void* w2p, const void* w1p_s, const void* w2p_s, const void* dy,
                     void* dx, float* dwr, float* dw1p, float* dw2p, float* dw1p_s,
                     float* dw2p_s, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------ */
/* Sequence parallelism                                                                        */
/* ------------------------------------------------------------------------------------------ */
/* "Why tensor parallelism has to stay in scale-up" (Keysight), "Where the 320 comes from": with
 * sequence parallelism each all-reduce becomes a reduce-scatter plus an all-gather, moving the
 * same bytes.  Between the row-parallel output of one block and the column-parallel input of the
 * next, shard i owns token rows i*T/p .. (i+1)*T/p - 1 of the [T][d] activation (a "slice"),
 * and the residual add and normalisation run on the slices.  Here every slice is its own device
 * buffer [T/p][d]: the slice arguments are HOST arrays of p device pointers (p <= 64), each
 * 16-byte aligned for the vectorised path (any alignment works).  p must divide T; a violation
 * returns TP_ERR_SHAPE.  The block calls accept only TP_REDUCE_SEPARATE (TP_ERR_UNSUPPORTED
 * otherwise). */

/* Reduce-scatter: out_slices[i][r] = residual_slices[i][r] + sum_{s=0}^{p-1} partials[s][i*T/p + r]
 * (fp32 in shard order, residual last, one rounding to out_dtype); with norm_slices, also
 * norm_slices[i][r] = RMSNorm(out_slices[i][r]) (unit weight; norm_dtype) computed from the
 * stored values.  eps is used exactly as given, as in tp_rmsnorm (0 is allowed and means no eps;
 * a negative or NaN eps returns TP_ERR_INVALID_ARG).  partials: [p][T][d] fp32.  residual_slices
 * and norm_slices may be NULL.  Adds 1 to the reduction counter. */
tp_status tp_reduce_scatter_partials(const void* partials, int32_t p, int64_t T, int64_t d,
                                     void* const* residual_slices, void* const* out_slices,
                                     int32_t out_dtype, void* const* norm_slices,
                                     int32_t norm_dtype, float eps, void* stream);

/* All-gather: out[i*rows_per_slice + r] = slices[i][r]; out is [p*rows_per_slice][d] of dtype. */
tp_status tp_all_gather_slices(const void* const* slices, int32_t p, int64_t rows_per_slice,
                               int64_t d, int32_t dtype, void* out, void* stream);

/* MLP forward, sequence-parallel.  The p slices of x ([T/p][d], dtype) are all-gathered, then
 * the block runs as in tp_mlp_fwd (the same packed weights and saved activations).  The partials
 * are then reduce-scattered into y_slices ([T/p][d], dtype, or fp32 with TP_FLAG_F32_RESIDUAL),
 * adding residual_slices (optional).  y_norm_slices (optional) receive RMSNorm of the y rows
 * (norm_eps).  workspace: tp_mlp_fwd_sp_workspace(desc) bytes (0 for an unsupported
 * descriptor).  Adds 1 to the reduction counter. */
size_t tp_mlp_fwd_sp_workspace(const tp_mlp_desc* desc);
tp_status tp_mlp_fwd_sp(const tp_mlp_desc* desc, const void* const* x_slices, const void* w1p,
                        const void* w2p, void* const* residual_slices, void* const* y_slices,
                        void* const* y_norm_slices, void* saved, void* workspace,
                        size_t ws_bytes, void* stream);

/* MLP backward, sequence-parallel.  The dy and x slices are all-gathered (the reduce-scatter's
 * gradient is an all-gather), and the backward runs as in tp_mlp_bwd.  The dx partials are then
 * reduce-scattered into dx_slices ([T/p][d], dtype; the all-gather's gradient).  dw1p and dw2p
 * are as in tp_mlp_bwd.  saved is the forward's saved activations.  workspace:
 * tp_mlp_bwd_sp_workspace(desc) bytes.  Adds 1 to the reduction counter. */
size_t tp_mlp_bwd_sp_workspace(const tp_mlp_desc* desc);
tp_status tp_mlp_bwd_sp(const tp_mlp_desc* desc, const void* const* dy_slices,
                        const void* const* x_slices, const void* saved, const void* w1p,
                        const void* w2p, void* const* dx_slices, void* dw1p, void* dw2p,
                        void* workspace, size_t ws_bytes, void* stream);

/* Attention forward, sequence-parallel over the b*s token rows.  It all-gathers the x slices
 * ([b*s/p][h]), runs tp_attn_fwd's block (KV caches as there), then reduce-scatters the output
 * partials into y_slices with residual_slices and y_norm_slices as in tp_mlp_fwd_sp.
 * workspace: tp_attn_fwd_sp_workspace(desc) bytes.  Adds 1 to the reduction counter. */
size_t tp_attn_fwd_sp_workspace(const tp_attn_desc* desc);
tp_status tp_attn_fwd_sp(const tp_attn_desc* desc, const void* const* x_slices,
                         const void* wqkv_p, const void* wo_p, void* k_cache, void* v_cache,
                         void* const* residual_slices, void* const* y_slices,
                         void* const* y_norm_slices, void* workspace, size_t ws_bytes,
                         void* stream);

/* Attention backward, sequence-parallel (self-attention, bf16, as tp_attn_bwd).  The x and dy
 * slices ([b*s/p][h]) are all-gathered (the reduce-scatter's gradient is an all-gather), the
 * backward runs as in tp_attn_bwd, and the dx partials are reduce-scattered into dx_slices (the
 * all-gather's gradient).  dwqkv_p and dwo_p as in tp_attn_bwd.  Takes TP_REDUCE_SEPARATE only.
 * workspace: tp_attn_bwd_sp_workspace(desc) bytes (0 for an unsupported descriptor).  Adds 1 to
 * the reduction counter. */
size_t tp_attn_bwd_sp_workspace(const tp_attn_desc* desc);
tp_status tp_attn_bwd_sp(const tp_attn_desc* desc, const void* const* x_slices,
                         const void* wqkv_p, const void* wo_p, const void* const* dy_slices,
                         void* const* dx_slices, void* dwqkv_p, void* dwo_p, void* workspace,
                         size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------ */
/* One shard per device                                                                        */
/* ------------------------------------------------------------------------------------------ */
/* "Tensor Parallelism" (klaylearn), Notes, and "How does tensor parallelism split a transformer
 * feed-forward block's two matmuls", "One collective" and "The backward pass": with one shard per
 * GPU, device i holds only shard i's slices -- the columns i*F_s .. of W1 (and Wu) and the
 * matching rows of W2; its n_q/p query heads and n_kv/p KV heads (columns of Wq, Wk, Wv, rows of
 * Wo) and its own KV cache -- computes its full-shape partial, and the devices' all-reduce (the
 * caller's collective, e.g. NCCL) adds the p partials.  Backward: dy is replicated, each device
 * keeps its weight gradients (no exchange) and its dx partial is all-reduced.
 * Shard i is the block with p = 1 and d_ff/p features (n_q/p, n_kv/p heads); its packed layout
 * equals shard i's slice of the p-shard packing above (so w1p + i * size and the like also work
 * on one device).  desc describes the whole block (its p, d_ff, heads); `shard` is in 0 .. p-1;
 * desc.flags must be 0.  The partial ([T][d], or [b][s][h]) is written in partial_dtype: TP_F32
 * or TP_BF16 (TP_F32 only for fp32 blocks).  These calls do no reduction and add nothing to the
 * reduction counter; the residual add that follows the all-reduce is tp_reduce_partials with
 * p = 1 on the summed partial. */
typedef struct {
  size_t col_weight_bytes;  /* packed column-parallel weights of one shard (w1p / wqkv slice)  */
  size_t row_weight_bytes;  /* packed row-parallel weights of one shard (w2p / wo slice)       */
  size_t saved_bytes;       /* MLP: activations tp_mlp_fwd_shard saves for tp_mlp_bwd_shard     */
  size_t fwd_workspace;     /* workspace of the *_fwd_shard call                              */
  size_t bwd_workspace;     /* workspace of the *_bwd_shard call (0: not supported)           */
  size_t partial_bytes;     /* one partial                                                    */
} tp_shard_sizes;

tp_status tp_mlp_shard_sizes(const tp_mlp_desc* desc, int32_t partial_dtype, tp_shard_sizes* out);
/* Pack shard `shard`'s slice from the user's full W1 / Wu [d][d_ff] and W2 [d_ff][d] (device
 * pointers, dtype) into w1p_shard / w2p_shard (col/row_weight_bytes). */
tp_status tp_mlp_pack_shard(const tp_mlp_desc* desc, int32_t shard, const void* w1,
                            const void* w_up, const void* w2, void* w1p_shard, void* w2p_shard,
                            void* stream);
/* partial = act(x W1_i) W2_i  [T][d].  saved_shard: NULL or saved_bytes for tp_mlp_bwd_shard. */
tp_status tp_mlp_fwd_shard(const tp_mlp_desc* desc, int32_t shard, int32_t partial_dtype,
                           const void* x, const void* w1p_shard, const void* w2p_shard,
                           void* partial, void* saved_shard, void* workspace, size_t ws_bytes,
                           void* stream);
/* dx_partial = dx_i [T][d] (partial_dtype); dw1p_shard / dw2p_shard: this shard's fp32 weight
 * gradients in its packed layout (no exchange). */
tp_status tp_mlp_bwd_shard(const tp_mlp_desc* desc, int32_t shard, int32_t partial_dtype,
                           const void* dy, const void* x, const void* saved_shard,
                           const void* w1p_shard, const void* w2p_shard, void* dx_partial,
                           void* dw1p_shard, void* dw2p_shard, void* workspace, size_t ws_bytes,
                           void* stream);

tp_status tp_attn_shard_sizes(const tp_attn_desc* desc, int32_t partial_dtype,
                              tp_shard_sizes* out);
/* Pack shard `shard`'s slice from the user's full wq [h][n_q*hd], wk, wv [h][n_kv*hd] and
 * wo [n_q*hd][h]. */
tp_status tp_attn_pack_shard(const tp_attn_desc* desc, int32_t shard, const void* wq,
                             const void* wk, const void* wv, const void* wo, void* wqkv_shard,
                             void* wo_shard, void* stream);
/* partial = Attn_i(x) Wo_i  [b][s][h].  Decode (desc.kv_len > 0): k_cache_shard / v_cache_shard
 * are this shard's caches [b][n_kv/p][kv_cap][hd]; the new token is appended there. */
tp_status tp_attn_fwd_shard(const tp_attn_desc* desc, int32_t shard, int32_t partial_dtype,
                            const void* x, const void* wqkv_shard, const void* wo_shard,
                            void* k_cache_shard, void* v_cache_shard, void* partial,
                            void* workspace, size_t ws_bytes, void* stream);
/* Self-attention backward of one shard (bf16; as tp_attn_bwd): dx_partial [b][s][h] bf16,
 * dwqkv_shard / dwo_shard fp32 in the shard's packed layout. */
tp_status tp_attn_bwd_shard(const tp_attn_desc* desc, int32_t shard, const void* x,
                            const void* wqkv_shard, const void* wo_shard, const void* dy,
                            void* dx_partial, void* dwqkv_shard, void* dwo_shard,
                            void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------ */
/* Diagnostics                                                                                 */
/* ------------------------------------------------------------------------------------------ */

/* Reductions of p partials enqueued so far (one per tp_mlp_fwd / tp_mlp_bwd / tp_attn_fwd /
 * tp_attn_bwd / tp_reduce_partials call that succeeded, and one per reduce-scatter of the
 * sequence-parallel calls), process-wide. */
uint64_t tp_reduction_count(void);
void tp_reset_reduction_count(void);

/* Kernels this library has launched so far, process-wide. */
uint64_t tp_launch_count(void);

/* Message of the last failed call on this host thread ("" if none). */
const char* tp_last_error(void);
const char* tp_status_string(int32_t status);

/* Waits for the stream, then reports (and clears) the device error word: TP_ERR_TIMEOUT if a
 * bounded device wait ran out since the last check, TP_ERR_CUDA on a CUDA error, else TP_OK. */
tp_status tp_check_device_error(void* stream);

/* 1 if this build contains the sm_100a tensor-core kernels and the current device runs them. */
int32_t tp_tensor_core_path_available(void);

/* Failure-detection self-test (the pages have no counterpart; it exercises the timeout path
 * behind TP_ERR_TIMEOUT without any fault).  Enqueues one small kernel that waits, through the
 * same bounded mbarrier wait the tensor-core kernels use, on a barrier that nothing completes,
 * then through the bounded cross-CTA counter wait of the one-launch decode MLP on a counter that
 * nothing increments; after limit_us microseconds (1 .. 1000000) each wait gives up and records
 * its site in the device error word (bits 1 and 32), and the kernel returns.  A following tp_check_device_error() reports TP_ERR_TIMEOUT
 * and clears the word; the CUDA context stays usable.  Returns TP_ERR_INVALID_ARG for a limit
 * out of range (checked before anything is enqueued). */
tp_status tp_selftest_wait_timeout(uint32_t limit_us, void* stream);

/* Per-kernel timing.  While enabled, every kernel the library launches is bracketed by two CUDA
 * events recorded on the launching stream (skipped while the stream is being captured into a
 * graph).  tp_profile_read synchronizes the device and returns, for entry i (0-based, in order
 * of first appearance), the kernel label, its launch count and the summed event time in ms;
 * it returns 0 once i is past the last entry.  tp_profile_reset drops all records. */
void tp_profile_enable(int32_t on);
int32_t tp_profile_read(int32_t i, char* label, int32_t label_len, uint64_t* launches,
                        double* total_ms);
/* Duration in ms of launch j (0-based, in launch order) of entry i of tp_profile_read; returns 1,
 * or 0 when i or j is out of range.  Synchronizes the device.  Gives the distribution of one
 * kernel's launches, e.g. the latency of every reduction in a decoded token. */
int32_t tp_profile_read_launch(int32_t i, int64_t j, double* ms);
void tp_profile_reset(void);

/* Library version, major*10000 + minor*100 + patch. */
int32_t tp_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TP_BLOCK_H */
