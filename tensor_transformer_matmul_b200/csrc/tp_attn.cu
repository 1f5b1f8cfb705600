// Tensor-parallel grouped-query attention block.
//   "Tensor Parallelism" (klaylearn), Notes, grouped-query paragraph: per shard n_q/p query heads
//   and n_kv/p KV heads (column-parallel Q/K/V), local attention, row-parallel output projection
//   giving a full-width partial, partials summed.
#include "attn.cuh"

extern "C" size_t tp_attn_wqkv_packed_bytes(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  return tp::attn_layout_of(desc, &L) == TP_OK ? L.wqkv_bytes : 0;
}
extern "C" size_t tp_attn_wo_packed_bytes(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  return tp::attn_layout_of(desc, &L) == TP_OK ? L.wo_bytes : 0;
}
extern "C" size_t tp_attn_fwd_workspace(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  return tp::attn_layout_of(desc, &L) == TP_OK ? L.ws_bytes : 0;
}

extern "C" tp_status tp_attn_pack(const tp_attn_desc* desc, const void* wq, const void* wk,
                                  const void* wv, const void* wo, void* wqkv_p, void* wo_p,
                                  void* stream) {
  tp::clear_error();
  tp::AttnLayout L;
  tp_status st = tp::attn_layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (!wq || !wk || !wv || !wo || !wqkv_p || !wo_p)
    return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  return tp::attn_pack(L, wq, wk, wv, wo, wqkv_p, wo_p, static_cast<cudaStream_t>(stream));
}

extern "C" tp_status tp_attn_fwd(const tp_attn_desc* desc, const void* x, const void* wqkv_p,
                                 const void* wo_p, void* k_cache, void* v_cache,
                                 const void* residual, void* y, void* y_norm, void* workspace,
                                 size_t ws_bytes, void* stream) {
  tp::clear_error();
  tp::AttnLayout L;
  tp_status st = tp::attn_layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (desc->reduce_mode == TP_REDUCE_FUSED && !L.tc)
    return tp::set_error(TP_ERR_UNSUPPORTED,
                         "TP_REDUCE_FUSED needs the tensor-core path (bf16, h a multiple of 8)");
  if (L.tokens == 0) {
    tp::count_reduction();
    return TP_OK;
  }
  if (!x || !wqkv_p || !wo_p || !y) return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (L.kv_len > 0 && (!k_cache || !v_cache))
    return tp::set_error(TP_ERR_INVALID_ARG, "decode needs k_cache and v_cache");
  if (L.kv_len > 0 && ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15))
    return tp::set_error(TP_ERR_INVALID_ARG, "k_cache and v_cache must be 16-byte aligned");
  if (!workspace) return tp::set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < L.ws_bytes) return tp::set_error(TP_ERR_WORKSPACE, "workspace too small");
  st = tp::attn_forward(L, x, wqkv_p, wo_p, k_cache, v_cache, residual, y, y_norm, workspace,
                        static_cast<cudaStream_t>(stream));
  if (st == TP_OK) tp::count_reduction();
  return st;
}

// Sequence-parallel forward: the input arrives as the p shards' token slices and is all-gathered
// before the QKV GEMM; the output partials are reduce-scattered into the slices (with the residual
// add and the RMSNorm on the slices).  "Why tensor parallelism has to stay in scale-up"
// (Keysight), "Where the 320 comes from".
namespace {
size_t sp_act_bytes(const tp::AttnLayout& L) {
  return tp::align256(static_cast<size_t>(L.tokens * L.h) * tp::elem_bytes(L.dtype));
}
tp_status sp_layout(const tp_attn_desc* desc, tp::AttnLayout* L) {
  tp_status st = tp::attn_layout_of(desc, L);
  if (st != TP_OK) return st;
  if (desc->reduce_mode != TP_REDUCE_SEPARATE)
    return tp::set_error(TP_ERR_UNSUPPORTED,
                         "the sequence-parallel calls reduce-scatter the partials: use TP_REDUCE_SEPARATE");
  if (L->p > tp::seqpar::kMaxSlices) return tp::set_error(TP_ERR_SHAPE, "p must be <= 64 for slices");
  if (L->tokens % L->p) return tp::set_error(TP_ERR_SHAPE, "sequence parallelism needs p to divide b*s");
  return TP_OK;
}
}  // namespace

extern "C" size_t tp_attn_fwd_sp_workspace(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  if (sp_layout(desc, &L) != TP_OK) return 0;
  return sp_act_bytes(L) + L.ws_bytes;
}

extern "C" tp_status tp_attn_fwd_sp(const tp_attn_desc* desc, const void* const* x_slices,
                                    const void* wqkv_p, const void* wo_p, void* k_cache,
                                    void* v_cache, void* const* residual_slices,
                                    void* const* y_slices, void* const* y_norm_slices,
                                    void* workspace, size_t ws_bytes, void* stream) {
  tp::clear_error();
  tp::AttnLayout L;
  tp_status st = sp_layout(desc, &L);
  if (st != TP_OK) return st;
  if (L.tokens == 0) {
    tp::count_reduction();
    return TP_OK;
  }
  using tp::seqpar::check_slices;
  if ((st = check_slices(L.p, L.tokens, const_cast<void* const*>(x_slices), "x_slices")) != TP_OK ||
      (st = check_slices(L.p, L.tokens, y_slices, "y_slices")) != TP_OK)
    return st;
  if (residual_slices && (st = check_slices(L.p, L.tokens, residual_slices, "residual_slices")) != TP_OK)
    return st;
  if (y_norm_slices && (st = check_slices(L.p, L.tokens, y_norm_slices, "y_norm_slices")) != TP_OK)
    return st;
  if (!wqkv_p || !wo_p) return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (L.kv_len > 0 && (!k_cache || !v_cache))
    return tp::set_error(TP_ERR_INVALID_ARG, "decode needs k_cache and v_cache");
  if (L.kv_len > 0 && ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15))
    return tp::set_error(TP_ERR_INVALID_ARG, "k_cache and v_cache must be 16-byte aligned");
  if (!workspace) return tp::set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < sp_act_bytes(L) + L.ws_bytes) return tp::set_error(TP_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* x = workspace;
  void* ws = static_cast<uint8_t*>(workspace) + sp_act_bytes(L);
  st = tp::seqpar::all_gather(x_slices, L.p,
                              (L.tokens / L.p) * L.h * tp::elem_bytes(L.dtype), x, s);
  if (st != TP_OK) return st;
  const tp::seqpar::SpOut sp{residual_slices, y_slices, y_norm_slices};
  st = tp::attn_forward(L, x, wqkv_p, wo_p, k_cache, v_cache, nullptr, nullptr, nullptr, ws, s, &sp);
  if (st == TP_OK) tp::count_reduction();
  return st;
}

// ------------------------------------------------------------------------------------ backward
#include "attn_bwd.cuh"

namespace {
tp_status attn_bwd_check(const tp_attn_desc* desc, tp::AttnLayout* L) {
  tp_status st = tp::attn_layout_of(desc, L);
  if (st != TP_OK) return st;
  if (L->kv_len != 0) return tp::set_error(TP_ERR_UNSUPPORTED, "backward is for self-attention (kv_len == 0)");
  if (!L->tc) return tp::set_error(TP_ERR_UNSUPPORTED, "backward needs bf16 with h a multiple of 8");
  if (L->hd > 256) return tp::set_error(TP_ERR_UNSUPPORTED, "backward needs head_dim <= 256");
  if (desc->flags != 0) return tp::set_error(TP_ERR_UNSUPPORTED, "backward takes no flags");
  return TP_OK;
}
}  // namespace

extern "C" size_t tp_attn_bwd_workspace(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  if (attn_bwd_check(desc, &L) != TP_OK) return 0;
  return tp::attn_bwd_layout(L).bytes;
}

extern "C" tp_status tp_attn_bwd(const tp_attn_desc* desc, const void* x, const void* wqkv_p,
                                 const void* wo_p, const void* dy, void* dx, void* dwqkv_p,
                                 void* dwo_p, void* workspace, size_t ws_bytes, void* stream) {
  tp::clear_error();
  tp::AttnLayout L;
  tp_status st = attn_bwd_check(desc, &L);
  if (st != TP_OK) return st;
  if (L.tokens == 0) {
    tp::count_reduction();
    return TP_OK;
  }
  if (!x || !wqkv_p || !wo_p || !dy || !dx || !dwqkv_p || !dwo_p || !workspace)
    return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  for (const void* q : {x, wqkv_p, wo_p, dy, static_cast<const void*>(dx),
                        static_cast<const void*>(dwqkv_p), static_cast<const void*>(dwo_p)})
    if (reinterpret_cast<uintptr_t>(q) & 15)
      return tp::set_error(TP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const tp::AttnBwdLayout B = tp::attn_bwd_layout(L);
  if (ws_bytes < B.bytes) return tp::set_error(TP_ERR_WORKSPACE, "workspace too small");
  if (!tp::tensor_cores_usable())
    return tp::set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
  st = tp::attn_backward(L, x, wqkv_p, wo_p, dy, dx, static_cast<float*>(dwqkv_p),
                         static_cast<float*>(dwo_p), workspace, static_cast<cudaStream_t>(stream));
  if (st == TP_OK) tp::count_reduction();
  return st;
}

// Sequence-parallel backward: x and dy arrive as the p shards' token slices and are all-gathered
// (the reduce-scatter's gradient is an all-gather); the dx partials are reduce-scattered into the
// slices (the all-gather's gradient).  "Why tensor parallelism has to stay in scale-up",
// "Where the 320 comes from".
extern "C" size_t tp_attn_bwd_sp_workspace(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  if (attn_bwd_check(desc, &L) != TP_OK || sp_layout(desc, &L) != TP_OK) return 0;
  return 2 * sp_act_bytes(L) + tp::attn_bwd_layout(L).bytes;
}

extern "C" tp_status tp_attn_bwd_sp(const tp_attn_desc* desc, const void* const* x_slices,
                                    const void* wqkv_p, const void* wo_p,
                                    const void* const* dy_slices, void* const* dx_slices,
                                    void* dwqkv_p, void* dwo_p, void* workspace, size_t ws_bytes,
                                    void* stream) {
  tp::clear_error();
  tp::AttnLayout L;
  tp_status st = attn_bwd_check(desc, &L);
  if (st != TP_OK) return st;
  if ((st = sp_layout(desc, &L)) != TP_OK) return st;
  if (L.tokens == 0) {
    tp::count_reduction();
    return TP_OK;
  }
  using tp::seqpar::check_slices;
  if ((st = check_slices(L.p, L.tokens, const_cast<void* const*>(x_slices), "x_slices")) != TP_OK ||
      (st = check_slices(L.p, L.tokens, const_cast<void* const*>(dy_slices), "dy_slices")) != TP_OK ||
      (st = check_slices(L.p, L.tokens, dx_slices, "dx_slices")) != TP_OK)
    return st;
  if (!wqkv_p || !wo_p || !dwqkv_p || !dwo_p || !workspace)
    return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  for (const void* q : {wqkv_p, wo_p, static_cast<const void*>(dwqkv_p),
                        static_cast<const void*>(dwo_p), static_cast<const void*>(workspace)})
    if (reinterpret_cast<uintptr_t>(q) & 15)
      return tp::set_error(TP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t act = sp_act_bytes(L);
  const tp::AttnBwdLayout B = tp::attn_bwd_layout(L);
  if (ws_bytes < 2 * act + B.bytes) return tp::set_error(TP_ERR_WORKSPACE, "workspace too small");
  if (!tp::tensor_cores_usable())
    return tp::set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  void* x = w;
  void* dy = w + act;
  const int64_t slice_bytes = (L.tokens / L.p) * L.h * tp::elem_bytes(L.dtype);
  if ((st = tp::seqpar::all_gather(x_slices, L.p, slice_bytes, x, s)) != TP_OK) return st;
  if ((st = tp::seqpar::all_gather(dy_slices, L.p, slice_bytes, dy, s)) != TP_OK) return st;
  const tp::seqpar::SpOut sp{nullptr, dx_slices, nullptr};
  st = tp::attn_backward(L, x, wqkv_p, wo_p, dy, nullptr, static_cast<float*>(dwqkv_p),
                         static_cast<float*>(dwo_p), w + 2 * act, s, &sp);
  if (st == TP_OK) tp::count_reduction();
  return st;
}

extern "C" tp_status tp_attn_unpack_grads(const tp_attn_desc* desc, const void* dwqkv_p,
                                          const void* dwo_p, void* dwq, void* dwk, void* dwv,
                                          void* dwo, void* stream) {
  tp::clear_error();
  tp::AttnLayout L;
  tp_status st = tp::attn_layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (!dwqkv_p || !dwo_p || !dwq || !dwk || !dwv || !dwo)
    return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  return tp::attn_unpack_grads(L, static_cast<const float*>(dwqkv_p),
                               static_cast<const float*>(dwo_p), static_cast<float*>(dwq),
                               static_cast<float*>(dwk), static_cast<float*>(dwv),
                               static_cast<float*>(dwo), static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------------ one shard per device
// "Tensor Parallelism" (klaylearn), Notes: with one shard per GPU, device i owns n_q/p query heads
// and n_kv/p KV heads (its column slices of Wq, Wk, Wv and its KV cache), runs attention over
// them locally, and turns its heads' output into a full-width partial through its row slice of
// Wo; the devices' all-reduce adds the partials.  Shard i on its own is the block with p = 1 and
// n_q/p, n_kv/p heads, whose packed layout is exactly shard i's slice of the p-shard packing;
// these calls run that problem and leave the sum to the caller's collective (nothing is added to
// the reduction counter).
namespace {
tp_status attn_shard_desc(const tp_attn_desc* desc, int32_t shard, int32_t partial_dtype,
                          tp_attn_desc* sd, tp::AttnLayout* LS) {
  tp::AttnLayout L;
  tp_status st = tp::attn_layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (shard < 0 || shard >= L.p) return tp::set_error(TP_ERR_INVALID_ARG, "shard must be in 0 .. p-1");
  if (partial_dtype != TP_F32 && partial_dtype != TP_BF16)
    return tp::set_error(TP_ERR_INVALID_ARG, "partial_dtype must be TP_F32 or TP_BF16");
  if (L.dtype == TP_F32 && partial_dtype != TP_F32)
    return tp::set_error(TP_ERR_UNSUPPORTED, "fp32 blocks give fp32 partials");
  if (desc->flags != 0)
    return tp::set_error(TP_ERR_INVALID_ARG, "shard calls take no flags (partial_dtype sets the type)");
  *sd = *desc;
  sd->n_q = desc->n_q / desc->p;
  sd->n_kv = desc->n_kv / desc->p;
  sd->p = 1;
  sd->flags = (L.dtype == TP_BF16 && partial_dtype == TP_F32) ? TP_FLAG_F32_RESIDUAL : 0;
  sd->reduce_mode = L.tc ? TP_REDUCE_FUSED : TP_REDUCE_SEPARATE;
  return tp::attn_layout_of(sd, LS);
}
}  // namespace

extern "C" tp_status tp_attn_shard_sizes(const tp_attn_desc* desc, int32_t partial_dtype,
                                         tp_shard_sizes* out) {
  tp::clear_error();
  if (!out) return tp::set_error(TP_ERR_INVALID_ARG, "out is null");
  tp_attn_desc sd;
  tp::AttnLayout L;
  tp_status st = attn_shard_desc(desc, 0, partial_dtype, &sd, &L);
  if (st != TP_OK) return st;
  out->col_weight_bytes = L.wqkv_bytes;
  out->row_weight_bytes = L.wo_bytes;
  out->saved_bytes = 0;
  out->fwd_workspace = L.ws_bytes;
  tp::AttnLayout LB;
  const bool bwd_ok = partial_dtype == TP_BF16 && attn_bwd_check(&sd, &LB) == TP_OK;
  tp::clear_error();
  out->bwd_workspace = bwd_ok ? tp::attn_bwd_layout(LB).bytes : 0;
  out->partial_bytes = static_cast<size_t>(L.tokens * L.h) * tp::elem_bytes(partial_dtype);
  return TP_OK;
}

extern "C" tp_status tp_attn_pack_shard(const tp_attn_desc* desc, int32_t shard, const void* wq,
                                        const void* wk, const void* wv, const void* wo,
                                        void* wqkv_shard, void* wo_shard, void* stream) {
  tp::clear_error();
  tp_attn_desc sd;
  tp::AttnLayout L;
  tp_status st = attn_shard_desc(desc, shard, desc ? desc->dtype : TP_F32, &sd, &L);
  if (st != TP_OK) return st;
  if (!wq || !wk || !wv || !wo || !wqkv_shard || !wo_shard)
    return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  const size_t eb = static_cast<size_t>(L.eb);
  const int64_t qcols = static_cast<int64_t>(L.n_q) * L.hd;    // this shard's Wq columns
  const int64_t kcols = static_cast<int64_t>(L.n_kv) * L.hd;
  const int64_t q0 = static_cast<int64_t>(shard) * qcols, k0 = static_cast<int64_t>(shard) * kcols;
  return tp::attn_pack(L, static_cast<const uint8_t*>(wq) + q0 * eb,
                       static_cast<const uint8_t*>(wk) + k0 * eb,
                       static_cast<const uint8_t*>(wv) + k0 * eb,
                       static_cast<const uint8_t*>(wo) + q0 * L.h * eb, wqkv_shard, wo_shard,
                       static_cast<cudaStream_t>(stream), static_cast<int64_t>(desc->n_q) * L.hd,
                       static_cast<int64_t>(desc->n_kv) * L.hd);
}

extern "C" tp_status tp_attn_fwd_shard(const tp_attn_desc* desc, int32_t shard,
                                       int32_t partial_dtype, const void* x,
                                       const void* wqkv_shard, const void* wo_shard,
                                       void* k_cache_shard, void* v_cache_shard, void* partial,
                                       void* workspace, size_t ws_bytes, void* stream) {
  tp::clear_error();
  tp_attn_desc sd;
  tp::AttnLayout L;
  tp_status st = attn_shard_desc(desc, shard, partial_dtype, &sd, &L);
  if (st != TP_OK) return st;
  if (L.tokens == 0) return TP_OK;
  if (!x || !wqkv_shard || !wo_shard || !partial) return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (L.kv_len > 0 && (!k_cache_shard || !v_cache_shard))
    return tp::set_error(TP_ERR_INVALID_ARG, "decode needs k_cache and v_cache");
  if (L.kv_len > 0 &&
      ((reinterpret_cast<uintptr_t>(k_cache_shard) | reinterpret_cast<uintptr_t>(v_cache_shard)) & 15))
    return tp::set_error(TP_ERR_INVALID_ARG, "k_cache and v_cache must be 16-byte aligned");
  if (!workspace) return tp::set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < L.ws_bytes) return tp::set_error(TP_ERR_WORKSPACE, "workspace too small");
  return tp::attn_forward(L, x, wqkv_shard, wo_shard, k_cache_shard, v_cache_shard, nullptr,
                          partial, nullptr, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" tp_status tp_attn_bwd_shard(const tp_attn_desc* desc, int32_t shard, const void* x,
                                       const void* wqkv_shard, const void* wo_shard,
                                       const void* dy, void* dx_partial, void* dwqkv_shard,
                                       void* dwo_shard, void* workspace, size_t ws_bytes,
                                       void* stream) {
  tp::clear_error();
  tp_attn_desc sd;
  tp::AttnLayout L0;
  tp_status st = attn_shard_desc(desc, shard, TP_BF16, &sd, &L0);
  if (st != TP_OK) return st;
  tp::AttnLayout L;
  if ((st = attn_bwd_check(&sd, &L)) != TP_OK) return st;
  if (L.tokens == 0) return TP_OK;
  if (!x || !wqkv_shard || !wo_shard || !dy || !dx_partial || !dwqkv_shard || !dwo_shard || !workspace)
    return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  for (const void* q : {x, wqkv_shard, wo_shard, dy, static_cast<const void*>(dx_partial),
                        static_cast<const void*>(dwqkv_shard), static_cast<const void*>(dwo_shard)})
    if (reinterpret_cast<uintptr_t>(q) & 15)
      return tp::set_error(TP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const tp::AttnBwdLayout B = tp::attn_bwd_layout(L);
  if (ws_bytes < B.bytes) return tp::set_error(TP_ERR_WORKSPACE, "workspace too small");
  if (!tp::tensor_cores_usable())
    return tp::set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
  return tp::attn_backward(L, x, wqkv_shard, wo_shard, dy, dx_partial,
                           static_cast<float*>(dwqkv_shard), static_cast<float*>(dwo_shard),
                           workspace, static_cast<cudaStream_t>(stream));
}
