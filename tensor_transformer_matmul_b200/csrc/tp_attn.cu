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
